"""The Python example in README.md uses only names the binding exports, with
keyword arguments its functions accept (checked without a GPU: the example
itself runs on one)."""
import ast
import inspect
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fp8():
    import fp8_delayed_scaling_03_b200 as m
    return m


def test_readme_example_matches_binding(fp8):
    text = open(os.path.join(ROOT, "README.md")).read()
    blocks = re.findall(r"```python\n(.*?)```", text, re.S)
    assert blocks, "README has no Python example"
    tree = ast.parse(blocks[0])
    calls = 0
    for node in ast.walk(tree):
        if isinstance(node, ast.Attribute) and isinstance(node.value, ast.Name) and node.value.id == "F":
            assert hasattr(fp8, node.attr), node.attr
        if isinstance(node, ast.Call) and isinstance(node.func, ast.Attribute) and \
                isinstance(node.func.value, ast.Name) and node.func.value.id == "F":
            params = inspect.signature(getattr(fp8, node.func.attr)).parameters
            for kw in node.keywords:
                assert kw.arg in params, (node.func.attr, kw.arg)
            calls += 1
    assert calls >= 4
