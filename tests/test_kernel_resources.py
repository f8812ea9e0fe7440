"""Per-thread registers, spills and static shared memory of the kernels, as
ptxas reports them for sm_100a (nvcc only, no GPU).

The step overlaps each quantize grid with the tail of the GEMM before it
(programmatic dependent launch): a 256-thread quantize block becomes resident
beside a still-running GEMM CTA only while both fit one SM together -- 320
GEMM threads x R registers + 256 x 64 <= 65536, i.e. R <= 128, and the
quantize block's static shared memory next to the GEMM's 225 KB.  An epilogue
variant once raised the data-parallel GEMM builds to 161-168 registers
without any spill and so, silently, took that overlap away; these checks pin
the budget."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def ptxas_report(src):
    from fp8_delayed_scaling_03_b200 import build as B
    if not shutil.which(B.NVCC) and not os.path.exists(B.NVCC):
        pytest.skip("no nvcc")
    out = os.path.join(B.BUILD, os.path.basename(src) + ".resources.o")
    os.makedirs(B.BUILD, exist_ok=True)
    r = subprocess.run([B.NVCC, *B.ARCH, *B.FLAGS, "-Xptxas", "-v", "-c", os.path.join(B.CSRC, src), "-o", out],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    kernels, name = {}, None
    for line in (r.stdout + r.stderr).splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            name = m.group(1)
            kernels[name] = {"regs": None, "spill": 0, "smem": 0}
            continue
        if name is None:
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m:
            kernels[name]["spill"] = int(m.group(1)) + int(m.group(2))
        m = re.search(r"Used (\d+) registers", line)
        if m:
            kernels[name]["regs"] = int(m.group(1))
            s = re.search(r"(\d+) bytes smem", line)
            kernels[name]["smem"] = int(s.group(1)) if s else 0
    assert kernels and all(k["regs"] is not None for k in kernels.values()), r.stderr
    return kernels


@pytest.fixture(scope="module")
def gemm():
    return ptxas_report("gemm.cu")


@pytest.fixture(scope="module")
def quant():
    return ptxas_report("quantize.cu")


def gemm_builds(kernels):
    """(BN, pair, split, stream-K) -> resources, from the mangled template arguments."""
    out = {}
    for name, res in kernels.items():
        m = re.search(r"fp8_gemm_kernelILi(\d+)ELb([01])ELb([01])ELb([01])E", name)
        if m:
            out[(int(m.group(1)), m.group(2) == "1", m.group(3) == "1", m.group(4) == "1")] = res
    return out


def test_spills(gemm, quant):
    """No GEMM build spills.  The flat quantize and amax builds for 2-byte
    inputs (both prefetch their input into L2 before the dependency wait)
    keep a small stack slot at their 64-register cap, at most 28 bytes of
    spill traffic (12 stored, 16 loaded), no more."""
    for name, res in gemm.items():
        assert res["spill"] == 0, (name, res)
    for name, res in quant.items():
        two_byte = "__half" in name or "bfloat16" in name
        allowed = 28 if two_byte and ("15quantize_kernelI" in name or "11amax_kernelI" in name) else 0
        assert res["spill"] <= allowed, (name, res)


def test_data_parallel_gemm_fits_beside_a_quantize_block(gemm):
    builds = gemm_builds(gemm)
    dp = {k: v for k, v in builds.items() if not k[2] and not k[3]}
    assert set(dp) == {(128, False, False, False), (256, False, False, False), (256, True, False, False)}
    for cfg, res in dp.items():
        assert res["regs"] <= 128, (cfg, res)
        assert 320 * 128 + 256 * 64 <= 65536


def test_flat_quantize_block_budget(quant):
    flat = {n: r for n, r in quant.items() if "quantize_kernel" in n and "colsum" not in n}
    assert len(flat) == 6  # {bf16, fp16, fp32} x {E4M3, E5M2}
    for name, res in flat.items():
        assert res["regs"] <= 64 and res["smem"] <= 1024, (name, res)
