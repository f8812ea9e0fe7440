"""bench.py's end-to-end timing harness, host logic only: CUDA streams,
events and the C-ABI calls are replaced by recorders, and the test checks the
order the harness imposes -- each linear's forward waits for that linear's
input copies, each output copy waits for the kernel that wrote it, a step's
input copies wait for the previous step's kernels and a step's kernels for
the previous step's output copies -- and that every byte is copied in and
out."""
import contextlib
import ctypes

import torch

import bench


def test_e2e_harness_orders_copies_and_kernels(monkeypatch):
    ops = []            # (stream name, op, payload) in issue order
    records = {}        # event id -> index in ops of its record
    current = {"s": None}

    class Stream:
        count = 0

        def __init__(self, *a):
            Stream.count += 1
            self.name = f"s{Stream.count}"
            self.cuda_stream = Stream.count

        def wait_event(self, e):
            assert e.id in records, "waiting on an event that was never recorded"
            ops.append((self.name, "wait", e.id))

    class Event:
        n = 0

        def __init__(self, enable_timing=False):
            Event.n += 1
            self.id = Event.n

        def record(self, s):
            records[self.id] = len(ops)
            ops.append((s.name, "record", self.id))

        def elapsed_time(self, other):
            return 2.0

    @contextlib.contextmanager
    def stream_ctx(s):
        prev, current["s"] = current["s"], s
        try:
            yield
        finally:
            current["s"] = prev

    real_copy = torch.Tensor.copy_

    def copy_(self, src, non_blocking=False):
        ops.append((current["s"].name, "copy", id(self)))
        return real_copy(self, src)

    monkeypatch.setattr(torch.cuda, "Stream", Stream)
    monkeypatch.setattr(torch.cuda, "Event", Event)
    monkeypatch.setattr(torch.cuda, "stream", stream_ctx)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a: None)
    monkeypatch.setattr(torch.Tensor, "copy_", copy_)

    class Lib:
        def fp8_linear_forward(self, args, h):
            ops.append((f"s{h}", "fwd", args._obj.value))
            return 0

        def fp8_linear_backward(self, args, h):
            ops.append((f"s{h}", "bwd", args._obj.value - 100))
            return 0

    class F:
        _lib = Lib()

        class Fp8Error(RuntimeError):
            def __init__(self, status, where):
                super().__init__(where)

    class Lin:
        def __init__(self, i):
            self.i = i
            self.x, self.w, self.b, self.g = (torch.zeros(3) for _ in range(4))
            self.y, self.dx, self.dw, self.db = (torch.full((3,), float(i + 1)) for _ in range(4))
            self.fwd, self.bwd = ctypes.c_int(i), ctypes.c_int(100 + i)

        def inputs(self):
            return [self.x, self.w, self.b, self.g]

        def outputs(self):
            return [self.y, self.dx, self.dw, self.db]

    n, steps = 3, 2
    lins = [Lin(i) for i in range(n)]
    host_in = [[torch.full((3,), 7.0) for _ in range(4)] for _ in range(n)]
    host_out = [[torch.zeros(3) for _ in range(4)] for _ in range(n)]
    comp = Stream()                                  # s1; the harness makes s2 (in) and s3 (out)
    assert bench.time_e2e(F, lins, host_in, host_out, comp, None, steps) == 2.0
    assert all(bool((t == 7).all()) for L in lins for t in L.inputs())
    assert all(bool((h == L.i + 1).all()) for L, hs in zip(lins, host_out) for h in hs)

    def last_wait_before(k, stream):
        w = [o for o in ops[:k] if o[0] == stream and o[1] == "wait"]
        assert w, f"no wait on {stream} before op {k}"
        return records[w[-1][2]]                     # index of the awaited record

    fwd = [k for k, o in enumerate(ops) if o[1] == "fwd"]
    bwd = [k for k, o in enumerate(ops) if o[1] == "bwd"]
    assert len(fwd) == len(bwd) == n * (steps + 1)   # warm-up step + timed steps
    assert all(ops[k][0] == "s1" for k in fwd + bwd)
    # forward i waits for the event recorded on the input stream right after
    # linear i's last input copy (g)
    for k in fwd:
        r = last_wait_before(k, "s1")
        assert ops[r][0] == "s2" and ops[r - 1] == ("s2", "copy", id(lins[ops[k][2]].g))
    # input copies only on s2, output copies only on s3
    dev_in = {id(t) for L in lins for t in L.inputs()}
    host_o = {id(h): (i, j) for i, hs in enumerate(host_out) for j, h in enumerate(hs)}
    for k, o in enumerate(ops):
        if o[1] != "copy":
            continue
        assert (o[0], o[2] in dev_in) in (("s2", True), ("s3", False))
        if o[0] == "s3":
            # waits for the event recorded right after the kernel that wrote it
            i, j = host_o[o[2]]
            r = last_wait_before(k, "s3")
            assert ops[r][0] == "s1" and ops[r - 1] == ("s1", "fwd" if j == 0 else "bwd", i)
    # step boundaries
    h2d_waits = [k for k, o in enumerate(ops) if o[0] == "s2" and o[1] == "wait"]
    comp_step_waits = [k for k, o in enumerate(ops)
                       if o[0] == "s1" and o[1] == "wait" and ops[records[o[2]]][0] in ("s1", "s3")]
    # (the compute stream also joins the last step's output copies before the end event)
    assert len(h2d_waits) == steps and len(comp_step_waits) == steps + 1
    for k in h2d_waits:        # after every kernel issued so far (previous step's last backward, or e0)
        r = records[ops[k][2]]
        assert ops[r][0] == "s1" and all(j < r for j in fwd + bwd if j < k)
    for k in comp_step_waits:  # after every output copy issued so far
        r = records[ops[k][2]]
        copies_out = [j for j, o in enumerate(ops[:k]) if o[0] == "s3" and o[1] == "copy"]
        assert all(j < r for j in copies_out)


def test_fp8_peak_denominator_choice():
    """Burst bf16 x 2 while the timed region held the maximum clock with no
    power-cap reason; the sustained figure under the cap or a lowered clock."""
    import bench
    pk = {"bf16_tflops": 1644.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6551.0}
    assert bench.fp8_peak_for(pk, {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}) == (3288.0, "bf16_tflops")
    assert bench.fp8_peak_for(pk, {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}) == \
        (2800.0, "bf16_tflops_sustained")
    assert bench.fp8_peak_for(pk, {"sm_mhz": 1500, "sm_max_mhz": 1965, "reasons": []})[1] == "bf16_tflops_sustained"
    burst_only = {"bf16_tflops": 1644.0}
    assert bench.fp8_peak_for(burst_only, {"sm_mhz": 1500, "sm_max_mhz": 1965, "reasons": []}) == \
        (3288.0, "bf16_tflops")


def test_gemm_compulsory_bytes_and_operand_sets():
    import bench
    M, N, K = 2048, 6912, 1536
    assert bench.gemm_min_bytes("fwd", M, N, K) == M * K + N * K + 2 * M * N
    assert bench.gemm_min_bytes("fwd", M, N, K, bias_bytes=N) == M * K + N * K + 2 * M * N + N
    assert bench.gemm_min_bytes("dX", M, N, K) == M * N + N * K + 2 * M * K
    assert bench.gemm_min_bytes("dW", M, N, K) == M * N + M * K + 2 * N * K
    for per in (1, 10 << 20, 100 << 20, 1 << 30):
        n = bench._sets_for(per)
        assert 2 <= n <= 12 and (n * per >= (320 << 20) or n == 12)


def test_traffic_summary_is_tied_to_the_gemm_source(monkeypatch):
    """roofline.traffic comes from the committed ncu summary only while
    gemm.cu still has the hash recorded there."""
    import bench
    got = bench.gemm_traffic_per_launch("c4")
    if got is not None:
        assert got > 0
        monkeypatch.setattr(bench, "gemm_source_sha", lambda: "0000000000000000")
        assert bench.gemm_traffic_per_launch("c4") is None
    assert bench.gemm_traffic_per_launch("no-such-workload") is None


def test_clock_sampler_against_fake_nvml(monkeypatch):
    """The sampler reads the SM clock and the clock-event reason bits through
    NVML in a thread (reads only) and reports their median and the union of
    the reasons by name; without NVML it reports that instead of clocks."""
    import sys
    import time
    import types

    import bench

    clocks = iter([1965, 1965, 1800, 1965, 1700] + [1965] * 10000)
    reasons = iter([0, 0x4, 0, 0x4 | 0x40, 0] + [0] * 10000)
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=0,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByPciBusId=lambda bus: "h",
        nvmlDeviceGetHandleByIndex=lambda i: "h",
        nvmlDeviceGetMaxClockInfo=lambda h, c: 1965,
        nvmlDeviceGetClockInfo=lambda h, c: next(clocks),
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: next(reasons))
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    props = types.SimpleNamespace(pci_domain_id=0, pci_bus_id=0x1b, pci_device_id=0)
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties", lambda i: props)
    with bench.ClockSampler(0) as clk:
        t0 = time.time()
        while len(clk.samples) < 5 and time.time() - t0 < 5:
            time.sleep(0.01)
    r = clk.report()
    assert r["sm_max_mhz"] == 1965 and r["samples"] >= 5
    assert "sw_power_cap" in r["reasons"] and "hw_thermal_slowdown" in r["reasons"]
    assert set(r["reasons"]) <= set(bench.ClockSampler.REASONS.values())

    def broken():
        raise RuntimeError("no NVML here")
    monkeypatch.setattr(fake, "nvmlInit", broken)
    r = bench.ClockSampler(0).report()
    assert r["sm_mhz"] is None and r["reasons"] == [] and "no NVML" in r["error"]
