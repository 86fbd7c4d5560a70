"""The benchmark's per-op work model (algorithmic bytes and flops behind every roofline figure),
checked against plain counts on CPU: the op list follows the layer's launch order, the recompute
variant adds exactly one GEMM1 and drops the h13 store from the forward one, and the MXFP8 step's
activations leave their producers quantised."""
import bench
from moe_workloads import WORKLOADS


def test_bf16_op_order_is_the_launch_order():
    w = WORKLOADS["e128_bf16"]
    assert list(bench.op_work(w)) == [
        "route_metadata", "dispatch", "gemm_fwd1_swiglu", "gemm_fwd2", "combine", "combine_bwd",
        "gemm_dgrad2_swiglu", "gemm_dgrad1", "token_reduce", "gemm_wgrad2", "gemm_wgrad1"]


def test_recompute_adds_one_gemm1_and_drops_the_h13_store():
    w = WORKLOADS["e128_bf16"]
    R, d, F, E = w.T * w.k, w.d, w.F, w.E
    st, rc = bench.op_work(w), bench.op_work(w, recompute=True)
    names = list(rc)
    assert names.index("gemm_fwd1_recompute") == names.index("combine_bwd") + 1
    assert names.index("gemm_dgrad2_swiglu") == names.index("gemm_fwd1_recompute") + 1
    assert rc["gemm_fwd1_recompute"] == st["gemm_fwd1_swiglu"]
    assert st["gemm_fwd1_swiglu"][0] - rc["gemm_fwd1_swiglu"][0] == R * 2 * F * 2
    assert rc["gemm_fwd1_swiglu"][1] == st["gemm_fwd1_swiglu"][1] == 2 * R * d * 2 * F
    # every other op is unchanged
    for n in st:
        if n != "gemm_fwd1_swiglu":
            assert rc[n] == st[n], n
    # GEMM1 stored: x_perm and W13 read, h13 and a written, all bf16
    assert st["gemm_fwd1_swiglu"][0] == (R * d + E * 2 * F * d + R * 2 * F + R * F) * 2


def test_total_flops_are_the_layer_count():
    """Six expert GEMMs: 3 forward-equivalents of 2 R d (3F) flops (GEMM1 2F wide, GEMM2 F)."""
    w = WORKLOADS["e128_bf16"]
    R = w.T * w.k
    gemm = sum(f for n, (b, f) in bench.op_work(w).items() if n.startswith("gemm_"))
    assert gemm == 3 * 2 * R * w.d * 3 * w.F


def test_mxfp8_activations_leave_their_producers_quantised():
    """MXFP8 step: no separate quantisation launch. Each routed activation is written only as its two
    quantised forms (codes + 1/32 scale bytes each) by the kernel that produces it, which reads its bf16
    inputs once; the op list is the fused layer's launch order."""
    w = WORKLOADS["e128_mxfp8"]
    T, R, d, F, E, k = w.T, w.T * w.k, w.d, w.F, w.E, w.k
    ops = bench.op_work(w)
    q = lambda n: n + n // 32
    assert list(ops) == [
        "route_metadata", "dispatch_quant", "gemm_fwd1_swiglu_quant", "gemm_fwd2", "combine",
        "combine_bwd_quant", "gemm_dgrad2_swiglu_quant", "gemm_wgrad2", "gemm_dgrad1", "gemm_wgrad1",
        "token_reduce"]
    assert not any(n.startswith("quant_") for n in ops)
    assert ops["dispatch_quant"] == (T * d * 2 + R * 4 + 2 * q(R * d), 0)
    # GEMM1: fp8 x_perm and W13 read, bf16 h13 written, a written as two quantised forms
    assert ops["gemm_fwd1_swiglu_quant"][0] == q(R * d) + q(E * 2 * F * d) + R * 2 * F * 2 + 2 * q(R * F)
    assert ops["combine_bwd_quant"][0] == (T * d + R * d) * 2 + T * k * 8 + R * 4 + 2 * q(R * d)
    assert ops["gemm_dgrad2_swiglu_quant"][0] == q(R * d) + q(E * d * F) + R * 2 * F * 2 + 2 * q(R * 2 * F)


class _FakeNvml:
    """Enough of NVML for the bench's clock sampler: a fixed max clock, a clock sequence and the
    throttle-reason bits (the values NVML defines)."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonSwPowerCap = 0x4

    class NVMLError(Exception):
        pass

    def __init__(self, clocks, reasons):
        self.clocks, self.reasons, self.i = clocks, reasons, 0

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        self.i += 1
        return self.clocks[self.i % len(self.clocks)]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.reasons

    def nvmlShutdown(self):
        pass


def test_clock_sampler_reads_clocks_and_reasons_from_nvml():
    import time
    fake = _FakeNvml([1965, 1950, 120], 0x4 | 0x1)  # sw_power_cap, plus an idle bit that is not reported
    cs = bench.ClockSampler(0)
    cs._nvml_handle = lambda: (fake, object())
    cs.start()
    time.sleep(0.12)
    out = cs.stop()
    assert out["samples"] >= 3 and out["source"].startswith("nvml")
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]
    # the idle 120 MHz samples are dropped before the median
    assert out["sm_mhz"] in (1950.0, 1957.5, 1965.0)
    fake2 = _FakeNvml([1965], 0x0)
    cs2 = bench.ClockSampler(0)
    cs2._nvml_handle = lambda: (fake2, object())
    cs2.start()
    time.sleep(0.02)
    assert cs2.stop()["reasons"] == []
