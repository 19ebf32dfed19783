"""Host-side helpers of the benchmark, on the CPU: the packed input buffer of the end-to-end arm and the
algorithmic byte counts behind the roofline fraction."""

import numpy as np
import torch

import bench
from kv_cache_quantized_b200 import workloads as W


def test_packed_inputs_views_hold_the_tensors():
    q = torch.randn(8, 32, 128)
    k = torch.randn(8, 8, 128).half()
    v = torch.randn(8, 8, 128).half()
    buf, (qv, kv, vv) = bench._packed_inputs([q, k, v])
    assert buf.dtype == torch.uint8
    assert buf.numel() == q.numel() * 4 + k.numel() * 2 + v.numel() * 2  # offsets already 16-byte multiples
    for view, t in ((qv, q), (kv, k), (vv, v)):
        assert view.dtype == t.dtype and view.shape == t.shape and view.is_contiguous()
        assert view.data_ptr() % 16 == 0
        assert torch.equal(view, t)
    # one copy into the buffer refreshes every view
    buf2, views2 = bench._packed_inputs([torch.zeros_like(q), torch.zeros_like(k), torch.zeros_like(v)])
    buf2.copy_(buf)
    assert all(torch.equal(a, b) for a, b in zip(views2, (q, k, v)))


def test_packed_inputs_pads_odd_sizes_to_16_bytes():
    a = torch.arange(3, dtype=torch.float16)   # 6 bytes
    b = torch.arange(5, dtype=torch.float32)   # 20 bytes, starts at 16
    buf, (av, bv) = bench._packed_inputs([a, b])
    assert buf.numel() == 16 + 20
    assert bv.data_ptr() - buf.data_ptr() == 16
    assert torch.equal(av, a) and torch.equal(bv, b)


def test_algorithmic_bytes_per_key_head():
    # long context: 64 B key codes + 2 B norm, and the same for quantized values
    assert bench._bytes_per_key_head(W.LONG_CONTEXT) == 132
    # Llama-shaped: 66 B of key codes and norm + 256 B of fp16 values
    assert bench._bytes_per_key_head(W.LLAMA8B_DECODE) == 322
    w = W.LONG_CONTEXT
    units = w.B * w.Hkv * w.T
    assert units * bench._bytes_per_key_head(w) == 276_824_064
    # the measured DRAM traffic of the decode kernel (when the bench carries a figure for this kernel version) is
    # the algorithmic bytes plus the partials and the new tokens' writes: at least the algorithmic bytes, and no
    # re-reads beyond a percent or two
    if w.name in bench.TRAFFIC:
        ratio = bench.TRAFFIC[w.name] / (units * bench._bytes_per_key_head(w))
        assert 1.0 <= ratio <= 1.02, ratio


def test_step_kernel_label_follows_the_library_routing():
    """The bench line names the decode kernel the library picks for a contiguous step: the streaming kernel for the
    long-context step and for fp16 values, the row kernel for small problems with quantized values."""
    import dataclasses
    assert bench._step_kernel(W.LONG_CONTEXT) == "attend_stream_kernel"
    assert bench._step_kernel(W.LLAMA8B_DECODE) == "attend_stream_kernel"
    assert bench._step_kernel(dataclasses.replace(W.LONG_CONTEXT, B=1, T=4096)) == "attend_rows_kernel"
    assert bench._step_kernel(dataclasses.replace(W.LONG_CONTEXT, B=1, T=4096, Hq=64)) == "attend_stream_kernel"


class _FakeNvml:
    """The NVML calls the clock sampler makes, answering fixed readings (no GPU, no driver)."""
    NVML_CLOCK_SM = 1
    nvmlClocksThrottleReasonSwPowerCap = 0x4
    nvmlClocksThrottleReasonHwSlowdown = 0x8
    nvmlClocksThrottleReasonSwThermalSlowdown = 0x20
    nvmlClocksThrottleReasonHwThermalSlowdown = 0x40

    def __init__(self, sm, reasons):
        self.sm, self.reasons = sm, reasons

    def nvmlDeviceGetClockInfo(self, h, kind):
        return self.sm

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetPowerUsage(self, h):
        return 812_500  # mW

    def nvmlDeviceGetCurrentClocksThrottleReasons(self, h):
        return self.reasons


def test_clock_sampler_reads_nvml_samples_into_the_summary():
    """NVML readings become nvidia-smi-style CSV samples: the summary takes the median SM clock, the maximum and the
    throttle reasons seen (sw_power_cap is reported, an idle reason is not)."""
    c = bench.ClockSampler(0)
    c.lines.append(c._nvml_line(_FakeNvml(1965, 0x0), None))
    c.lines.append(c._nvml_line(_FakeNvml(1890, 0x4), None))
    c.lines.append(c._nvml_line(_FakeNvml(1950, 0x1), None))
    assert c.lines[0].split(", ")[1:4] == ["1965", "1965", "812.50"]
    s = c.summary()
    assert s == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    c2 = bench.ClockSampler(0)
    c2.lines.append(c2._nvml_line(_FakeNvml(1200, 0x8 | 0x40), None))
    assert c2.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]
