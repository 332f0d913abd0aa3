"""CPU checks of the measurement helpers: the algorithmic bytes that the roofline's
numerator uses, written out for the workloads from their shapes, and the clock summary
of nvidia-smi samples (median SM clock, throttle reasons seen inside the timed window)."""
import numpy as np

from rank_kv_cache_head_b200.metrics import ClockSampler, step_bytes
from rank_kv_cache_head_b200.workloads import WORKLOADS, seqlens_for


def test_step_bytes_of_the_vlm_workload():
    wl = WORKLOADS["vlm7b-bf16"]
    sb = step_bytes(wl, seqlens_for(wl))
    # 8 rows x 4096 tokens x 32 KV heads, K and V rows of 32 bf16 each
    assert sb["latent"] == 8 * 4096 * 32 * 2 * 32 * 2
    assert sb["scales"] == 0
    assert sb["factors"] == 2 * 32 * 32 * 128 * 2
    assert sb["q"] == sb["out"] == 8 * 32 * 128 * 2
    assert sb["split_kernel"] == sb["latent"] + sb["factors"] + sb["q"]
    assert sb["total"] == sb["split_kernel"] + sb["out"]
    assert sb["token_heads"] == 8 * 4096 * 32
    two = step_bytes(wl, seqlens_for(wl), factor_sets=2)
    assert two["factors"] == 2 * sb["factors"] and two["latent"] == sb["latent"]


def test_step_bytes_of_quantised_and_ragged_workloads():
    wl = WORKLOADS["quant-i8"]
    sb = step_bytes(wl, seqlens_for(wl))
    th = 32 * 8192 * 8
    assert sb["latent"] == th * 2 * 32 * 1 and sb["scales"] == th * 2 * 4
    wl = WORKLOADS["gqa-ragged-bf16"]
    lens = seqlens_for(wl)
    sb = step_bytes(wl, lens)
    assert sb["latent"] == int(np.sum(lens)) * 8 * 2 * 48 * 2


def _sample(t, mhz, reasons=("Not Active",) * 4):
    return (t, float(mhz), 1965.0, 700.0, "0x0", *reasons)


def test_clock_summary_median_and_reasons_inside_the_window():
    cs = ClockSampler(0)
    cs.samples = [_sample(0.0, 1000, ("Active", "Not Active", "Not Active", "Not Active"))]
    cs.samples += [_sample(1.0 + 0.1 * i, 1965 - i) for i in range(5)]
    cs.samples += [_sample(1.25, 1900, ("Not Active", "Not Active", "Not Active", "Active"))]
    s = cs.summary(0.5, 2.0)
    assert s["window"] == "timed" and s["samples"] == 6
    assert s["sm_mhz"] == float(np.median([1965, 1964, 1963, 1962, 1961, 1900]))
    assert s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]      # the hw_slowdown sample was outside


def test_clock_summary_without_samples():
    s = ClockSampler(0).summary(0.0, 1.0)
    assert s["sm_mhz"] is None and s["reasons"] == ["nvidia-smi unavailable"]
