"""The bench's roofline arithmetic on CPU: the reported fraction is the
combined bound max(F / tensor peak, B / HBM peak) over the measured time,
with the sustained tensor peak when the kernel's own loop ran power-capped,
and the native MXFP4 path's quantised activations counted in B."""
import types

import pytest

import bench

PEAKS = {"bf16_tflops": 1656.8, "bf16_tflops_sustained": 1388.7, "hbm_gbs": 6520.2}


def _wl(native=False, M=32768, N=4096, K=7168, native_rows=1413):
    p = types.SimpleNamespace(N=N, K=K, name="gate_up")
    wl = types.SimpleNamespace(p1=p, M=M, dgrad=False, w4a8=False, a4=False, split=False, swiglu=False, decode=False,
                               native=native, native_rows=[native_rows], wl=types.SimpleNamespace(fmt="mxfp4"))
    wl.weight_bytes = lambda pp, hit: int(hit * pp.N * (pp.K // 2 + pp.K / 32))
    return wl


def _stats(capped):
    return {"clocks": {"sm_mhz": 1792.0 if capped else 1965.0, "sm_max_mhz": 1965.0,
                       "reasons": ["sw_power_cap"] if capped else []}}


@pytest.mark.parametrize("capped", [False, True])
@pytest.mark.parametrize("native", [False, True])
def test_roofline_is_the_combined_bound(capped, native):
    wl = _wl(native=native)
    M, N, K, hit, ms = wl.M, wl.p1.N, wl.p1.K, 133, 2.36
    r = bench.roofline(wl, None, PEAKS, "measured", ms, hit, _stats(capped), None)
    F = 2.0 * M * N * K
    B = hit * N * (K // 2 + K / 32) + 2 * M * K + 2 * M * N + (4 * 1413 * (K + K // 32) if native else 0)
    peak = PEAKS["bf16_tflops_sustained" if capped else "bf16_tflops"]
    t = ms / 1e3
    assert r["algorithmic_flops_per_launch"] == int(F)
    assert r["algorithmic_bytes_per_launch"] == int(B)
    assert r["frac"] == pytest.approx(max(F / (peak * 1e12), B / (PEAKS["hbm_gbs"] * 1e9)) / t, abs=1e-4)
    assert r["tensor"]["peak_measured"] == pytest.approx(peak, abs=0.05)
    assert r["bound"] == "tensor"  # this shape sits on the tensor side of the ridge
    nominal = max(F / (bench.NOMINAL["bf16"] * 1e12), B / (bench.NOMINAL["hbm_gbs"] * 1e9)) / t
    assert r["frac_nominal"] == pytest.approx(nominal, abs=1e-4)
    assert r["combined_bound_us"] == pytest.approx(max(F / (peak * 1e12), B / (PEAKS["hbm_gbs"] * 1e9)) * 1e6,
                                                   abs=1e-2)


def test_roofline_small_groups_are_hbm_bound():
    wl = _wl(M=2048, N=5760, K=2880, native_rows=2048, native=True)
    r = bench.roofline(wl, None, PEAKS, "measured", 0.423, 128, _stats(False), None)
    assert r["bound"] == "hbm"
    assert r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(r["algorithmic_bytes_per_launch"] / 0.423e-3 / 1e9, rel=1e-3)


def test_engagement_lists_the_called_entry_points_only():
    """The bench line's engagement object: one record per entry point called in the timed steps, zero fields
    dropped except `calls`, read from the library's own host-side counters."""
    import ctypes

    from bit_grouped_moe_b200 import build
    build.build()
    from bit_grouped_moe_b200 import gnf4 as g
    g.call_stats_get(None, reset=True)
    assert bench.engagement(g) == {}
    f = g._lib.gnf4_grouped_gemm_nf4
    f(None, None, None, ctypes.c_void_p(16), None, 0, 64, 64, 8, None, None)  # refused: E = 0
    f(None, None, None, ctypes.c_void_p(16), None, 4, 64, 64, 0, None, None)  # accepted, nothing to enqueue
    assert bench.engagement(g) == {"grouped_gemm_nf4": {"calls": 2, "refused": 1}}
    g.call_stats_get(None, reset=True)


def test_clock_sampler_names_the_gpu_by_uuid_and_falls_back_to_the_index(monkeypatch):
    """nvidia-smi numbers GPUs physically, CUDA after CUDA_VISIBLE_DEVICES: the sampler asks for the device's
    UUID, and takes the index only when nvidia-smi does not know that UUID (or is missing)."""
    import subprocess
    import types as _t

    seen = []

    def fake_run(cmd, **kw):
        seen.append(cmd)
        ok = cmd[2] == "GPU-1234-abcd"
        return _t.SimpleNamespace(returncode=0 if ok else 6, stdout="GPU-1234-abcd\n" if ok else "")

    monkeypatch.setattr(subprocess, "run", fake_run)
    assert bench.ClockSampler(3, "1234-abcd").gpu_id() == "GPU-1234-abcd"
    assert bench.ClockSampler(3, "GPU-1234-abcd").gpu_id() == "GPU-1234-abcd"
    assert bench.ClockSampler(3, "ffff").gpu_id() == "3"
    assert bench.ClockSampler(5, None).gpu_id() == "5"

    def missing(cmd, **kw):
        raise FileNotFoundError("nvidia-smi")

    monkeypatch.setattr(subprocess, "run", missing)
    assert bench.ClockSampler(2, "1234-abcd").gpu_id() == "2"
    s = bench.ClockSampler(0)
    assert s.summary(0.0, 1.0) == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "gpu": None}
