"""Host-side logic of bench.py on the CPU: the nvidia-smi clock parser that
fills the line's `clocks` field, and the CPU-baseline leg's sampling of the
routing bank (the float64 oracle on a small bank)."""

import os
import tempfile

import numpy as np
import torch

import bench
import oracle


class _Done:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _clocks_from(lines):
    c = bench.Clocks.__new__(bench.Clocks)
    c.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
    c.f.write("\n".join(lines) + "\n")
    c.f.flush()
    c.p = _Done()
    return c


def test_clock_parser_median_max_and_reasons(monkeypatch):
    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    fields = "{sm}, 1965, 700.5, 0x0000000000000000, Not Active, Not Active, Not Active, {cap}"
    c = _clocks_from([fields.format(sm=1965, cap="Not Active"),
                      fields.format(sm=1800, cap="Active"),
                      fields.format(sm=1950, cap="Not Active"),
                      "garbage line",
                      "[N/A], 1965, 1, 0x0, Not Active, Not Active, Not Active, Not Active"])
    path = c.f.name
    got = c.stop()
    assert got["sm_mhz"] == 1950 and got["sm_max_mhz"] == 1965 and got["samples"] == 3
    assert got["reasons"] == ["sw_power_cap"]
    assert not os.path.exists(path)


def test_clock_parser_reports_hardware_slowdowns(monkeypatch):
    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    got = _clocks_from(["1400, 1965, 990, 0x8, Active, Not Active, Active, Active"]).stop()
    assert got["reasons"] == ["hw_slowdown", "sw_power_cap", "sw_thermal_slowdown"]


def test_clock_parser_without_nvidia_smi():
    c = bench.Clocks.__new__(bench.Clocks)
    c.p = None
    assert c.stop()["reasons"] == ["nvidia-smi unavailable"]


def _small_workload(n_docs=40, seed=3):
    g = torch.Generator().manual_seed(seed)
    lengths = torch.randint(64, 4000, (n_docs,), generator=g)
    coff_h = oracle.chunk_offsets_from_lengths(lengths.numpy())
    C = int(coff_h[-1])
    H, D, Hq, T = 2, 16, 4, 8
    bf = torch.bfloat16
    w = dict(q_r=torch.randn((1, T, H, D), generator=g).to(bf),
             kr_bar=torch.randn((C, H, D), generator=g).to(bf),
             k_bar=torch.randn((C, H, D), generator=g).to(bf),
             v_bar=torch.randn((C, H, D), generator=g).to(bf),
             q=torch.randn((1, T, Hq, D), generator=g).to(bf),
             k_loc=torch.randn((1, T, H, D), generator=g).to(bf),
             v_loc=torch.randn((1, T, H, D), generator=g).to(bf),
             k=4, pos0=4)

    class P:
        pass
    p = P()
    p.coff = torch.from_numpy(coff_h)
    p.n_docs = n_docs
    return w, p, C


def test_cpu_baseline_samples_slices_spread_over_the_bank():
    w, p, C = _small_workload()
    one = bench.cpu_baseline(w, p, C, route_seconds=0.0, slice_chunks=64)
    assert one["kind"] == "oracle" and one["value"] > 0 and one["cores"] >= 1
    assert one["sample"].startswith("routing timed on 1 slices of 64 chunks")
    full = bench.cpu_baseline(w, p, C, route_seconds=1e9, slice_chunks=64)
    n_slices = C // 64
    assert full["sample"].startswith(f"routing timed on {n_slices} slices of 64 chunks")
    assert f"{min(n_slices * 64, C)} of {C} chunks" in full["sample"]


def test_cpu_baseline_visiting_order_is_a_spread_of_distinct_slices():
    """The order in which cpu_baseline visits slices (bit-reversed counter
    scaled to the slice count) starts at both ends and the middle and stays
    in range."""
    for n in (1, 2, 7, 64, 98):
        order = [int(f"{d:032b}"[::-1], 2) * n >> 32 for d in range(n)]
        assert all(0 <= i < n for i in order)
        if n >= 2:
            assert order[:2] == [0, n // 2]
        if n in (2, 64):  # a power of two: every slice exactly once
            assert sorted(order) == list(range(n))


def test_clock_merge_prefers_timed_region_samples():
    nvml = {"sm_mhz": 1950.0, "sm_min_mhz": 1900, "sm_max_mhz": 1965, "samples": 12,
            "reasons": ["sw_power_cap"], "source": "NVML, ~1 ms polling"}
    smi = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "samples": 2, "reasons": ["hw_slowdown"]}
    got = bench.merge_clocks(nvml, smi)
    assert got["sm_mhz"] == 1950.0 and got["samples"] == 12
    assert got["reasons"] == ["hw_slowdown", "sw_power_cap"]  # either source's reason is kept
    assert got["nvidia_smi"] == smi
    assert bench.merge_clocks(None, smi) is smi


def test_nvml_sampler_without_a_gpu_reports_nothing():
    s = bench.NvmlSampler(0).start()
    assert s.stop() is None
