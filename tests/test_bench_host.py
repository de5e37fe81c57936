"""Host-side logic of bench.py: the DRAM-traffic figure is taken from a committed
profile summary only while its source digest matches the kernel sources, the HBM
peak falls back to the fixed figure without a measured one, and the clock sampler's
CSV parsing (median SM clock, throttle reasons that were active)."""
import json
import os

import bench


def _tree(tmp_path, src=b"__global__ void k() {}\n"):
    csrc = tmp_path / "quantized_decode_q4_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cu").write_bytes(src)
    (tmp_path / "profiles").mkdir()
    return csrc


def test_recorded_traffic_follows_source_digest(tmp_path, monkeypatch):
    csrc = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("w", 1) is None           # no summary
    digest = bench.source_digest()
    (tmp_path / "profiles" / "gemv_launches_w_b1.txt").write_text(
        f"# summary\n\ndram_bytes_per_launch: 12345\nsource_digest: {digest}\n")
    assert bench.recorded_traffic("w", 1) == 12345.0
    assert bench.recorded_traffic("w", 16) is None          # other batch: no summary
    (csrc / "a.cu").write_bytes(b"__global__ void k() { int changed; }\n")
    assert bench.source_digest() != digest
    assert bench.recorded_traffic("w", 1) is None           # kernel changed since


def test_source_digest_covers_every_file_and_its_name(tmp_path, monkeypatch):
    csrc = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d0 = bench.source_digest()
    (csrc / "b.h").write_bytes(b"#pragma once\n")
    d1 = bench.source_digest()
    os.rename(csrc / "b.h", csrc / "c.h")
    d2 = bench.source_digest()
    assert len({d0, d1, d2}) == 3


def test_hbm_peak_measured_and_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peak, src = bench.hbm_peak()
    assert peak == bench.FALLBACK_HBM_GBS and src.startswith("fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6548.5}))
    peak, src = bench.hbm_peak()
    assert peak == 6548.5 and src.startswith("measured")


class _Done:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def kill(self):
        pass


def test_clock_sampler_parsing(tmp_path):
    out = tmp_path / "clocks.csv"
    rows = [
        "0, 1965, 1965, 650.10, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1912, 1965, 990.50, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 700.00, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    out.write_text("\n".join(rows) + "\n")
    c = bench.Clocks(0)
    c.proc = _Done()
    c.out = open(out, "a")
    info = c.stop()
    assert info["sm_mhz"] == 1965 and info["sm_mhz_min"] == 1912 and info["sm_max_mhz"] == 1965
    assert info["samples"] == 3
    assert info["reasons"] == ["sw_power_cap"]
    assert info["power_w_max"] == 990.5
    assert not out.exists()                                 # the sample file is removed


def test_clock_sampler_without_nvidia_smi_reports_nothing():
    c = bench.Clocks(0)
    assert c.stop() is None


def test_pack_dequant_timing_arithmetic(monkeypatch):
    """time_pack_dequant on the CPU with stand-ins for the device pieces: 3 warm-up
    and 10 timed calls of each, outputs reused, bytes 4nk + 9nk/16, GB/s and the
    fraction of the given peak from the event time."""
    import torch

    from quantized_decode_q4_b200 import q4, synth

    class Event:
        def __init__(self, enable_timing=False):
            self.t = None

        def record(self, stream=None):
            self.t = calls["n"]

        def synchronize(self):
            pass

        def elapsed_time(self, end):
            return 0.05 * (end.t - self.t)      # 50 us per call

    calls = {"n": 0, "pack": 0, "dequant": 0}
    real_empty = torch.empty

    def fake_pack(w, out=None, stream=None):
        calls["n"] += 1
        calls["pack"] += 1
        return out if out is not None else "planes"

    def fake_dequant(m, out=None, stream=None):
        calls["n"] += 1
        calls["dequant"] += 1
        assert m == "planes" and out is not None
        return out

    monkeypatch.setattr(torch.cuda, "Event", Event)
    monkeypatch.setattr(torch.cuda, "empty_cache", lambda: None)
    monkeypatch.setattr(torch, "empty", lambda *a, **kw: real_empty(1))
    monkeypatch.setattr(q4, "pack", fake_pack)
    monkeypatch.setattr(q4, "dequant", fake_dequant)
    monkeypatch.setattr(synth, "matrix", lambda *a, **kw: "w")
    n, k = 14336, 4096
    res = bench.time_pack_dequant(6548.5, n, k, reps=10)
    assert calls["pack"] == 1 + 3 + 10 and calls["dequant"] == 3 + 10
    nbytes = 4 * n * k + 9 * n * k // 16
    assert res["bytes_per_call"] == nbytes
    for name in ("pack", "dequant"):
        assert abs(res[name]["us_per_call"] - 50.0) < 1e-9
        assert abs(res[name]["gbs"] - nbytes / 50e-6 / 1e9) < 1e-6
        assert abs(res[name]["frac"] - res[name]["gbs"] / 6548.5) < 1e-12


def test_step_percentiles_match_linear_interpolation():
    import numpy as np
    rng = np.random.default_rng(5)
    for n in (1, 2, 3, 10, 200):
        ms = list(rng.uniform(1.0, 2.0, n))
        d = bench.step_percentiles(ms)
        assert d["steps"] == n
        for key, p in (("median_ms", 50), ("p10_ms", 10), ("p90_ms", 90)):
            assert abs(d[key] - float(np.percentile(ms, p))) < 1e-12, (n, key)
