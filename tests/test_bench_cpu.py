"""The benchmark's CPU baseline does the oracle's whole work: its phase-by-
phase composition (scoring, selection, packing, decode) gives the same
strategies and packed bytes as the oracle's one-call compress, and the
record extrapolates linearly by unit count."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_phase_composition_matches_one_call_compress(orc):
    sys.path.insert(0, ROOT)
    import bench
    from kv_cache_compression_kv2d_b200 import synth
    wl = synth.WORKLOADS["tiny"]
    batch = synth.generate(wl, seed=0)
    units = bench.cpu_sample_units(wl, 0, 4)
    assert units == [(0, 0)]
    xs = bench.host_units(batch, wl, units)
    p = orc.params(wl.head_dim, wl.group, wl.segment_len, wl.window, wl.r, wl.c,
                   float(np.float32(wl.budget)), float(np.float32(1 / np.sqrt(wl.head_dim))))
    ph = bench.oracle_unit_phases(orc, p, xs[0])
    assert set(ph) == {"scoring", "selection", "packing", "decode"}
    assert all(t >= 0 for t in ph.values())
    x = xs[0]
    ref = orc.compress_unit(p, x["T"], 0, x["K"], x["V"], x["qw"])
    # the same pipeline, step by step, as the timed baseline runs it
    Kd = x["K"].astype(np.float64)
    a = orc.win_stats(p, x["qw"].astype(np.float64))
    _, s = orc.score(p, x["T"], 0, Kd, x["qw"].astype(np.float64))
    S, nseg = wl.segment_len, x["T"] // wl.segment_len
    cidx, g = orc.channel(p, Kd[:nseg * S], a)
    E = np.array([orc.segment_errors(p, s[j * S:(j + 1) * S], g[j * S:(j + 1) * S],
                                     orc.topr(p, s[j * S:(j + 1) * S])) for j in range(nseg)])
    st, strat, used = orc.budget(p, E)
    assert st == 0 and np.array_equal(strat, ref["strat"]) and used == ref["used"]
    seg = [orc.pack_segment(p, int(strat[j]), x["K"][j * S:(j + 1) * S], x["V"][j * S:(j + 1) * S],
                            orc.topr(p, s[j * S:(j + 1) * S]), cidx[j * S:(j + 1) * S])
           for j in range(nseg)]
    assert np.array_equal(np.concatenate(seg), ref["arena"])


def test_cpu_record_extrapolates_by_units():
    sys.path.insert(0, ROOT)
    import bench
    from kv_cache_compression_kv2d_b200 import synth
    wl = synth.WORKLOADS["llama3_8b_b16_128k_mix"]
    units = bench.cpu_sample_units(wl, 0, 8)
    assert len(units) == 8 and len(set(units)) == 8
    assert units == bench.cpu_sample_units(wl, 0, 8)          # seeded: both arms agree
    xs = [dict(T=131072)] * 8
    rec = bench.cpu_record(wl, units, xs, 10.0, {"scoring": 60.0, "selection": 20.0,
                                                 "packing": 0.0, "decode": 0.0}, 8 * 131072 * 512)
    assert rec["cores"] == 8
    assert abs(rec["extrapolated_step_s"] - 10.0 * 128 / 8) < 1e-9
    assert abs(rec["value"] - 8 * 131072 * 512 / 10.0 / 1e9) < 1e-12
    assert abs(rec["phase_share"]["scoring"] - 0.75) < 1e-12


def test_roofline_hbm_and_tensor_peaks():
    import bench
    # 4.7 GB in 2.676 ms against a 6555.5 GB/s copy
    r = bench.roofline_of("hbm", 4.7e9, 2.676e-3, 6555.5, 1595.8, 1385.2, "measured")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6555.5
    assert abs(r["achieved"] - 4.7e9 / 2.676e-3 / 1e9) < 1e-9
    assert abs(r["frac"] - r["achieved"] / 6555.5) < 1e-15
    # a tensor kernel timed inside the step: sustained peak, burst beside it
    t = bench.roofline_of("tensor", 1.1e12, 1.4e-3, 6555.5, 1595.8, 1385.2, "measured")
    assert t["peak"] == 1385.2 and "sustained" in t["peak_source"]
    assert abs(t["achieved"] - 1.1e12 / 1.4e-3 / 1e12) < 1e-9
    assert abs(t["frac"] * 1385.2 - t["frac_of_burst"] * 1595.8) < 1e-9
    # without a sustained figure the burst one is the peak
    b = bench.roofline_of("tensor", 1.1e12, 1.4e-3, 6555.5, 1595.8, 0.0, "fallback")
    assert b["peak"] == 1595.8 and "burst" in b["peak_source"] and b["frac"] == b["frac_of_burst"]


def test_scoring_both_passes():
    import bench
    # two passes of 1.1 TFLOP in 1.4 ms and 1.6 ms: 2.2 TFLOP / 3.0 ms
    s = bench.scoring_of(1.1e12, 1.1e12, 1400.0, 1600.0, 1595.8, 1385.2, "measured")
    assert abs(s["tflops"] - 2.2e12 / 3.0e-3 / 1e12) < 1e-9
    assert abs(s["frac"] - s["tflops"] / 1385.2) < 1e-15
    assert abs(s["frac_of_burst"] - s["tflops"] / 1595.8) < 1e-15
    assert abs(s["pass1_tflops"] - 1.1e12 / 1.4e-3 / 1e12) < 1e-9
    assert abs(s["pass2_tflops"] - 1.1e12 / 1.6e-3 / 1e12) < 1e-9
    assert s["peak"] == 1385.2 and s["burst_peak"] == 1595.8
