"""Host-side arithmetic of bench.py (CPU only): algorithmic work, routing bytes
and the roofline numbers, each against an independent count."""
import types

import numpy as np
import torch

import bench
import workloads


def test_kept_work_matches_pair_enumeration():
    # ragged tails in both directions (1000 = 7*128 + 104 = 15*64 + 40), 2x32 centroids
    for name in ("ragged_pe", "ragged_pe_2x32"):
        w = workloads.get(name)
        rng = np.random.default_rng(1)
        m = (rng.random((w.B, w.H, w.nQB, w.nKB)) < 0.3).astype(np.uint8)
        wk = bench.kept_work(types.SimpleNamespace(kept_mask=torch.from_numpy(m)), w)
        c = w.centroid_mode
        f = 0
        for b in range(w.B):
            for h in range(w.H):
                for i in range(w.nQB):
                    ni = min(128, w.Lq - 128 * i)
                    for j in range(w.nKB):
                        nj = min(64, w.Lk - 64 * j)
                        # kept: every (row, key) pair; skipped: c centroid terms per row
                        f += 2 * w.d * ni * (nj if m[b, h, i, j] else c)
        assert wk["f_qk"] == f and wk["f_pv"] == f
        assert wk["kept_blocks"] == int(m.sum()) and wk["routed_blocks"] == m.size
        assert abs(wk["sparsity"] - (1 - m.mean())) < 1e-12


def test_route_bytes_formula_at_the_headline_shape():
    w = workloads.get("wan14b")
    BH, L, d, nQB, nKB = 40, 32760, 128, 256, 512
    expect = (2 * BH * 2 * L * d          # read bf16 Q and K
              + BH * 2 * L * d            # write int8 Q and K
              + 4 * BH * (nQB + nKB)      # scales
              + 2 * 4 * BH * (nQB + 2 * nKB) * d   # pools written, then read by the router
              + 5 * BH * nQB * nKB        # kept mask + kept list
              + 4 * BH * nQB)             # counts
    assert bench.route_bytes(w) == expect == 1085194240


def test_roofline_numbers_are_consistent():
    w = workloads.get("tiny")
    work = dict(f_qk=1e12, f_pv=1e12)
    r = dict(attn_ms=1.0, route_ms=0.1, centroid_ms=0.05, ms=1.25)
    rf = bench.roofline_numbers(w, work, r, dict(bf16=1000.0, hbm=6000.0, src="test"))
    # int8 at twice the bf16 peak on one tensor pipe: t_roof = 1e12/2e15 + 1e12/1e15 = 1.5 ms
    assert abs(rf["attn"]["peak"] - 2e12 / 1.5e-3 / 1e12) < 0.01
    assert abs(rf["attn"]["achieved"] - 2000.0) < 0.01
    assert abs(rf["attn"]["frac"] - 1.5) < 1e-4
    assert abs(rf["kept_tflops"] - 2e12 / 1.25e-3 / 1e12) < 0.01
    assert abs(rf["route"]["achieved"] - bench.route_bytes(w) / 1e-4 / 1e9) < 0.1
    assert abs(rf["route"]["frac_of_spec"] * 8000.0 - rf["route"]["achieved"]) < 0.5
    # dense-equivalent work over the whole call against the same effective tensor peak
    assert abs(rf["dense_equiv_frac"] - w.dense_flops() / 1.25e-3 / 1e12 / rf["attn"]["peak"]) < 1e-3


def test_centroid_bytes_and_mufu_bound_at_the_headline_shape():
    w = workloads.get("wan14b")
    # V read once (40 x 32760 x 128 bf16) + 32 tiles of 64 rows x (int8 key + bf16 value) + 8 B per group
    assert bench.centroid_bytes(w) == 2 * 40 * 32760 * 128 + 40 * 32 * 64 * 128 * 3 + 40 * 32 * 32 * 8
    # one exponential per logit: f_qk / (2 d); 16 per SM per clock on 148 SMs at 1965 MHz
    work = dict(f_qk=2.0 * 128 * 1e9, f_pv=0.0)
    mb = bench.mufu_bound(work, w, 2.0)
    assert mb["exps"] == 1e9
    assert abs(mb["t_bound_ms"] - 1e9 / (16 * 148 * 1965e6) * 1e3) < 1e-4
    assert abs(mb["frac"] - mb["t_bound_ms"] / 2.0) < 1e-3


def test_virtual_work_counts_exact_pairs_and_virtual_groups():
    w = workloads.get("h3_virtual")
    f_qk, f_pv = bench.virtual_work(w, 5)
    # 8064 x 8064 exact pairs per head, plus 5 slices x 63 blocks x 2 groups centroid terms per row
    per_head = 8064 * (8064 + 5 * 63 * 2)
    assert f_qk == f_pv == 2 * 128 * 40 * per_head
    assert bench.virtual_work(w, 0)[0] == 2 * 128 * 40 * 8064 * 8064
