"""Pins for the oracle's proxy scores and Sol routing (CPU only).

Independent references: hand-derived rows (tests/golden/sol_rule_rows.txt),
Python's exact-rational ``statistics`` module, brute-force token-pair sums of
the dequantised INT8 tensors, and structural properties (nesting in tau,
prefix protection).
"""
import math
import os
import statistics

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_golden_rows():
    for line in open(os.path.join(GOLDEN, "sol_rule_rows.txt")):
        if line.startswith("#") or not line.strip():
            continue
        tau, scores, want = (t.strip() for t in line.split("|"))
        tau = float(tau)
        s = np.array([[float(v) for v in scores.split()]])
        keep, stats, _ = oracle.sol_route(s, tau)
        assert keep[0].astype(int).tolist() == [int(v) for v in want.split()], line


def test_statistics_match_exact_rational_reference():
    rng = np.random.default_rng(11)
    s = rng.standard_normal((40, 97)) * rng.uniform(0.1, 10, (40, 1)) + rng.uniform(-5, 5, (40, 1))
    for tau in (-0.7, 0.5, 1.0, 1.5):
        keep, stats, band = oracle.sol_route(s, tau)
        for i in range(40):
            row = [float(v) for v in s[i]]
            mu = statistics.fmean(row)
            sd = statistics.pstdev(row)
            assert abs(stats[i, 0] - mu) <= 1e-12 * (abs(mu) + sd)
            assert abs(stats[i, 1] - sd) <= 1e-12 * sd
            T = mu + tau * sd
            ref = np.array([v >= T for v in row])
            ok = ~band[i]
            assert (keep[i][ok] == ref[ok]).all()


def test_nested_in_tau_and_counts_fall():
    rng = np.random.default_rng(12)
    s = rng.standard_normal((30, 200))
    prev = None
    for tau in (-math.inf, -1.0, 0.0, 0.5, 1.0, 1.5, 2.5):
        keep, _, _ = oracle.sol_route(s, tau)
        if prev is not None:
            assert (keep <= prev).all()          # raising tau only skips more
        prev = keep
    keep, _, _ = oracle.sol_route(s, -math.inf)
    assert keep.all()


def test_prefix_protection():
    rng = np.random.default_rng(13)
    s = rng.standard_normal((10, 40))
    n_prefix = 256                                # 2 query blocks, 4 key blocks
    keep, stats, _ = oracle.sol_route(s, 0.8, n_prefix)
    assert keep[:2].all()                         # protected query blocks: all exact
    assert keep[:, :4].all()                      # protected key blocks: always exact
    sub_keep, sub_stats, _ = oracle.sol_route(s[:, 4:], 0.8, 0)
    assert (keep[2:, 4:] == sub_keep[2:]).all()
    assert np.allclose(stats[2:, :2], sub_stats[2:, :2], rtol=0, atol=0)


def test_near_threshold_band_is_relative_to_sigma():
    # mean 0 exactly (symmetric pairs), sigma ~ 577, tau = 0 -> T = 0; the band is 1e-6 sigma ~ 5.8e-4 wide
    s = np.array([[-1000.0, 1000.0, 1e-4, -1e-4, 1e-2, -1e-2]])
    keep, stats, band = oracle.sol_route(s, 0.0)
    assert stats[0, 0] == 0.0 and stats[0, 2] == 0.0
    assert abs(stats[0, 1] - statistics.pstdev(s[0].tolist())) <= 1e-9
    assert band[0].tolist() == [False, False, True, True, False, False]
    assert keep[0].tolist() == [False, True, True, False, True, False]


def test_topk_row_statistics_are_population_moments():
    rng = np.random.default_rng(21)
    s = rng.standard_normal((6, 37)) * 3.0 + 1.0
    _, stats = oracle.topk_route(s, 0.6)
    for i in range(6):
        row = s[i].tolist()
        assert abs(stats[i, 0] - statistics.fmean(row)) <= 1e-12 * 4
        assert abs(stats[i, 1] - statistics.pstdev(row)) <= 1e-12 * 3


def test_equal_rows_and_empty_routed_set():
    s = np.full((3, 8), 2.5)
    keep, _, _ = oracle.sol_route(s, 1.0)
    assert keep.all()
    keep, _, _ = oracle.sol_route(np.random.default_rng(0).standard_normal((2, 4)), 1.0, n_prefix=256)
    assert keep.all()                            # every key block in the prefix


def _dequant_mean_logit(q8, sq, k8, sk, i, j, Lq, Lk):
    rows = range(128 * i, min(Lq, 128 * i + 128))
    toks = range(64 * j, min(Lk, 64 * j + 64))
    tot = 0.0
    for r in rows:
        qr = q8[r].astype(np.float64) * float(sq[i])
        for t in toks:
            tot += float(qr @ (k8[t].astype(np.float64) * float(sk[j])))
    return tot / (len(rows) * len(toks))


def test_proxy_is_mean_dequantised_logit_up_to_row_factor():
    x = np.random.default_rng(14).standard_normal((2, 300, 16)).astype(np.float32)
    q = torch.from_numpy(x[0]).to(torch.bfloat16).float().numpy()
    k = torch.from_numpy(x[1]).to(torch.bfloat16).float().numpy()
    r = oracle.route_head(q, k, 1.0)
    nQB, nKB = r["scores"].shape
    assert (nQB, nKB) == (3, 5)
    for i in range(nQB):
        n_i = min(300, 128 * i + 128) - 128 * i
        for j in range(nKB):
            ref = _dequant_mean_logit(r["q8"], r["q_scale"], r["k8"], r["k_scale"], i, j, 300, 300)
            got = r["scores"][i, j] * float(r["q_scale"][i]) / n_i
            assert abs(got - ref) <= 1e-11 * max(1.0, abs(ref)), (i, j, got, ref)


def test_integer_dot_equals_token_pair_sum():
    x = np.random.default_rng(15).standard_normal((2, 200, 8)).astype(np.float32)
    r = oracle.route_head(x[0], x[1], 1.0)
    q8, k8 = r["q8"], r["k8"]
    PK = r["k_pool"].sum(axis=1)
    for i in range(2):
        for j in range(4):
            brute = sum(int(q8[a, c]) * int(k8[b, c])
                        for a in range(128 * i, min(200, 128 * i + 128))
                        for b in range(64 * j, min(200, 64 * j + 64))
                        for c in range(8))
            assert int(r["q_pool"][i] @ PK[j]) == brute


def test_route_independent_of_centroid_mode_and_nested_on_workload():
    w = workloads.get("ragged_pe")
    q, k, _ = workloads.head_qkv(w, 0, 1)
    keeps = []
    for tau in (0.5, 1.0, 1.5):
        r = oracle.route_head(q.float().numpy(), k.float().numpy(), tau)
        keeps.append(r["keep"])
    assert (keeps[1] <= keeps[0]).all() and (keeps[2] <= keeps[1]).all()
    assert keeps[0].sum() > keeps[2].sum()


# ------------------------------------------------------ fixed-sparsity top-k
def test_topk_keep_count_closed_form():
    # k = |R| - floor(sparsity * |R|): the recipe's 0.75 keeps a quarter
    assert oracle.topk_keep_count(512, 0.75) == 128
    assert oracle.topk_keep_count(1323, 0.75) == 331       # floor(992.25) = 992 skipped
    assert oracle.topk_keep_count(10, 0.0) == 10
    assert oracle.topk_keep_count(10, 1.0) == 0
    assert oracle.topk_keep_count(0, 0.5) == 0
    for bad in (-0.01, 1.01, float("nan")):
        with pytest.raises(ValueError):
            oracle.topk_keep_count(10, bad)


def test_topk_separates_kept_from_skipped_and_breaks_ties_by_index():
    rng = np.random.default_rng(23)
    # coarse integer scores: many exact ties
    s = rng.integers(-4, 5, (30, 53)).astype(np.float64)
    for sp in (0.0, 0.3, 0.5, 0.75, 0.9, 1.0):
        keep, stats = oracle.topk_route(s, sp)
        k = oracle.topk_keep_count(53, sp)
        for i in range(30):
            kept = np.nonzero(keep[i])[0]
            skipped = np.nonzero(~keep[i])[0]
            assert len(kept) == k
            if len(kept) and len(skipped):
                lo, hi = s[i, kept].min(), s[i, skipped].max()
                assert lo >= hi
                # at the boundary value every kept index precedes every skipped one
                if lo == hi:
                    assert kept[s[i, kept] == lo].max() < skipped[s[i, skipped] == hi].min()
                assert stats[i, 2] == lo
            if k == 0:
                assert stats[i, 2] == math.inf
            if k == 53:
                assert stats[i, 2] == -math.inf


def test_topk_brute_force_on_tiny_rows():
    # the kept set is the lexicographically first k-subset under (score desc, index asc)
    import itertools
    rng = np.random.default_rng(5)
    for _ in range(40):
        n = int(rng.integers(1, 8))
        row = rng.integers(-2, 3, n).astype(np.float64)
        for k in range(n + 1):
            sp = (n - k) / n
            if oracle.topk_keep_count(n, sp) != k:
                continue
            best = None
            for sub in itertools.combinations(range(n), k):
                key = (-sum(row[list(sub)]), sorted(sub))
                if best is None or key < best[0]:
                    best = (key, sub)
            keep, _ = oracle.topk_route(row[None, :], sp)
            assert sorted(np.nonzero(keep[0])[0].tolist()) == sorted(best[1])


def test_topk_matches_sol_rule_at_the_same_count():
    # two independent selection rules agree: with distinct scores, keeping the
    # top m routed blocks is the Sol set whenever the Sol rule keeps m of them
    rng = np.random.default_rng(8)
    n = 64                                   # |R| a power of two: (n - m)/n is exact
    for _ in range(50):
        row = rng.standard_normal(n) * rng.uniform(0.5, 3) + rng.uniform(-2, 2)
        for tau in (0.0, 0.5, 1.0, 1.5):
            keep_sol, _, _ = oracle.sol_route(row[None, :], tau)
            m = int(keep_sol.sum())
            sp = (n - m) / n
            assert oracle.topk_keep_count(n, sp) == m
            keep_tk, _ = oracle.topk_route(row[None, :], sp)
            assert (keep_tk == keep_sol).all()


def test_topk_nested_in_sparsity_and_prefix_dense():
    rng = np.random.default_rng(4)
    s = rng.standard_normal((12, 40))
    prev = None
    for sp in (0.0, 0.25, 0.5, 0.75, 1.0):
        keep, _ = oracle.topk_route(s, sp, n_prefix=256)     # key blocks 0-3 and query blocks 0-1 dense
        assert keep[:, :4].all() and keep[:2].all()
        assert (keep[2:, 4:].sum(axis=1) == oracle.topk_keep_count(36, sp)).all()
        if prev is not None:
            assert (keep <= prev).all()
        prev = keep
    keep, stats = oracle.topk_route(s, 0.5, n_prefix=64 * 40)  # nothing routed
    assert keep.all() and (stats[:, 2] == -math.inf).all()
