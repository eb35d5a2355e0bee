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
