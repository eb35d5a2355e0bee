"""Proxy block scores and the Sol routing rule (oracle; test infrastructure only).

Source: "Configure Sol Sparse Attention", *How it works*: every 128-token
query block scores each 64-token K/V block with a cheap proxy computed on the
prequantized INT8 Q/K, and compares it with mean + routing_threshold * std
over its row; *The inputs that matter*: routing_threshold defaults to 1.0,
lowering it keeps more blocks exact and raising it skips more; prefix_policy
manual keeps the leading manual_prefix_tokens exact ("Ref2VA VSA", *2-stage
attention patch*: conditioning tokens stay fully dense, pruning touches only
generated-video key tiles).

Readings where the pages are silent or garbled:

* Proxy score. The pages only call it cheap and INT8-based. It is taken as the
  mean-pooled dequantised logit sq_i*sk_j*dot_ij/(n_i*n_j*sqrt(d)) with
  dot_ij = sum_c PQ_i[c]*PK_j[c] (exact integer dot of the block sum-pools).
  The factors constant along a row (sq_i, n_i, sqrt(d)) are dropped, since
  mean + tau*std commutes with a positive row scale; sk_j and n_j vary along
  the row and stay: s_ij = fl64(fl64(dot_ij * sk_j) / n_j), in that order.
* Direction. One sentence says a block is skipped when its score beats the
  threshold, but the same page says raising routing_threshold skips more,
  which only holds if blocks above the threshold stay exact. Keep-above is
  adopted: keep exact iff s_ij >= T_i = mu_i + tau*sigma_i.
* Statistics over the routed key blocks R_i of the row (all key blocks, or
  those starting at or after n_prefix): mu = sum(s)/|R| summed in ascending j,
  sigma = sqrt(sum((s - mu)^2)/|R|) (population form).
* Special rows keep every block: a query block that starts before n_prefix,
  a row whose routed scores are all equal (max == min), an empty R_i, and
  tau = -inf.
* Key blocks that start before n_prefix are always kept and are not in R_i.
* Near-threshold band: a routed block with |s - T| <= 1e-6 * sigma is flagged;
  reduction order may legitimately decide it either way.

Fixed-sparsity top-k routing ("Ref2VA VSA", *2-stage attention patch* and
*Wiring it into a workflow*: top-k pruning applies only to the generated-video
key tiles, the reference/conditioning prefix stays dense, and the recipe runs
at sparsity 0.75). The pages' gate is a learned projection; here the same
proxy scores as the Sol rule rank the blocks. Readings:

* Each routed row keeps k = |R| - floor(sparsity * |R|) blocks (the product in
  fp64), so "sparsity" is the skipped fraction of the routed blocks.
* Ranking: score descending, ties to the lower key-block index.
* Prefix query rows, an empty R, and k = |R| keep every block; key blocks
  before n_prefix are always kept; skipped blocks keep their centroid terms
  in the attention step exactly as under the Sol rule.
* Row statistics: (mu, sigma) as for the Sol rule, and T = the k-th largest
  routed score (-inf when every routed block is kept, +inf when k = 0).
"""
import math

import numpy as np

from .quant import quantize_blocks, q_pools, k_half_pools, block_rows, Q_ROWS, K_ROWS

BAND_REL = 1e-6


def proxy_scores(PQ, PK_half, k_scale, Lk: int):
    """fp64 proxy scores s [nQB, nKB] from pools and K block scales."""
    PK = PK_half.sum(axis=1)                         # whole 64-row block pools
    dot = PQ.astype(np.int64) @ PK.astype(np.int64).T  # exact int64 dot products
    n_j = np.array([t1 - t0 for t0, t1 in block_rows(Lk, K_ROWS)], dtype=np.float64)
    prod = dot.astype(np.float64) * k_scale.astype(np.float64)[None, :]
    return prod / n_j[None, :]


def _sequential_sum(a):
    """Row sums accumulated left to right (ascending j) in fp64."""
    if a.shape[1] == 0:
        return np.zeros(a.shape[0])
    return np.cumsum(a, axis=1)[:, -1]


def sol_route(s, tau: float, n_prefix: int = 0):
    """Sol rule over one head's score matrix s [nQB, nKB].

    Returns (keep bool [nQB, nKB], stats fp64 [nQB, 3] = (mu, sigma, T),
    band bool [nQB, nKB]).
    """
    nQB, nKB = s.shape
    routed = (K_ROWS * np.arange(nKB)) >= n_prefix
    R = s[:, routed]
    nR = R.shape[1]
    keep = np.zeros((nQB, nKB), dtype=bool)
    band = np.zeros((nQB, nKB), dtype=bool)
    stats = np.zeros((nQB, 3), dtype=np.float64)
    if nR > 0:
        mu = _sequential_sum(R) / nR
        var = _sequential_sum((R - mu[:, None]) ** 2) / nR
        sigma = np.sqrt(var)
    else:
        mu = np.zeros(nQB)
        sigma = np.zeros(nQB)
    for i in range(nQB):
        all_kept = (
            tau == -math.inf
            or nR == 0
            or Q_ROWS * i < n_prefix
            or R[i].max() == R[i].min()
        )
        if all_kept:
            T = -math.inf
        else:
            T = mu[i] + tau * sigma[i]
        stats[i] = (mu[i], sigma[i], T)
        if all_kept:
            keep[i, :] = True
            continue
        keep[i, routed] = R[i] >= T
        keep[i, ~routed] = True
        band[i, routed] = np.abs(R[i] - T) <= BAND_REL * sigma[i]
    return keep, stats, band


def topk_keep_count(n_routed: int, sparsity: float) -> int:
    """Routed blocks a row keeps at a fixed sparsity: |R| - floor(sparsity * |R|)."""
    sparsity = float(sparsity)
    if not 0.0 <= sparsity <= 1.0:
        raise ValueError(f"sparsity must be in [0, 1], got {sparsity}")
    return n_routed - int(math.floor(sparsity * n_routed))


def topk_route(s, sparsity: float, n_prefix: int = 0):
    """Fixed-sparsity top-k selection over one head's score matrix s [nQB, nKB].

    Returns (keep bool [nQB, nKB], stats fp64 [nQB, 3] = (mu, sigma, T)).
    """
    nQB, nKB = s.shape
    routed = (K_ROWS * np.arange(nKB)) >= n_prefix
    ridx = np.nonzero(routed)[0]
    nR = len(ridx)
    k = topk_keep_count(nR, sparsity)
    keep = np.zeros((nQB, nKB), dtype=bool)
    stats = np.zeros((nQB, 3), dtype=np.float64)
    R = s[:, routed]
    if nR > 0:
        mu = _sequential_sum(R) / nR
        sigma = np.sqrt(_sequential_sum((R - mu[:, None]) ** 2) / nR)
    else:
        mu = np.zeros(nQB)
        sigma = np.zeros(nQB)
    for i in range(nQB):
        if Q_ROWS * i < n_prefix or k >= nR:
            keep[i, :] = True
            T = -math.inf
        else:
            keep[i, ~routed] = True
            if k == 0:
                T = math.inf
            else:
                # primary key: score descending; secondary: key-block index ascending
                order = ridx[np.lexsort((ridx, -s[i, ridx]))]
                keep[i, order[:k]] = True
                T = s[i, order[k - 1]]
        stats[i] = (mu[i], sigma[i], T)
    return keep, stats


def route_head(q, k, tau: float, n_prefix: int = 0):
    """Quantise, pool, score and route one (batch, head).

    ``q`` [Lq, d] and ``k`` [Lk, d] hold bf16 values (any dtype that widens
    exactly to fp32). Returns a dict of every intermediate.
    """
    q = np.asarray(q, dtype=np.float32)
    k = np.asarray(k, dtype=np.float32)
    q8, sq = quantize_blocks(q, Q_ROWS)
    k8, sk = quantize_blocks(k, K_ROWS)
    PQ = q_pools(q8)
    PKh = k_half_pools(k8)
    s = proxy_scores(PQ, PKh, sk, k.shape[0])
    keep, stats, band = sol_route(s, tau, n_prefix)
    return dict(q8=q8, q_scale=sq, k8=k8, k_scale=sk, q_pool=PQ, k_pool=PKh,
                scores=s, keep=keep, stats=stats, band=band)
