"""Block-sparse softmax attention with centroid terms, and the block-mask entry (oracle).

TEST INFRASTRUCTURE ONLY.

Source: "Configure Sol Sparse Attention", *How it works*: kept blocks are
computed exactly; a skipped 64-token block is not dropped but replaced by one
64-token centroid (1x64) that still enters the online softmax, so the output
stays approximately right; 2x32 keeps two 32-token centroids per skipped
block without changing which blocks route. "FlashVSR Sparge Attention",
intro and *How it works*: the LCSA mask lives on logical 128-query x 128-key
blocks and is converted to the kernel's physical block geometry after
routing; only allowed blocks run.

Readings:

* Exact term, query row r of block i, key token t of kept block j:
  logit = (sq_i * sk_j * scale) * sum_c q8[r,c]*k8[t,c], scale = 1/sqrt(d)
  unless the caller gives one; value V[t].
* Centroid term of a skipped block j, for each group g (1x64: the block's
  valid rows; 2x32: its halves, an empty half omitted):
  kbar_g = sk_j * sum_{t in g} k8[t] / |g| (the dequantised INT8 K that the
  exact path uses), vbar_g = mean of V over g,
  logit = (sq_i * scale) * (q8[r] . kbar_g) + ln|g|, value vbar_g.
  |g| is the actual valid count (56 in a 56-row tail block).
* Output o_r = sum exp(logit - m) * value / sum exp(logit - m), lse = m + ln(sum),
  over exact terms and centroid terms together, in fp64.
* Query blocks that start before n_prefix keep every key block and so carry no
  centroids (they come out of the routing with every block kept).
* Mask entry: physical 64-key block j of query block i runs iff
  mask[b, h mod Hm, i, floor(j/2)]; exact terms only, no centroids; the
  granularity is block-level (no token-causal mask inside a block). A row with
  no allowed block gives o = 0 and lse = -inf.
* Virtual K/V, residual mode ("Configure H3 Static Virtual KV", the mode
  list and "What virtual means physically"): queries stay on the physical
  slices; the physical keys all stay exact; every added virtual slice
  re-reads one source slice through the logical source map and enters only as
  skipped-block centroid terms (2x32 on the page) in the same softmax.
  Reading: a slice is ``slice_tokens`` consecutive tokens, a multiple of 64,
  so that its blocks are whole source blocks; the source keys are taken as
  given (INT8 codes and per-block scales of the source), so a temporal phase
  a caller wants on a virtual slice is already in the source it passes.
* LCSA mask from frame geometry ("FlashVSR Sparge Attention", intro: each
  query block attends only to a small, locally causal set of key blocks; the
  sampler builds the mask). Reading: a logical 128-token block belongs to the
  frame of its first token, floor(128*x / frame_tokens); key block x_k is
  allowed for query block x_q iff f_q - window <= f_k <= f_q.
"""
import math

import numpy as np

from .quant import block_rows, Q_ROWS, K_ROWS


def resolve_scale(d: int, softmax_scale: float) -> float:
    """softmax_scale <= 0 selects 1/sqrt(d)."""
    return 1.0 / math.sqrt(d) if softmax_scale is None or softmax_scale <= 0 else float(softmax_scale)


def centroid_groups(t0: int, t1: int, mode: int):
    """Token spans of the centroid groups of key block [t0, t1)."""
    if mode == 1:
        return [(t0, t1)]
    if mode == 2:
        mid = min(t1, t0 + 32)
        return [(a, b) for a, b in ((t0, mid), (mid, t1)) if b > a]
    raise ValueError("centroid mode must be 1 (1x64) or 2 (2x32)")


def centroid_table(k8, k_scale, v, mode: int):
    """Per key block j: list of (|g|, kbar_g fp64 [d], vbar_g fp64 [d])."""
    Lk = k8.shape[0]
    v = np.asarray(v, dtype=np.float64)
    table = []
    for j, (t0, t1) in enumerate(block_rows(Lk, K_ROWS)):
        groups = []
        for g0, g1 in centroid_groups(t0, t1, mode):
            n = g1 - g0
            kbar = float(k_scale[j]) * k8[g0:g1].astype(np.float64).sum(axis=0) / n
            vbar = v[g0:g1].mean(axis=0)
            groups.append((n, kbar, vbar))
        table.append(groups)
    return table


def _softmax_rows(logits, values):
    """fp64 softmax(logits) @ values with its log-sum-exp, row-wise."""
    m = logits.max(axis=1)
    e = np.exp(logits - m[:, None])
    l = e.sum(axis=1)
    return (e @ values) / l[:, None], m + np.log(l)


def sol_attention_head(q8, q_scale, k8, k_scale, v, keep, centroid_mode: int,
                       softmax_scale: float = 0.0, q_blocks=None):
    """Sol sparse attention of one (batch, head).

    keep: bool [nQB, nKB] from the routing. Returns (O fp64 [Lq, d],
    lse fp64 [Lq]); rows of q-blocks not in ``q_blocks`` are left NaN.
    """
    Lq, d = q8.shape
    Lk = k8.shape[0]
    scale = resolve_scale(d, softmax_scale)
    v = np.asarray(v, dtype=np.float64)
    kspans = block_rows(Lk, K_ROWS)
    table = centroid_table(k8, k_scale, v, centroid_mode) if centroid_mode else None
    O = np.full((Lq, d), np.nan)
    lse = np.full(Lq, np.nan)
    qspans = block_rows(Lq, Q_ROWS)
    for i in (range(len(qspans)) if q_blocks is None else q_blocks):
        r0, r1 = qspans[i]
        Qi = q8[r0:r1].astype(np.float64)
        logits, values = [], []
        for j, (t0, t1) in enumerate(kspans):
            if keep[i, j]:
                dots = Qi @ k8[t0:t1].astype(np.float64).T   # exact integer dots
                logits.append((float(q_scale[i]) * float(k_scale[j]) * scale) * dots)
                values.append(v[t0:t1])
            elif centroid_mode:
                for n, kbar, vbar in table[j]:
                    lg = (float(q_scale[i]) * scale) * (Qi @ kbar) + math.log(n)
                    logits.append(lg[:, None])
                    values.append(vbar[None, :])
        if not logits:
            O[r0:r1] = 0.0
            lse[r0:r1] = -math.inf
            continue
        O[r0:r1], lse[r0:r1] = _softmax_rows(np.concatenate(logits, axis=1),
                                             np.concatenate(values, axis=0))
    return O, lse


def virtual_kv_residual_head(q8, q_scale, k8, k_scale, v, src_k8, src_k_scale, src_v,
                             slice_tokens: int, src_map, centroid_mode: int = 2,
                             softmax_scale: float = 0.0, q_blocks=None):
    """Residual virtual K/V attention of one (batch, head).

    Exact terms: every physical key block (k8, k_scale, v). Centroid terms:
    for each added virtual slice l, the groups of source blocks
    src_map[l]*bps .. (src_map[l]+1)*bps - 1, bps = slice_tokens / 64, built
    from (src_k8, src_k_scale, src_v) exactly as a skipped block's are.
    Returns (O fp64 [Lq, d], lse fp64 [Lq]); rows outside ``q_blocks`` stay NaN.
    """
    if slice_tokens <= 0 or slice_tokens % K_ROWS:
        raise ValueError("slice_tokens must be a positive multiple of 64")
    n_src = src_k8.shape[0] // slice_tokens
    if n_src * slice_tokens != src_k8.shape[0]:
        raise ValueError("the source holds a whole number of slices")
    if any(not 0 <= s < n_src for s in src_map):
        raise ValueError("source map entry out of range")
    Lq, d = q8.shape
    scale = resolve_scale(d, softmax_scale)
    v = np.asarray(v, dtype=np.float64)
    kspans = block_rows(k8.shape[0], K_ROWS)
    table = centroid_table(src_k8, src_k_scale, src_v, centroid_mode)
    bps = slice_tokens // K_ROWS
    virtual = [grp for s in src_map for j in range(s * bps, (s + 1) * bps) for grp in table[j]]
    O = np.full((Lq, d), np.nan)
    lse = np.full(Lq, np.nan)
    qspans = block_rows(Lq, Q_ROWS)
    for i in (range(len(qspans)) if q_blocks is None else q_blocks):
        r0, r1 = qspans[i]
        Qi = q8[r0:r1].astype(np.float64)
        logits, values = [], []
        for j, (t0, t1) in enumerate(kspans):
            dots = Qi @ k8[t0:t1].astype(np.float64).T
            logits.append((float(q_scale[i]) * float(k_scale[j]) * scale) * dots)
            values.append(v[t0:t1])
        for n, kbar, vbar in virtual:
            logits.append(((float(q_scale[i]) * scale) * (Qi @ kbar) + math.log(n))[:, None])
            values.append(vbar[None, :])
        O[r0:r1], lse[r0:r1] = _softmax_rows(np.concatenate(logits, axis=1),
                                             np.concatenate(values, axis=0))
    return O, lse


def lcsa_mask(Lq: int, Lk: int, frame_tokens: int, window: int):
    """Logical LCSA mask, uint8 [ceil(Lq/128), ceil(Lk/128)], built block by block."""
    if frame_tokens <= 0 or window < 0:
        raise ValueError("frame_tokens must be > 0 and window >= 0")
    nq, nk = -(-Lq // 128), -(-Lk // 128)
    m = np.zeros((nq, nk), dtype=np.uint8)
    for xq in range(nq):
        fq = (128 * xq) // frame_tokens
        for xk in range(nk):
            fk = (128 * xk) // frame_tokens
            m[xq, xk] = 1 if fq - window <= fk <= fq else 0
    return m


def physical_allowed(mask_bh, nKB: int):
    """Logical 128x128 mask of one head [nQB, nLK] -> physical [nQB, nKB] (64-key blocks)."""
    mask_bh = np.asarray(mask_bh).astype(bool)
    cols = np.arange(nKB) // 2
    return mask_bh[:, cols]


def masked_attention_head(q8, q_scale, k8, k_scale, v, allowed,
                          softmax_scale: float = 0.0, q_blocks=None):
    """Exact attention over the allowed physical blocks only (no centroids)."""
    return sol_attention_head(q8, q_scale, k8, k_scale, v, allowed, 0,
                              softmax_scale, q_blocks)
