"""Helpers for the GPU-vs-oracle parity tests (imported by tests only).

The CUDA path and the oracle both start from the same seeded bf16 inputs
(``workloads``); no value computed on the GPU is ever fed to the oracle.
Bars (as the method is specified): INT8 tensors, scales, pools and the kept
mask bit-exact, except routed blocks whose score lies within 1e-6*std of the
threshold (counted); outputs within max-abs 1e-2 and relative L2 5e-3. The
output comparison runs on the fp32 output; the bf16 output must then equal
that fp32 output rounded to bf16, bit for bit (a bf16 value near 4 cannot
itself be closer than half an ulp, 2^-7, to the exact result).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

import oracle
import workloads

ATOL = 1e-2
REL_L2 = 5e-3
LSE_ATOL = 1e-3


@dataclass
class Report:
    blocks: int = 0               # routed (query block, key block) pairs whose routing was compared
    band: int = 0                 # near-threshold routed blocks in the compared rows
    band_mismatch: int = 0        # of which the GPU decided differently
    rows_skipped: int = 0         # query blocks left out of the output check
    max_abs: float = 0.0
    rel_l2: float = 0.0
    lse_max_abs: float = 0.0
    notes: list = field(default_factory=list)


def lcsa_input_mask(w) -> torch.Tensor:
    """The logical LCSA mask of a mask-entry workload, uint8 [B, 1, nQB, nLK] (shared by heads),
    built by the oracle from the workload's frame geometry."""
    m = oracle.lcsa_mask(w.Lq, w.Lk, w.frame_tokens, w.lcsa_window)
    return torch.from_numpy(np.broadcast_to(m, (w.B, 1) + m.shape).copy())


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def inputs(w, device="cuda"):
    Q, K, V = workloads.batch_qkv(w)
    return Q.to(device), K.to(device), V.to(device)


def head_np(w, b, h, qkv=None):
    """fp32 numpy Q, K, V of one head: the workload's own, or those of the given CPU bf16 tensors."""
    if qkv is not None:
        return tuple(x[b, h].float().numpy() for x in qkv)
    q, k, v = workloads.head_qkv(w, b, h)
    return q.float().numpy(), k.float().numpy(), v.float().numpy()


def _device_inputs(w, qkv):
    return inputs(w) if qkv is None else tuple(x.to("cuda") for x in qkv)


def check_quant(route, ref, b, h):
    """INT8 tensors, scales and pools of one head, bit for bit."""
    assert np.array_equal(to_np(route.q8[b, h]), ref["q8"]), "q8 differs"
    assert np.array_equal(to_np(route.k8[b, h]), ref["k8"]), "k8 differs"
    assert np.array_equal(to_np(route.q_scale[b, h]), ref["q_scale"]), "q_scale differs"
    assert np.array_equal(to_np(route.k_scale[b, h]), ref["k_scale"]), "k_scale differs"
    assert np.array_equal(to_np(route.q_pool[b, h]).astype(np.int64), ref["q_pool"]), "q_pool differs"
    assert np.array_equal(to_np(route.k_pool[b, h]).astype(np.int64), ref["k_pool"]), "k_pool differs"


def check_route(route, ref, b, h, rep: Report):
    """Kept mask bit-exact outside the near-threshold band; lists consistent with the mask."""
    gm = to_np(route.kept_mask[b, h]).astype(bool)
    om = ref["keep"]
    diff = gm != om
    band = ref["band"]
    rep.blocks += int(gm.size)
    rep.band += int(band.sum())
    rep.band_mismatch += int((diff & band).sum())
    bad = diff & ~band
    assert not bad.any(), f"kept mask differs outside the band at {np.argwhere(bad)[:5].tolist()}"
    cnt = to_np(route.kept_cnt[b, h])
    idx = to_np(route.kept_idx[b, h])
    assert np.array_equal(cnt, gm.sum(axis=1)), "kept_cnt != popcount(kept_mask)"
    for i in range(gm.shape[0]):
        assert np.array_equal(idx[i, :cnt[i]], np.nonzero(gm[i])[0]), f"kept_idx row {i}"
    if route.row_stats is not None:
        st = to_np(route.row_stats[b, h])
        ref_st = ref["stats"]
        fin = np.isfinite(ref_st[:, 2])
        assert np.array_equal(np.isfinite(st[:, 2]), fin), "all-kept rows differ"
        scale = np.abs(ref_st[:, 0]) + ref_st[:, 1] + 1e-300
        assert (np.abs(st[:, 0] - ref_st[:, 0]) <= 1e-12 * scale).all(), "mu differs"
        assert (np.abs(st[:, 1] - ref_st[:, 1]) <= 1e-12 * scale).all(), "sigma differs"
    return diff


def compare_rows(O_gpu, lse_gpu, O_ref, lse_ref, rows, rep: Report):
    """Accumulate output error over the given row indices."""
    if len(rows) == 0:
        return
    g = O_gpu[rows].astype(np.float64)
    r = O_ref[rows]
    err = np.abs(g - r)
    rep.max_abs = max(rep.max_abs, float(err.max()))
    num = float(np.sqrt((err ** 2).sum()))
    den = float(np.sqrt((r ** 2).sum())) + 1e-300
    rep.rel_l2 = max(rep.rel_l2, num / den)
    if lse_gpu is not None:
        lg, lr = lse_gpu[rows].astype(np.float64), lse_ref[rows]
        both_inf = np.isneginf(lg) & np.isneginf(lr)
        assert (np.isneginf(lg) == np.isneginf(lr)).all(), "empty-row lse differs"
        if (~both_inf).any():
            rep.lse_max_abs = max(rep.lse_max_abs, float(np.abs(lg[~both_inf] - lr[~both_inf]).max()))


def assert_band_small(rep: Report, what: str):
    """The near-threshold exemption must stay negligible: at most 1e-4 of the compared routed
    blocks (and never more than a handful in a small case) may be exempt from bit-exactness,
    so that a systematic routing error cannot hide in the band."""
    print(f"{what}: {rep.band} near-threshold blocks of {rep.blocks} compared, {rep.band_mismatch} decided "
          f"differently")
    assert rep.band <= max(4, 1e-4 * rep.blocks), f"{what}: {rep.band} band blocks of {rep.blocks}"


def assert_within(rep: Report, what: str):
    assert rep.max_abs <= ATOL, f"{what}: max-abs {rep.max_abs:.3e} > {ATOL}"
    assert rep.rel_l2 <= REL_L2, f"{what}: rel-L2 {rep.rel_l2:.3e} > {REL_L2}"
    assert rep.lse_max_abs <= LSE_ATOL, f"{what}: lse max-abs {rep.lse_max_abs:.3e} > {LSE_ATOL}"


def q_rows(Lq, blocks):
    rows = []
    for i in blocks:
        rows.extend(range(128 * i, min(Lq, 128 * i + 128)))
    return np.array(rows, dtype=np.int64)


def sol_parity(bsva, w, tau, heads=None, q_blocks=None, centroid_mode=None, qkv=None, attn_heads=None):
    """Route + fwd on the GPU over the whole workload. Routing and quantisation are compared
    bit for bit on ``heads`` (all by default); outputs on ``attn_heads`` (default: ``heads``)
    and ``q_blocks``. ``qkv`` replaces the workload's inputs by CPU bf16 tensors."""
    mode = centroid_mode or w.centroid_mode
    Q, K, V = _device_inputs(w, qkv)
    route = bsva.sparse_attn_route(Q, K, tau, n_prefix=w.n_prefix, row_stats=True)
    out, lse = bsva.sparse_attn_fwd(route, V, mode, with_lse=True, out_dtype=torch.float32)
    out16 = bsva.sparse_attn_fwd(route, V, mode)
    torch.cuda.synchronize()
    # the bf16 output is exactly the rounding of the fp32 output
    assert torch.equal(out16, out.to(torch.bfloat16)), "bf16 output != round(fp32 output)"
    heads = heads or [(b, h) for b in range(w.B) for h in range(w.H)]
    attn_heads = set(attn_heads or heads)
    rep = Report()
    for b, h in heads:
        q, k, v = head_np(w, b, h, qkv)
        ref = oracle.route_head(q, k, tau, w.n_prefix)
        check_quant(route, ref, b, h)
        diff = check_route(route, ref, b, h, rep)
        if (b, h) not in attn_heads:
            continue
        blocks = list(range(w.nQB)) if q_blocks is None else [i for i in q_blocks if i < w.nQB]
        clean = [i for i in blocks if not diff[i].any()]
        rep.rows_skipped += len(blocks) - len(clean)
        O_ref, lse_ref = oracle.sol_attention_head(ref["q8"], ref["q_scale"], ref["k8"], ref["k_scale"], v,
                                                   ref["keep"], mode, 0.0, q_blocks=clean)
        compare_rows(to_np(out[b, h].float()), to_np(lse[b, h]), O_ref, lse_ref, q_rows(w.Lq, clean), rep)
    return route, out, lse, rep


def masked_parity(bsva, w, mask, heads=None, q_blocks=None, softmax_scale=0.0, qkv=None):
    """Quantise on the GPU, run the mask entry, compare with the oracle's masked attention."""
    Q, K, V = _device_inputs(w, qkv)
    qk = bsva.quantize_qk(Q, K)
    m_dev = mask.to("cuda")
    out, lse = bsva.masked_block_attn_fwd(qk["q8"], qk["q_scale"], qk["k8"], qk["k_scale"], V, m_dev,
                                          softmax_scale=softmax_scale, with_lse=True, out_dtype=torch.float32)
    out16 = bsva.masked_block_attn_fwd(qk["q8"], qk["q_scale"], qk["k8"], qk["k_scale"], V, m_dev,
                                       softmax_scale=softmax_scale)
    torch.cuda.synchronize()
    assert torch.equal(out16, out.to(torch.bfloat16)), "bf16 output != round(fp32 output)"
    heads = heads or [(b, h) for b in range(w.B) for h in range(w.H)]
    rep = Report()
    Hm = mask.shape[1]
    for b, h in heads:
        q, k, v = head_np(w, b, h, qkv)
        ref = oracle.route_head(q, k, -math.inf, 0)
        assert np.array_equal(to_np(qk["q8"][b, h]), ref["q8"]) and np.array_equal(to_np(qk["k8"][b, h]), ref["k8"])
        allowed = oracle.physical_allowed(mask[b, h % Hm].numpy(), w.nKB)
        blocks = list(range(w.nQB)) if q_blocks is None else [i for i in q_blocks if i < w.nQB]
        O_ref, lse_ref = oracle.masked_attention_head(ref["q8"], ref["q_scale"], ref["k8"], ref["k_scale"], v,
                                                      allowed, softmax_scale, q_blocks=blocks)
        compare_rows(to_np(out[b, h].float()), to_np(lse[b, h]), O_ref, lse_ref, q_rows(w.Lq, blocks), rep)
    return out, lse, rep


def topk_parity(bsva, w, sparsity, heads=None, q_blocks=None, centroid_mode=None, attn_heads=None):
    """Top-k route + fwd on the GPU; the kept mask and T must match the oracle's
    top-k selection over its own scores bit for bit (no tolerance band: the
    scores are bit-exact and the ranking is a total order)."""
    mode = centroid_mode or w.centroid_mode
    Q, K, V = inputs(w)
    route = bsva.sparse_attn_route_topk(Q, K, sparsity, n_prefix=w.n_prefix, row_stats=True)
    out, lse = bsva.sparse_attn_fwd(route, V, mode, with_lse=True, out_dtype=torch.float32)
    torch.cuda.synchronize()
    heads = heads or [(b, h) for b in range(w.B) for h in range(w.H)]
    attn_heads = set(attn_heads or heads)
    rep = Report()
    for b, h in heads:
        q, k, v = head_np(w, b, h)
        ref = oracle.route_head(q, k, 1.0, w.n_prefix)      # quantisation and scores
        keep, stats = oracle.topk_route(ref["scores"], sparsity, w.n_prefix)
        check_quant(route, ref, b, h)
        gm = to_np(route.kept_mask[b, h]).astype(bool)
        assert np.array_equal(gm, keep), f"top-k kept mask differs at {np.argwhere(gm != keep)[:5].tolist()}"
        cnt = to_np(route.kept_cnt[b, h])
        idx = to_np(route.kept_idx[b, h])
        assert np.array_equal(cnt, keep.sum(axis=1)), "kept_cnt"
        for i in range(keep.shape[0]):
            assert np.array_equal(idx[i, :cnt[i]], np.nonzero(keep[i])[0]), f"kept_idx row {i}"
        st = to_np(route.row_stats[b, h])
        assert np.array_equal(st[:, 2], stats[:, 2]), "top-k threshold T differs"
        scale = np.abs(stats[:, 0]) + stats[:, 1] + 1e-300
        assert (np.abs(st[:, 0] - stats[:, 0]) <= 1e-12 * scale).all(), "mu differs"
        rep.blocks += int(gm.size)
        if (b, h) not in attn_heads:
            continue
        blocks = list(range(w.nQB)) if q_blocks is None else [i for i in q_blocks if i < w.nQB]
        O_ref, lse_ref = oracle.sol_attention_head(ref["q8"], ref["q_scale"], ref["k8"], ref["k_scale"], v,
                                                   keep, mode, 0.0, q_blocks=blocks)
        compare_rows(to_np(out[b, h].float()), to_np(lse[b, h]), O_ref, lse_ref, q_rows(w.Lq, blocks), rep)
    return route, out, lse, rep


def masked_parity_v8(bsva, w, mask, heads=None, q_blocks=None, softmax_scale=0.0, V=None):
    """The mask entry on INT8 V: the GPU quantises V and runs the entry; the oracle
    quantises V with its own quantiser (checked bit for bit) and attends over the
    dequantised values."""
    Q, K, V0 = inputs(w)
    V = V0 if V is None else V.to("cuda")
    qk = bsva.quantize_qk(Q, K)
    vq = bsva.quantize_v(V)
    m_dev = mask.to("cuda")
    out, lse = bsva.masked_block_attn_fwd_v8(qk["q8"], qk["q_scale"], qk["k8"], qk["k_scale"], vq["v8"],
                                             vq["v_scale"], m_dev, softmax_scale=softmax_scale, with_lse=True,
                                             out_dtype=torch.float32)
    out16 = bsva.masked_block_attn_fwd_v8(qk["q8"], qk["q_scale"], qk["k8"], qk["k_scale"], vq["v8"],
                                          vq["v_scale"], m_dev, softmax_scale=softmax_scale)
    torch.cuda.synchronize()
    assert torch.equal(out16, out.to(torch.bfloat16)), "bf16 output != round(fp32 output)"
    heads = heads or [(b, h) for b in range(w.B) for h in range(w.H)]
    rep = Report()
    Hm = mask.shape[1]
    for b, h in heads:
        q, k, _ = head_np(w, b, h)
        v = V[b, h].float().cpu().numpy()
        ref = oracle.route_head(q, k, -math.inf, 0)
        v8, sv = oracle.quantize_blocks(v, 64)
        assert np.array_equal(to_np(vq["v8"][b, h]), v8), "v8 differs"
        assert np.array_equal(to_np(vq["v_scale"][b, h]), sv), "v_scale differs"
        vdeq = oracle.dequantize_blocks(v8, sv, 64)
        allowed = oracle.physical_allowed(mask[b, h % Hm].numpy(), w.nKB)
        blocks = list(range(w.nQB)) if q_blocks is None else [i for i in q_blocks if i < w.nQB]
        O_ref, lse_ref = oracle.masked_attention_head(ref["q8"], ref["q_scale"], ref["k8"], ref["k_scale"], vdeq,
                                                      allowed, softmax_scale, q_blocks=blocks)
        compare_rows(to_np(out[b, h].float()), to_np(lse[b, h]), O_ref, lse_ref, q_rows(w.Lq, blocks), rep)
    return out, lse, rep


def source_batch(w, device="cuda"):
    """[B, H, Ls, d] bf16 source K and V of a virtual K/V workload with a separate source."""
    n = w.n_source_slices * w.slice_tokens
    KS = torch.zeros((w.B, w.H, n, w.d), dtype=torch.bfloat16)
    VS = torch.zeros((w.B, w.H, n, w.d), dtype=torch.bfloat16)
    for b in range(w.B):
        for h in range(w.H):
            ks, vs = workloads.source_kv(w, b, h)
            KS[b, h].copy_(ks)
            VS[b, h].copy_(vs)
    return KS.to(device), VS.to(device)


def virtual_parity(bsva, w, heads=None, q_blocks=None, centroid_mode=None, src_map=None, softmax_scale=0.0):
    """Residual virtual K/V: the GPU quantises the physical Q/K (and a separate source's keys, through
    the K half of quantize_qk) and runs the entry; the oracle quantises with its own quantiser (checked
    bit for bit) and computes each head from the same bf16 inputs."""
    mode = w.centroid_mode if centroid_mode is None else centroid_mode
    src_map = tuple(w.virtual_map if src_map is None else src_map)
    Q, K, V = inputs(w)
    qk = bsva.quantize_qk(Q, K)
    source = src_v = None
    if w.n_source_slices:
        KS, src_v = source_batch(w)
        source = bsva.quantize_qk(KS, KS)
    out, lse = bsva.virtual_kv_residual_fwd(qk, V, w.slice_tokens, src_map, source=source, src_v=src_v,
                                            centroid_mode=mode, softmax_scale=softmax_scale, with_lse=True,
                                            out_dtype=torch.float32)
    out16 = bsva.virtual_kv_residual_fwd(qk, V, w.slice_tokens, src_map, source=source, src_v=src_v,
                                         centroid_mode=mode, softmax_scale=softmax_scale)
    torch.cuda.synchronize()
    assert torch.equal(out16, out.to(torch.bfloat16)), "bf16 output != round(fp32 output)"
    heads = heads or [(b, h) for b in range(w.B) for h in range(w.H)]
    rep = Report()
    for b, h in heads:
        q, k, v = head_np(w, b, h)
        ref = oracle.route_head(q, k, -math.inf, 0)
        assert np.array_equal(to_np(qk["q8"][b, h]), ref["q8"]), "q8 differs"
        assert np.array_equal(to_np(qk["k8"][b, h]), ref["k8"]), "k8 differs"
        if source is None:
            ks8, kss, vs = ref["k8"], ref["k_scale"], v
        else:
            ks, vs = (t.float().numpy() for t in workloads.source_kv(w, b, h))
            ks8, kss = oracle.quantize_blocks(ks, 64)
            assert np.array_equal(to_np(source["k8"][b, h]), ks8), "source k8 differs"
            assert np.array_equal(to_np(source["k_scale"][b, h]), kss), "source k_scale differs"
        blocks = list(range(w.nQB)) if q_blocks is None else [i for i in q_blocks if i < w.nQB]
        O_ref, lse_ref = oracle.virtual_kv_residual_head(ref["q8"], ref["q_scale"], ref["k8"], ref["k_scale"], v,
                                                         ks8, kss, vs, w.slice_tokens, src_map, mode,
                                                         softmax_scale, q_blocks=blocks)
        compare_rows(to_np(out[b, h].float()), to_np(lse[b, h]), O_ref, lse_ref, q_rows(w.Lq, blocks), rep)
    return out, lse, rep
