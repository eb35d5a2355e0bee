"""Pins for the oracle's sparse attention and mask entry (CPU only).

The independent reference is torch's fp64 scaled-dot-product attention on
tensors the tests build themselves: dense attention over the dequantised
INT8 Q/K (tau = -inf, all-ones mask), dense attention over K'/V' in which
every skipped centroid group's rows are replaced by their mean (|g| equal
keys contribute |g| * exp(q.kbar), which is exactly the ln|g| term), and a
token-level boolean mask expanded from the logical block mask.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads


def _head(name, b=0, h=0):
    w = workloads.get(name)
    q, k, v = workloads.head_qkv(w, b, h)
    return w, q.float().numpy(), k.float().numpy(), v.float().numpy()


def _dequant(x8, scale, rows):
    out = np.zeros(x8.shape, np.float64)
    for b, (r0, r1) in enumerate(oracle.block_rows(x8.shape[0], rows)):
        out[r0:r1] = x8[r0:r1].astype(np.float64) * float(scale[b])
    return out


def _sdpa(q, k, v, scale, mask=None):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))[None, None]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    o = F.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=m, scale=scale)
    return o[0, 0].numpy()


@pytest.mark.parametrize("name", ["ragged_pe", "ragged_d64", "cross"])
def test_all_kept_equals_dense_attention(name):
    w, q, k, v = _head(name)
    r = oracle.route_head(q, k, -math.inf)
    assert r["keep"].all()
    O, lse = oracle.sol_attention_head(r["q8"], r["q_scale"], r["k8"], r["k_scale"], v,
                                       r["keep"], w.centroid_mode)
    scale = 1.0 / math.sqrt(w.d)
    ref = _sdpa(_dequant(r["q8"], r["q_scale"], 128), _dequant(r["k8"], r["k_scale"], 64), v, scale)
    assert np.abs(O - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
    # lse against a direct log-sum-exp of the dequantised logits
    lg = scale * _dequant(r["q8"], r["q_scale"], 128) @ _dequant(r["k8"], r["k_scale"], 64).T
    ref_lse = torch.logsumexp(torch.from_numpy(lg), dim=1).numpy()
    assert np.abs(lse - ref_lse).max() <= 1e-10


@pytest.mark.parametrize("name,mode", [("ragged_pe", 1), ("ragged_pe", 2),
                                       ("ragged_d64", 2), ("cross", 1)])
def test_centroids_equal_dense_attention_over_mean_replaced_kv(name, mode):
    w, q, k, v = _head(name, 0, 1)
    r = oracle.route_head(q, k, 0.7)
    keep = r["keep"]
    assert (~keep).any() and keep.any()
    O, lse = oracle.sol_attention_head(r["q8"], r["q_scale"], r["k8"], r["k_scale"], v, keep, mode)
    Qd = _dequant(r["q8"], r["q_scale"], 128)
    Kd = _dequant(r["k8"], r["k_scale"], 64)
    Vd = np.asarray(v, np.float64)
    scale = 1.0 / math.sqrt(w.d)
    Lq, Lk = Qd.shape[0], Kd.shape[0]
    for i, (r0, r1) in enumerate(oracle.block_rows(Lq, 128)):
        K2, V2 = Kd.copy(), Vd.copy()
        for j, (t0, t1) in enumerate(oracle.block_rows(Lk, 64)):
            if keep[i, j]:
                continue
            spans = [(t0, t1)] if mode == 1 else [(t0, min(t1, t0 + 32)), (min(t1, t0 + 32), t1)]
            for g0, g1 in spans:
                if g1 > g0:
                    K2[g0:g1] = Kd[g0:g1].mean(axis=0)
                    V2[g0:g1] = Vd[g0:g1].mean(axis=0)
        ref = _sdpa(Qd[r0:r1], K2, V2, scale)
        assert np.abs(O[r0:r1] - ref).max() <= 1e-10, (i, np.abs(O[r0:r1] - ref).max())


@pytest.mark.parametrize("mode", [1, 2])
def test_identical_token_block_same_kept_or_skipped(mode):
    w, q, k, v = _head("ragged_pe")
    k = k.copy(); v = v.copy()
    k[320:384] = k[320]                 # key block 5: 64 identical tokens
    v[320:384] = v[320]
    r = oracle.route_head(q, k, 1.0)
    keep = r["keep"].copy()
    keep[:, 5] = True
    O1, l1 = oracle.sol_attention_head(r["q8"], r["q_scale"], r["k8"], r["k_scale"], v, keep, mode)
    keep[:, 5] = False
    O2, l2 = oracle.sol_attention_head(r["q8"], r["q_scale"], r["k8"], r["k_scale"], v, keep, mode)
    assert np.abs(O1 - O2).max() <= 1e-12
    assert np.abs(l1 - l2).max() <= 1e-12


def test_mask_entry_matches_token_level_masked_dense():
    w, q, k, v = _head("lcsa_small")
    r = oracle.route_head(q, k, -math.inf)
    logical = oracle.lcsa_mask(w.Lq, w.Lk, w.frame_tokens, w.lcsa_window)
    allowed = oracle.physical_allowed(logical, w.nKB)
    O, lse = oracle.masked_attention_head(r["q8"], r["q_scale"], r["k8"], r["k_scale"], v, allowed)
    Lq, Lk = w.Lq, w.Lk
    tok = np.zeros((Lq, Lk), bool)
    for i in range(logical.shape[0]):
        for x in range(logical.shape[1]):
            if logical[i, x]:
                tok[128 * i:128 * i + 128, 128 * x:128 * x + 128] = True
    ref = _sdpa(_dequant(r["q8"], r["q_scale"], 128), _dequant(r["k8"], r["k_scale"], 64), v,
                1.0 / math.sqrt(w.d), tok)
    assert np.abs(O - ref).max() <= 1e-12


def test_mask_all_ones_is_dense_and_empty_row_is_zero():
    w, q, k, v = _head("cross")
    r = oracle.route_head(q, k, -math.inf)
    nQB, nLK = w.nQB, w.nLK
    ones = np.ones((nQB, nLK), np.uint8)
    ones[2] = 0                                    # query block 2 sees nothing
    allowed = oracle.physical_allowed(ones, w.nKB)
    O, lse = oracle.masked_attention_head(r["q8"], r["q_scale"], r["k8"], r["k_scale"], v, allowed)
    Od, _ = oracle.sol_attention_head(r["q8"], r["q_scale"], r["k8"], r["k_scale"], v,
                                      np.ones((nQB, w.nKB), bool), 0)
    rows = np.r_[0:256, 384:w.Lq]
    assert np.abs(O[rows] - Od[rows]).max() == 0
    assert (O[256:384] == 0).all() and np.isneginf(lse[256:384]).all()


def test_physical_allowed_maps_logical_pairs():
    logical = np.array([[1, 0, 1], [0, 1, 0]], np.uint8)
    phys = oracle.physical_allowed(logical, 5)     # 5 physical = ceil(300/64) for Lk = 300
    assert phys.astype(int).tolist() == [[1, 1, 0, 0, 1], [0, 0, 1, 1, 0]]


def test_softmax_scale_argument():
    w, q, k, v = _head("cross")
    r = oracle.route_head(q, k, -math.inf)
    O, _ = oracle.sol_attention_head(r["q8"], r["q_scale"], r["k8"], r["k_scale"], v, r["keep"], 1,
                                     softmax_scale=0.05)
    ref = _sdpa(_dequant(r["q8"], r["q_scale"], 128), _dequant(r["k8"], r["k_scale"], 64), v, 0.05)
    assert np.abs(O - ref).max() <= 1e-12


# ------------------------------------------------------------ LCSA geometry
def test_lcsa_mask_density_closed_form():
    # 8 frames of 1536 tokens (12 logical blocks each), window 2: a query block in
    # frame f sees 12*(min(f, 2) + 1) key blocks, 144*(1 + 2 + 3*6) = 3024 of 96*96
    m = oracle.lcsa_mask(12288, 12288, 1536, 2)
    assert m.shape == (96, 96)
    assert int(m.sum()) == 3024 and int(m.sum()) * 64 == 21 * 96 * 96
    # window 0: only the block-diagonal frame squares
    assert int(oracle.lcsa_mask(12288, 12288, 1536, 0).sum()) == 8 * 12 * 12


def test_lcsa_mask_token_level_brute_force():
    # a logical block takes the frame of its first token; compare with an
    # enumeration over token positions for ragged geometries
    rng = np.random.default_rng(3)
    for _ in range(20):
        Lq, Lk = int(rng.integers(1, 1500)), int(rng.integers(1, 1500))
        F = int(rng.integers(1, 700))
        win = int(rng.integers(0, 4))
        m = oracle.lcsa_mask(Lq, Lk, F, win)
        first_q = list(range(0, Lq, 128))
        first_k = list(range(0, Lk, 128))
        for a, tq in enumerate(first_q):
            for b, tk in enumerate(first_k):
                frame_q, frame_k = tq // F, tk // F
                want = frame_k <= frame_q and frame_q - frame_k <= win
                assert bool(m[a, b]) == want


def test_lcsa_mask_is_causal_and_window_monotone():
    m1 = oracle.lcsa_mask(4000, 4000, 384, 1)
    m3 = oracle.lcsa_mask(4000, 4000, 384, 3)
    frame = (128 * np.arange(m1.shape[0])) // 384
    later = frame[None, :] > frame[:, None]      # key block in a later frame than the query block
    assert (m1[later] == 0).all() and (m3[later] == 0).all()
    assert m1[frame[None, :] == frame[:, None]].all()   # the whole own frame is visible
    assert (m1 <= m3).all() and m3.sum() > m1.sum()
    assert m1.diagonal().all()                  # every block sees its own frame
    with pytest.raises(ValueError):
        oracle.lcsa_mask(100, 100, 0, 1)


# ---------------------------------------------------------------- virtual K/V, residual mode
def _virtual_case(name, b=0, h=0):
    w = workloads.get(name)
    q, k, v = (t.float().numpy() for t in workloads.head_qkv(w, b, h))
    ks, vs = (t.float().numpy() for t in workloads.source_kv(w, b, h))
    r = oracle.route_head(q, k, -math.inf)
    ks8, kss = oracle.quantize_blocks(ks, 64)
    return w, r, v, ks8, kss, vs


def _materialised(w, r, v, ks8, kss, vs, src_map, mode, replace_by_mean):
    """Dequantised [physical ; virtual slices] K and V, virtual rows optionally mean-replaced per group."""
    T = w.slice_tokens
    Kd = _dequant(r["k8"], r["k_scale"], 64)
    Ksd = _dequant(ks8, kss, 64)
    Ks, Vs = [Kd], [np.asarray(v, np.float64)]
    for s in src_map:
        kk = Ksd[s * T:(s + 1) * T].copy()
        vv = np.asarray(vs[s * T:(s + 1) * T], np.float64).copy()
        if replace_by_mean:
            g = 64 // mode
            for g0 in range(0, T, g):
                kk[g0:g0 + g] = kk[g0:g0 + g].mean(axis=0)
                vv[g0:g0 + g] = vv[g0:g0 + g].mean(axis=0)
        Ks.append(kk)
        Vs.append(vv)
    return np.concatenate(Ks), np.concatenate(Vs)


def test_virtual_residual_without_virtual_slices_is_dense():
    w, r, v, ks8, kss, vs = _virtual_case("virtual_ragged")
    O, lse = oracle.virtual_kv_residual_head(r["q8"], r["q_scale"], r["k8"], r["k_scale"], v,
                                             ks8, kss, vs, w.slice_tokens, (), w.centroid_mode)
    ref = _sdpa(_dequant(r["q8"], r["q_scale"], 128), _dequant(r["k8"], r["k_scale"], 64), v,
                1.0 / math.sqrt(w.d))
    assert np.abs(O - ref).max() <= 1e-12


@pytest.mark.parametrize("name,mode", [("virtual_small", 2), ("virtual_small", 1),
                                       ("virtual_ragged", 2), ("virtual_ragged", 1)])
def test_virtual_residual_equals_dense_over_mean_replaced_virtual_context(name, mode):
    # each centroid group of a virtual slice is |g| equal keys at its mean: exactly the ln|g| term
    w, r, v, ks8, kss, vs = _virtual_case(name, 0, 1)
    O, lse = oracle.virtual_kv_residual_head(r["q8"], r["q_scale"], r["k8"], r["k_scale"], v,
                                             ks8, kss, vs, w.slice_tokens, w.virtual_map, mode)
    K2, V2 = _materialised(w, r, v, ks8, kss, vs, w.virtual_map, mode, True)
    Qd = _dequant(r["q8"], r["q_scale"], 128)
    scale = 1.0 / math.sqrt(w.d)
    assert np.abs(O - _sdpa(Qd, K2, V2, scale)).max() <= 1e-10
    lg = scale * Qd @ K2.T
    assert np.abs(lse - torch.logsumexp(torch.from_numpy(lg), dim=1).numpy()).max() <= 1e-10


@pytest.mark.parametrize("mode", [1, 2])
def test_virtual_residual_of_identical_token_groups_is_exact_materialisation(mode):
    # a source whose groups hold identical tokens: the residual mode equals attention over the
    # materialised seven-slice context, with no approximation at all
    w = workloads.get("virtual_ragged")
    q, k, v = (t.float().numpy() for t in workloads.head_qkv(w, 1, 0))
    ks, vs = (t.float().numpy().copy() for t in workloads.source_kv(w, 1, 0))
    g = 64 // mode
    for g0 in range(0, ks.shape[0], g):
        ks[g0:g0 + g] = ks[g0]
        vs[g0:g0 + g] = vs[g0]
    r = oracle.route_head(q, k, -math.inf)
    ks8, kss = oracle.quantize_blocks(ks, 64)
    src_map = (1, 0, 1)
    O, _ = oracle.virtual_kv_residual_head(r["q8"], r["q_scale"], r["k8"], r["k_scale"], v,
                                           ks8, kss, vs, w.slice_tokens, src_map, mode)
    K2, V2 = _materialised(w, r, v, ks8, kss, vs, src_map, mode, False)
    ref = _sdpa(_dequant(r["q8"], r["q_scale"], 128), K2, V2, 1.0 / math.sqrt(w.d))
    assert np.abs(O - ref).max() <= 1e-10


def test_virtual_residual_map_order_does_not_matter_and_each_slice_counts():
    w, r, v, ks8, kss, vs = _virtual_case("virtual_small")
    args = (r["q8"], r["q_scale"], r["k8"], r["k_scale"], v, ks8, kss, vs, w.slice_tokens)
    O1, l1 = oracle.virtual_kv_residual_head(*args, (0, 1, 1), 2)
    O2, l2 = oracle.virtual_kv_residual_head(*args, (1, 0, 1), 2)
    O3, _ = oracle.virtual_kv_residual_head(*args, (0, 1), 2)
    assert np.abs(O1 - O2).max() <= 1e-12 and np.abs(l1 - l2).max() <= 1e-12
    assert np.abs(O1 - O3).max() > 1e-4      # a repeated slice adds its terms again


def test_virtual_residual_rejects_bad_geometry():
    w, r, v, ks8, kss, vs = _virtual_case("virtual_small")
    args = (r["q8"], r["q_scale"], r["k8"], r["k_scale"], v, ks8, kss, vs)
    with pytest.raises(ValueError):
        oracle.virtual_kv_residual_head(*args, 100, (0,))
    with pytest.raises(ValueError):
        oracle.virtual_kv_residual_head(*args, 320, (2,))
    with pytest.raises(ValueError):
        oracle.virtual_kv_residual_head(*args, 256, (0,))
