"""Pins for the oracle's INT8 streaming K/V cache in 128-row slabs (CPU only).

Independent references: the mask entry's oracle over the concatenated cache
when every slab is full (its 64-row quantisation blocks then fall on the same
rows), torch's fp64 scaled-dot-product attention with a token-level mask built
here from slab membership (ragged slabs), the quantiser's error bound, and
first-in-first-out eviction checked against a cache that only ever saw the
surviving chunks.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle.kv_cache import KVCache, cache_attention_head

D = 64


def _chunks(lengths, seed):
    rng = np.random.default_rng(seed)
    out = []
    for n in lengths:
        k = torch.from_numpy(rng.standard_normal((n, D)).astype(np.float32)).to(torch.bfloat16).float().numpy()
        v = torch.from_numpy(rng.standard_normal((n, D)).astype(np.float32)).to(torch.bfloat16).float().numpy()
        out.append((k, v))
    return out


def _queries(Lq, seed):
    rng = np.random.default_rng(seed)
    q = torch.from_numpy(rng.standard_normal((Lq, D)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    return oracle.quantize_blocks(q, 128)


def _sdpa(q, k, v, scale, mask):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))[None, None]
    o = F.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=torch.from_numpy(mask)[None, None], scale=scale)
    return o[0, 0].numpy()


def test_full_slabs_equal_the_mask_entry_over_the_concatenated_cache():
    # three chunks of whole slabs, no eviction: the cache is the concatenation of the chunks,
    # quantised in the same 64-row blocks as the mask entry's K and INT8 V
    chunks = _chunks([256, 384, 128], 1)
    c = KVCache(capacity=8)
    for k, v in chunks:
        c.append(k, v)
    assert c.rows == [128] * 6
    q8, qs = _queries(300, 2)
    rng = np.random.default_rng(3)
    mask = (rng.random((3, 6)) < 0.6).astype(np.uint8)
    mask[1] = 0                                         # a query block with nothing allowed
    O, lse = cache_attention_head(q8, qs, c, mask)
    K = np.concatenate([k for k, _ in chunks])
    V = np.concatenate([v for _, v in chunks])
    k8, ks = oracle.quantize_blocks(K, 64)
    v8, vs = oracle.quantize_blocks(V, 64)
    allowed = oracle.physical_allowed(mask, k8.shape[0] // 64)
    O2, lse2 = oracle.masked_attention_head(q8, qs, k8, ks, oracle.dequantize_blocks(v8, vs, 64), allowed)
    assert np.abs(O - O2).max() <= 1e-13
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse2))
    fin = np.isfinite(lse)
    assert np.abs(lse[fin] - lse2[fin]).max() <= 1e-12
    assert (O[128:256] == 0).all() and np.isneginf(lse[128:256]).all()


def test_ragged_slabs_equal_token_masked_dense_attention():
    # chunks of 200 and 70 tokens leave slabs of 128, 72 and 70 rows; the 72-row slab has a
    # 64-row block and an 8-row block, the 70-row slab a 64-row and a 6-row block
    chunks = _chunks([200, 70], 4)
    c = KVCache(capacity=4)
    for k, v in chunks:
        c.append(k, v)
    assert c.rows == [128, 72, 70]
    q8, qs = _queries(256, 5)
    mask = np.array([[1, 0, 1], [1, 1, 1]], np.uint8)
    scale = 0.11
    O, lse = cache_attention_head(q8, qs, c, mask, softmax_scale=scale)
    # token-level reference: every slab quantised on its own rows, keys in slab order
    kd, vd, slab = [], [], []
    for x, (k, v) in enumerate(((chunks[0][0][:128], chunks[0][1][:128]), (chunks[0][0][128:], chunks[0][1][128:]),
                                (chunks[1][0], chunks[1][1]))):
        k8, ks = oracle.quantize_blocks(k, 64)
        v8, vs = oracle.quantize_blocks(v, 64)
        kd.append(oracle.dequantize_blocks(k8, ks, 64))
        vd.append(oracle.dequantize_blocks(v8, vs, 64))
        slab += [x] * k.shape[0]
    K, V, slab = np.concatenate(kd), np.concatenate(vd), np.array(slab)
    Q = oracle.dequantize_blocks(q8, qs, 128)
    tok = mask[np.arange(256) // 128][:, slab].astype(bool)
    ref = _sdpa(Q, K, V, scale, tok)
    assert np.abs(O - ref).max() <= 1e-12
    lg = scale * Q @ K.T
    lg[~tok] = -np.inf
    assert np.abs(lse - torch.logsumexp(torch.from_numpy(lg), dim=1).numpy()).max() <= 1e-10


def test_eviction_is_first_in_first_out():
    chunks = _chunks([128, 256, 100, 128, 384], 6)
    c = KVCache(capacity=5)
    for k, v in chunks:
        c.append(k, v)
    # 1 + 2 + 1 + 1 + 3 = 8 slabs appended, the oldest 3 evicted: the survivors are the last
    # slab of chunk 2 (100 rows), chunk 3 and chunk 4
    assert c.evicted == 3 and c.rows == [100, 128, 128, 128, 128]
    fresh = KVCache(capacity=5)
    for k, v in chunks[2:]:
        fresh.append(k, v)
    for a, b in zip(c.slabs, fresh.slabs):
        for key in ("k8", "v8", "k_scale", "v_scale"):
            assert np.array_equal(a[key], b[key])


def test_slab_quantisation_error_bound_and_codes():
    (k, v), = _chunks([200], 7)
    c = KVCache(capacity=2)
    c.append(k, v)
    k8, ks_row, v8, vs_row, slab = c.keys()
    assert np.array_equal(slab, np.repeat([0, 1], [128, 72]))
    for x8, s_row, ref in ((k8, ks_row, k), (v8, vs_row, v)):
        assert np.abs(x8.astype(np.int64)).max() <= 127
        err = np.abs(x8.astype(np.float64) * s_row[:, None] - ref)
        assert (err <= s_row[:, None] * (0.5 + 1e-6)).all()
    # a block's largest magnitude maps to +-127
    for s in c.slabs:
        for b, (t0, t1) in enumerate(oracle.block_rows(s["n"], 64)):
            assert np.abs(s["k8"][t0:t1].astype(np.int64)).max() == 127


def test_all_ones_mask_is_dense_attention_over_the_window():
    chunks = _chunks([128, 128, 128], 8)
    c = KVCache(capacity=2)
    for k, v in chunks:
        c.append(k, v)
    q8, qs = _queries(128, 9)
    O, _ = cache_attention_head(q8, qs, c, np.ones((1, 2), np.uint8))
    K = np.concatenate([oracle.dequantize_blocks(*oracle.quantize_blocks(k, 64), 64) for k, _ in chunks[1:]])
    V = np.concatenate([oracle.dequantize_blocks(*oracle.quantize_blocks(v, 64), 64) for _, v in chunks[1:]])
    ref = _sdpa(oracle.dequantize_blocks(q8, qs, 128), K, V, 1.0 / math.sqrt(D), np.ones((128, 256), bool))
    assert np.abs(O - ref).max() <= 1e-12


def test_bad_mask_shape_is_rejected():
    (k, v), = _chunks([128], 10)
    c = KVCache(capacity=1)
    c.append(k, v)
    q8, qs = _queries(128, 11)
    with pytest.raises(ValueError):
        cache_attention_head(q8, qs, c, np.ones((1, 2), np.uint8))
