"""GPU parity of the INT8 streaming K/V cache in 128-row slabs, through the C ABI.

A stream of appends (whole slabs, a ragged chunk, evictions, a chunk longer
than the ring) is run on the GPU and on the oracle's cache from the same bf16
chunks. After every append the GPU ring (codes, scales, valid rows, oldest
slot, live count) must equal the oracle's live slabs bit for bit; the mask
entry over the cache must match the oracle's attention over the same slabs
within the parity tolerances, every head and query block, with a per-head
random mask that leaves one query block empty.
"""
import math

import numpy as np
import pytest
import torch

from oracle.kv_cache import KVCache as OracleCache, cache_attention_head
from parity import Report, assert_within, compare_rows, q_rows, to_np

pytestmark = pytest.mark.gpu


def _bf16(rng, shape):
    return torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(torch.bfloat16)


def _check_ring(gpu, ref_caches, B, H):
    c = gpu.c
    n_live = len(ref_caches[0][0].slabs)
    assert c.count == n_live
    rows = to_np(gpu.slab_rows)
    k8, v8 = to_np(gpu.k8), to_np(gpu.v8)
    ks, vs = to_np(gpu.k_scale), to_np(gpu.v_scale)
    for x in range(n_live):
        slot = (c.first + x) % c.n_slots
        n = ref_caches[0][0].slabs[x]["n"]
        assert rows[slot] == n, f"slab {x}: rows {rows[slot]} != {n}"
        for b in range(B):
            for h in range(H):
                s = ref_caches[b][h].slabs[x]
                assert np.array_equal(k8[b, h, slot * 128:slot * 128 + n], s["k8"]), f"k8 slab {x} ({b},{h})"
                assert np.array_equal(v8[b, h, slot * 128:slot * 128 + n], s["v8"]), f"v8 slab {x} ({b},{h})"
                nb = len(s["k_scale"])
                assert np.array_equal(ks[b, h, 2 * slot:2 * slot + nb], s["k_scale"]), f"k_scale slab {x}"
                assert np.array_equal(vs[b, h, 2 * slot:2 * slot + nb], s["v_scale"]), f"v_scale slab {x}"


def _attend_and_compare(bsva, gpu, ref_caches, Q, rng, softmax_scale):
    B, H, Lq, d = Q.shape
    nQB = -(-Lq // 128)
    qq = bsva.quantize_q(Q.cuda())
    m = (rng.random((B, H, nQB, gpu.count)) < 0.6).astype(np.uint8)
    m[0, 0, min(1, nQB - 1), :] = 0                     # a query block with nothing allowed
    m[B - 1, H - 1, 0, :] = 1                           # one with the whole window
    out, lse = gpu.attend(qq, torch.from_numpy(m).cuda(), softmax_scale=softmax_scale, with_lse=True,
                          out_dtype=torch.float32)
    out16 = gpu.attend(qq, torch.from_numpy(m).cuda(), softmax_scale=softmax_scale)
    torch.cuda.synchronize()
    assert torch.equal(out16, out.to(torch.bfloat16))
    q8, qs = to_np(qq["q8"]), to_np(qq["q_scale"])
    rep = Report()
    for b in range(B):
        for h in range(H):
            O_ref, lse_ref = cache_attention_head(q8[b, h], qs[b, h], ref_caches[b][h], m[b, h], softmax_scale)
            compare_rows(to_np(out[b, h].float()), to_np(lse[b, h]), O_ref, lse_ref, q_rows(Lq, range(nQB)), rep)
    assert_within(rep, "INT8 K/V cache attention")
    e = min(1, nQB - 1)
    assert bool((out[0, 0, 128 * e:128 * e + 128] == 0).all())
    return rep


@pytest.mark.parametrize("d,n_slots,chunks", [
    (128, 6, [256, 200, 384, 128, 70, 900]),      # whole slabs, ragged chunks, evictions, a chunk > the ring
    (64, 3, [128, 64, 300, 40]),
])
def test_streaming_appends_match_the_oracle(gpu_lib, d, n_slots, chunks):
    bsva = gpu_lib
    B, H = 2, 3
    rng = np.random.default_rng(d + n_slots)
    gpu = bsva.KVCache(B, H, d, n_slots)
    ref = [[OracleCache(n_slots) for _ in range(H)] for _ in range(B)]
    for step, Lc in enumerate(chunks):
        K, V = _bf16(rng, (B, H, Lc, d)), _bf16(rng, (B, H, Lc, d))
        gpu.append(K.cuda(), V.cuda())
        for b in range(B):
            for h in range(H):
                ref[b][h].append(K[b, h].float().numpy(), V[b, h].float().numpy())
        torch.cuda.synchronize()
        _check_ring(gpu, ref, B, H)
        Q = _bf16(rng, (B, H, 300, d))
        rep = _attend_and_compare(bsva, gpu, ref, Q, rng, 0.0 if step % 2 else 0.09)
        print(f"d={d} append {step} (Lc={Lc}): live {gpu.count} slabs from slot {gpu.first}, {rep}")


def test_cache_rejects_bad_arguments(gpu_lib):
    bsva = gpu_lib
    gpu = bsva.KVCache(1, 2, 128, 2)
    k = torch.zeros((1, 2, 64, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        gpu.append(k, k)
    qq = bsva.quantize_q(torch.zeros((1, 2, 128, 128), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(bsva.BsvaError):                 # an empty cache has nothing to attend to
        lib = bsva.load()
        import ctypes
        ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
        rc = lib.masked_block_attn_fwd_kvcache(ctypes.byref(gpu.c), 128, ctypes.c_void_p(qq["q8"].data_ptr()),
                                               ctypes.c_void_p(qq["q_scale"].data_ptr()),
                                               ctypes.c_void_p(ws.data_ptr()), 1, ctypes.c_float(0), 0,
                                               ctypes.c_void_p(ws.data_ptr()), None, ctypes.c_void_p(ws.data_ptr()),
                                               ws.numel(), None)
        bsva._check(rc)
