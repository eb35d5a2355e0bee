"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small workloads are compared in full (every head, every query block); the
five method configurations run at full size in the launch configuration the
bench times, and are compared on sampled heads (all rows of their routing,
bit-exact) and sampled query blocks (attention outputs).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import (Report, assert_band_small, assert_within, compare_rows, head_np, inputs, lcsa_input_mask, masked_parity,
                    masked_parity_v8, q_rows, sol_parity, to_np, topk_parity, virtual_parity)

pytestmark = pytest.mark.gpu

SMALL_SOL = [("ragged_pe", 0.5), ("ragged_pe", 1.0), ("ragged_pe_2x32", 1.0), ("ragged_d64", 0.5),
             ("cross", 1.0), ("prefix_small", 1.0), ("tiny", 1.0)]


@pytest.mark.parametrize("name,tau", SMALL_SOL)
def test_sol_small_full_compare(gpu_lib, name, tau):
    w = workloads.get(name)
    _, _, _, rep = sol_parity(gpu_lib, w, tau)
    assert_within(rep, f"{name} tau={tau}")
    print(f"{name} tau={tau}: {rep}")


@pytest.mark.parametrize("mode", [1, 2])
def test_sol_dense_limit_tau_neginf(gpu_lib, mode):
    w = workloads.get("ragged_pe")
    route, out, lse, rep = sol_parity(gpu_lib, w, -math.inf, centroid_mode=mode)
    assert bool((route.kept_mask == 1).all())
    assert_within(rep, "tau=-inf")


def test_sol_high_tau_centroid_heavy(gpu_lib):
    w = workloads.get("ragged_pe_2x32")
    route, out, lse, rep = sol_parity(gpu_lib, w, 2.5)
    assert_within(rep, "tau=2.5")


def _zero_blocks(w):
    """The workload's inputs with an all-zero query block (rows 128..255 of head (0, 0)) and an
    all-zero key block (rows 64..127 of heads (0, 0) and (0, 1)): scale 0, every code 0."""
    Q, K, V = workloads.batch_qkv(w)
    Q[0, 0, 128:256] = 0
    K[0, 0, 64:128] = 0
    K[0, 1, 64:128] = 0
    return Q, K, V


@pytest.mark.parametrize("name,tau", [("ragged_pe", 1.0), ("ragged_pe", -math.inf), ("ragged_pe_2x32", 1.0),
                                      ("ragged_pe_2x32", -1.0)])
def test_sol_zero_q_and_k_blocks(gpu_lib, name, tau):
    # A zero Q block has scale 0: its logits are all 0 (every routed score ties, so the row keeps
    # every block) and the kernel's logit factor is 0 for every tile. A zero K block has scale 0:
    # its score is 0, and it enters exactly (factor 0) when kept, or through a centroid of key 0
    # when skipped.
    w = workloads.get(name)
    qkv = _zero_blocks(w)
    route, out, lse, rep = sol_parity(gpu_lib, w, tau, qkv=qkv)
    assert_within(rep, f"{name} zero blocks tau={tau}")
    assert float(route.q_scale[0, 0, 1]) == 0.0 and float(route.k_scale[0, 0, 1]) == 0.0
    assert bool((route.kept_mask[0, 0, 1] == 1).all())          # the zero query block keeps every block
    print(f"{name} zero blocks tau={tau}: {rep}")


def test_masked_zero_q_and_k_blocks(gpu_lib):
    w = workloads.get("cross")
    qkv = _zero_blocks(w)
    m = np.ones((w.B, w.H, w.nQB, w.nLK), np.uint8)
    m[0, 0, 2, :] = 0
    out, lse, rep = masked_parity(gpu_lib, w, torch.from_numpy(m), qkv=qkv)
    assert_within(rep, "mask entry zero blocks")


@pytest.mark.parametrize("mag", [1e-35, 3e-38])
def test_sol_tiny_scales_take_the_exact_division(gpu_lib, mag):
    # A block whose amax puts s = fl(amax/127) below 2^-120 (1e-35: a normal scale near 2^-121;
    # 3e-38: a subnormal scale) is quantised by IEEE division, element by element.
    w = workloads.get("ragged_pe")
    Q, K, V = workloads.batch_qkv(w)
    K[0, 0, 128:192] = (K[0, 0, 128:192].float() * mag).to(torch.bfloat16)
    Q[1, 2, 256:384] = (Q[1, 2, 256:384].float() * mag).to(torch.bfloat16)
    K[1, 2, 960:1000] = (K[1, 2, 960:1000].float() * mag).to(torch.bfloat16)    # the 40-row tail block
    route, out, lse, rep = sol_parity(gpu_lib, w, 1.0, qkv=(Q, K, V))
    assert_within(rep, f"tiny scales {mag}")
    s = float(route.k_scale[0, 0, 2])
    assert 0.0 < s < 2.0 ** -120


def test_sol_all_equal_routed_row_keeps_every_block(gpu_lib):
    # Identical keys make every routed score of a row equal (Lk = 2048 is a whole number of key
    # blocks, so no tail block differs): max == min, and the row keeps every block whatever tau
    # (T = -inf in the row statistics; sigma is 0 up to the rounding of the mean).
    w = workloads.get("tiny")
    Q, K, V = workloads.batch_qkv(w)
    K = K[:, :, :1, :].expand_as(K).contiguous()
    for tau in (1.0, 1.5):
        route, out, lse, rep = sol_parity(gpu_lib, w, tau, qkv=(Q, K, V))
        assert_within(rep, f"all-equal rows tau={tau}")
        assert bool((route.kept_mask == 1).all())
        st = route.row_stats.cpu().numpy()
        assert np.isneginf(st[..., 2]).all()
        assert (st[..., 1] <= 1e-12 * np.abs(st[..., 0])).all()


@pytest.mark.parametrize("name,sparsity", [("ragged_pe", 0.75), ("ragged_pe_2x32", 0.5), ("ragged_d64", 0.9),
                                           ("prefix_small", 0.75), ("cross", 0.3), ("tiny", 0.0),
                                           ("ragged_pe", 1.0)])
def test_topk_small_full_compare(gpu_lib, name, sparsity):
    w = workloads.get(name)
    route, _, _, rep = topk_parity(gpu_lib, w, sparsity)
    assert_within(rep, f"{name} top-k sparsity={sparsity}")
    print(f"{name} top-k sparsity={sparsity}: {rep}")


def test_topk_ties_broken_by_index(gpu_lib):
    # all-equal K rows: every routed score of a row ties, so the kept set is the
    # k lowest routed indices
    w = workloads.get("ragged_pe")
    Q, K, _ = inputs(w)
    K = K[:, :, :1, :].expand_as(K).contiguous()
    r = gpu_lib.sparse_attn_route_topk(Q, K, 0.75)
    torch.cuda.synchronize()
    k = oracle.topk_keep_count(w.nKB, 0.75)
    m = r.kept_mask.cpu().numpy().astype(bool)
    # the tail block has fewer rows and so a different score; the others tie
    q, kk, _ = head_np(w, 0, 0)
    ref = oracle.route_head(q, to_np(K[0, 0].float()), 1.0)
    keep, _ = oracle.topk_route(ref["scores"], 0.75)
    assert np.array_equal(m[0, 0], keep)
    assert (m.sum(axis=3) == k).all()


def test_masked_small_lcsa(gpu_lib):
    w = workloads.get("lcsa_small")
    _, _, rep = masked_parity(gpu_lib, w, lcsa_input_mask(w))
    assert_within(rep, "lcsa_small")


@pytest.mark.parametrize("Lq,Lk,F,win,batch", [(12288, 12288, 1536, 2, 1), (1000, 1304, 300, 1, 2),
                                               (4000, 700, 128, 0, 1), (129, 5000, 1, 3, 3)])
def test_lcsa_device_mask_matches_oracle(gpu_lib, Lq, Lk, F, win, batch):
    m = gpu_lib.build_lcsa_mask(Lq, Lk, F, win, batch=batch)
    torch.cuda.synchronize()
    ref = oracle.lcsa_mask(Lq, Lk, F, win)
    got = m.cpu().numpy()
    assert got.shape == (batch, 1) + ref.shape
    for b in range(batch):
        assert np.array_equal(got[b, 0], ref)


def test_masked_small_lcsa_device_mask(gpu_lib):
    # the mask path end to end with the device-built mask
    w = workloads.get("lcsa_small")
    m = gpu_lib.build_lcsa_mask(w.Lq, w.Lk, w.frame_tokens, w.lcsa_window, batch=w.B).cpu()
    assert np.array_equal(m[0, 0].numpy(), oracle.lcsa_mask(w.Lq, w.Lk, w.frame_tokens, w.lcsa_window))
    _, _, rep = masked_parity(gpu_lib, w, m)
    assert_within(rep, "lcsa_small device mask")


def test_masked_v8_small_lcsa(gpu_lib):
    w = workloads.get("lcsa_small")
    _, _, rep = masked_parity_v8(gpu_lib, w, lcsa_input_mask(w))
    assert_within(rep, "lcsa_small INT8 V")


@pytest.mark.parametrize("name", ["cross", "ragged_d64"])
def test_masked_v8_random_mask_zero_block_and_empty_rows(gpu_lib, name):
    w = workloads.get(name)
    rng = np.random.default_rng(9)
    m = (rng.random((w.B, w.H, w.nQB, w.nLK)) < 0.45).astype(np.uint8)
    m[0, 0, 1, :] = 0                       # a query block with nothing allowed
    m[0, 0, 0, :] = 1
    _, _, V = inputs(w)
    V[0, 0, 64:128] = 0                     # an all-zero V block: scale 0
    out, lse, rep = masked_parity_v8(gpu_lib, w, torch.from_numpy(m), softmax_scale=0.09, V=V)
    assert_within(rep, f"{name} INT8 V")
    assert bool((out[0, 0, 128:256] == 0).all()) and bool(torch.isneginf(lse[0, 0, 128:256]).all())


def test_masked_per_head_random_mask_with_empty_rows(gpu_lib):
    w = workloads.get("cross")
    rng = np.random.default_rng(5)
    m = (rng.random((w.B, w.H, w.nQB, w.nLK)) < 0.4).astype(np.uint8)
    m[0, 1, 2, :] = 0                       # a query block with nothing allowed
    m[1, 0, :, :] = 1                       # a head with everything allowed
    out, lse, rep = masked_parity(gpu_lib, w, torch.from_numpy(m), softmax_scale=0.07)
    assert_within(rep, "random per-head mask")
    assert bool((out[0, 1, 256:384] == 0).all())
    assert bool((out[0, 1, :256] != 0).any())
    assert bool(torch.isneginf(lse[0, 1, 256:384]).all())


def _order_edge_mask(w, rng):
    """Per-head masks that put the attention kernel's kept-tile order at its edges. Its kept tiles
    start at the first allowed block at or after the query block's own keys (the key block at the
    middle of its rows, sequence ends aligned) and wrap round, so: every allowed block before
    that anchor (the walk starts at the last one), every allowed block after it (no wrap), one far
    block alone, everything (the ragged tail block in the middle of the walk) and a random mask."""
    nLK = -(-w.Lk // 128)
    m = np.zeros((w.B, w.H, w.nQB, nLK), dtype=np.uint8)
    patterns = ["past", "future", "single", "all", "random", "past_incl"]
    k = 0
    for b in range(w.B):
        for h in range(w.H):
            pat = patterns[k % len(patterns)]
            k += 1
            for i in range(w.nQB):
                kc = min(max((128 * i + 64 + w.Lk - w.Lq) // 128, 0), nLK - 1)
                if pat == "past":
                    m[b, h, i, :kc] = 1
                elif pat == "past_incl":
                    m[b, h, i, :kc + 1] = 1
                elif pat == "future":
                    m[b, h, i, kc + 1:] = 1
                elif pat == "single":
                    m[b, h, i, (kc + nLK // 2) % nLK] = 1
                elif pat == "all":
                    m[b, h, i, :] = 1
                else:
                    m[b, h, i] = rng.random(nLK) < 0.5
    return m


@pytest.mark.parametrize("name", ["ragged_pe", "cross", "ragged_d64"])
def test_masked_kept_order_edges(gpu_lib, name):
    w = workloads.get(name)
    m = _order_edge_mask(w, np.random.default_rng(11))
    out, lse, rep = masked_parity(gpu_lib, w, torch.from_numpy(m), softmax_scale=0.09)
    assert_within(rep, f"kept-order edges ({name})")
    empty = m.sum(axis=3) == 0              # e.g. the first query block of a "past" head
    for b, h, i in zip(*np.nonzero(empty)):
        assert bool(torch.isneginf(lse[b, h, 128 * i:min(w.Lq, 128 * i + 128)]).all())


def test_deterministic_repeat(gpu_lib):
    w = workloads.get("ragged_pe_2x32")
    Q, K, V = inputs(w)
    r1 = gpu_lib.sparse_attn_route(Q, K, 1.0)
    o1 = gpu_lib.sparse_attn_fwd(r1, V, 2).clone()
    r2 = gpu_lib.sparse_attn_route(Q, K, 1.0)
    o2 = gpu_lib.sparse_attn_fwd(r2, V, 2)
    torch.cuda.synchronize()
    assert torch.equal(r1.kept_mask, r2.kept_mask)
    assert torch.equal(o1, o2)


def test_device_timeout_is_reported_and_context_survives(gpu_lib):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    gpu_lib.selftest_timeout(ws, 2_000_000)          # a 2 ms wait that nothing completes
    with pytest.raises(gpu_lib.BsvaError) as e:
        gpu_lib.check_status(ws)
    assert e.value.code == 5
    gpu_lib.check_status(ws)                         # cleared
    w = workloads.get("ragged_d64")                  # the context still works
    _, _, _, rep = sol_parity(gpu_lib, w, 0.5, heads=[(0, 0)])
    assert_within(rep, "after timeout")


def test_binding_rejects_bad_inputs(gpu_lib):
    q = torch.zeros((1, 1, 256, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gpu_lib.BsvaError) as e:
        gpu_lib.sparse_attn_route(q, q, 1.0)
    assert e.value.code == 2
    q = torch.zeros((1, 1, 256, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gpu_lib.BsvaError):
        gpu_lib.sparse_attn_route(q, q, 1.0, n_prefix=100)


@pytest.mark.parametrize("name,mode", [("virtual_small", 2), ("virtual_small", 1), ("virtual_ragged", 2),
                                       ("virtual_ragged", 1)])
def test_virtual_kv_small_full_compare(gpu_lib, name, mode):
    w = workloads.get(name)
    _, _, rep = virtual_parity(gpu_lib, w, centroid_mode=mode)
    print(f"{name} mode={mode}: {rep}")
    assert_within(rep, f"{name} virtual K/V mode {mode}")


@pytest.mark.parametrize("src_map", [(), (1,), (0, 1) * 16])
def test_virtual_kv_map_edges(gpu_lib, src_map):
    # no virtual slice (dense exact attention), one slice, and the maximum of 32
    w = workloads.get("virtual_small")
    _, _, rep = virtual_parity(gpu_lib, w, src_map=src_map, softmax_scale=0.1)
    assert_within(rep, f"virtual K/V map {src_map}")


# ---------------------------------------------------------------- full size
def _sample_blocks(nQB, n_extra=4, seed=0):
    rng = np.random.default_rng(seed)
    base = {0, 1, nQB // 2, nQB - 1}
    base |= set(int(x) for x in rng.choice(nQB, size=n_extra, replace=False))
    return sorted(base)


@pytest.mark.slow
def test_full_lcsa_v8(gpu_lib):
    w = workloads.get("lcsa")
    heads = [(0, 0), (0, w.H - 1)]
    _, _, rep = masked_parity_v8(gpu_lib, w, lcsa_input_mask(w), heads=heads,
                                 q_blocks=_sample_blocks(w.nQB))
    assert_within(rep, "lcsa full INT8 V")


@pytest.mark.slow
def test_full_virtual_kv(gpu_lib):
    w = workloads.get("h3_virtual")
    heads = [(0, 0), (0, w.H - 1)]
    _, _, rep = virtual_parity(gpu_lib, w, heads=heads, q_blocks=_sample_blocks(w.nQB))
    print(f"h3_virtual: {rep}")
    assert_within(rep, "h3 virtual K/V residual")


@pytest.mark.slow
def test_full_lcsa(gpu_lib):
    w = workloads.get("lcsa")
    heads = [(0, 0), (0, w.H - 1)]
    _, _, rep = masked_parity(gpu_lib, w, lcsa_input_mask(w), heads=heads,
                              q_blocks=_sample_blocks(w.nQB))
    assert_within(rep, "lcsa full")


@pytest.mark.slow
@pytest.mark.parametrize("name,sparsity", [("wan14b", 0.75), ("h3", 0.75)])
def test_full_topk(gpu_lib, name, sparsity):
    # routing and quantisation of every head bit for bit; outputs on heads {0, H-1}
    w = workloads.get(name)
    _, _, _, rep = topk_parity(gpu_lib, w, sparsity, attn_heads=[(0, 0), (0, w.H - 1)],
                               q_blocks=_sample_blocks(w.nQB))
    print(f"{name} top-k sparsity={sparsity}: {rep}")
    assert_within(rep, f"{name} top-k sparsity={sparsity}")
    assert rep.blocks == w.B * w.H * w.nQB * w.nKB


@pytest.mark.slow
@pytest.mark.parametrize("name,tau", [("wan13b", 1.0), ("wan14b", 0.5), ("wan14b", 1.0), ("wan14b", 1.5),
                                      ("h3", 1.0)])
def test_full_sol(gpu_lib, name, tau):
    # routing and quantisation of every head bit for bit (band excepted and bounded); outputs on
    # heads {0, H-1} over sampled query blocks
    w = workloads.get(name)
    _, _, _, rep = sol_parity(gpu_lib, w, tau, attn_heads=[(0, 0), (0, w.H - 1)], q_blocks=_sample_blocks(w.nQB))
    print(f"{name} tau={tau}: {rep}")
    assert_within(rep, f"{name} tau={tau}")
    assert rep.blocks == w.B * w.H * w.nQB * w.nKB
    assert_band_small(rep, f"{name} tau={tau}")
