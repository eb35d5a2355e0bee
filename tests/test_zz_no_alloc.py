"""The workspace-free mask entry, called through the C ABI.

``masked_block_attn_fwd_noalloc`` serves callers that cannot allocate device
memory (a plugin whose host application's allocator owns the device, or a
streaming path that must not call cudaMalloc because it can synchronise the
device): its kept-block lists live in a scratch array built into the library.
This test runs two calls in a row with different inputs and masks, so that a
result left over in the shared scratch from the first call would show up in
the second, and checks each against ``masked_block_attn_fwd`` with a caller
workspace and against the fp64 oracle (every head, every query block), within
the tolerances the parity tests use. It is collected last and needs no state
from other tests.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import Report, assert_within, compare_rows, head_np, lcsa_input_mask, q_rows, to_np

pytestmark = pytest.mark.gpu

ATOL, REL_L2 = 1e-2, 5e-3


def _noalloc(lib, bsva, qk, v, mask, out_dtype=torch.float32):
    B, H, Lq, d = qk["q8"].shape
    Lk = qk["k8"].shape[2]
    out = torch.full((B, H, Lq, d), float("nan"), dtype=out_dtype, device="cuda")
    lse = torch.full((B, H, Lq), float("nan"), dtype=torch.float32, device="cuda")
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = lib.masked_block_attn_fwd_noalloc(
        bsva.Shape(B, H, Lq, Lk, d, 0), P(qk["q8"]), P(qk["q_scale"]), P(qk["k8"]), P(qk["k_scale"]), P(v),
        P(mask), mask.shape[1], ctypes.c_float(0.0), bsva.OUT_DTYPES[out_dtype], P(out), P(lse),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, lib.bsva_last_error().decode()
    return out, lse


def _check(got, ref):
    g, r = got.double(), ref.double()
    err = (g - r).abs()
    assert float(err.max()) <= ATOL
    assert float(err.norm() / r.norm()) <= REL_L2


def _check_oracle(w, out, lse, mask, what):
    """Every head and query block of one call against the oracle's masked attention."""
    rep = Report()
    Hm = mask.shape[1]
    m = mask.cpu().numpy()
    for b in range(w.B):
        for h in range(w.H):
            q, k, v = head_np(w, b, h)
            ref = oracle.route_head(q, k, -math.inf, 0)
            allowed = oracle.physical_allowed(m[b, h % Hm], w.nKB)
            O_ref, lse_ref = oracle.masked_attention_head(ref["q8"], ref["q_scale"], ref["k8"], ref["k_scale"], v,
                                                          allowed)
            compare_rows(to_np(out[b, h].float()), to_np(lse[b, h]), O_ref, lse_ref,
                         q_rows(w.Lq, range(w.nQB)), rep)
    assert_within(rep, what)


def test_noalloc_mask_entry_matches_workspace_entry_twice(gpu_lib):
    bsva = gpu_lib
    lib = bsva.load()
    # call 1: the LCSA mask shared by all heads
    w = workloads.get("lcsa_small")
    Q, K, V = [x.cuda() for x in workloads.batch_qkv(w)]
    qk = bsva.quantize_qk(Q, K)
    mask1 = lcsa_input_mask(w).cuda()
    ref1, rl1 = bsva.masked_block_attn_fwd(qk["q8"], qk["q_scale"], qk["k8"], qk["k_scale"], V, mask1,
                                           with_lse=True, out_dtype=torch.float32)
    got1, gl1 = _noalloc(lib, bsva, qk, V, mask1)
    # call 2, right after: other inputs and a sparser per-head mask with an empty row
    w2 = workloads.get("cross")
    Q2, K2, V2 = [x.cuda() for x in workloads.batch_qkv(w2)]
    qk2 = bsva.quantize_qk(Q2, K2)
    rng = np.random.default_rng(3)
    m = (rng.random((w2.B, w2.H, w2.nQB, w2.nLK)) < 0.3).astype(np.uint8)
    m[1, 1, 3, :] = 0
    mask2 = torch.from_numpy(m).cuda()
    ref2, rl2 = bsva.masked_block_attn_fwd(qk2["q8"], qk2["q_scale"], qk2["k8"], qk2["k_scale"], V2, mask2,
                                           with_lse=True, out_dtype=torch.float32)
    got2, gl2 = _noalloc(lib, bsva, qk2, V2, mask2)
    torch.cuda.synchronize()
    _check(got1, ref1)
    _check(got2, ref2)
    _check_oracle(w, got1, gl1, mask1, "no-alloc call 1 vs oracle")
    _check_oracle(w2, got2, gl2, mask2, "no-alloc call 2 vs oracle")
    fin = torch.isfinite(rl2)
    assert torch.equal(fin, torch.isfinite(gl2))
    assert float((gl2[fin] - rl2[fin]).abs().max()) <= 1e-3
    assert bool((got2[1, 1, 384:512] == 0).all())


def test_noalloc_rejects_shapes_beyond_the_scratch(gpu_lib):
    lib = gpu_lib.load()
    P = ctypes.c_void_p(0x10000)
    big = gpu_lib.Shape(1, 40, 32760, 32760, 128, 0)       # 40*256*512 list entries > 2,097,152
    rc = lib.masked_block_attn_fwd_noalloc(big, P, P, P, P, P, P, 1, ctypes.c_float(0), 0, P, None, None)
    assert rc == 3
    assert b"scratch" in lib.bsva_last_error()
