"""Per-block symmetric INT8 quantiser and integer sum-pools (oracle; test infrastructure only).

Source: "Configure Sol Sparse Attention", *How it works*: routing scores and
the exact path both read the same prequantized INT8 Q/K tensors. The pages
state neither the block size nor the rounding; the readings used here are:

* Q is cut into 128-row blocks, K into 64-row blocks, per (batch, head), over
  the valid rows and all d columns (the routing granularity the same passage
  gives: 128-token query blocks, 64-token K/V blocks).
* amax = max |x| over the block (exact on bf16 inputs);
  s = fl32(amax / 127) (one IEEE fp32 division);
  q = clamp(rint_half_even(fl32(x / s)), -127, 127) (one IEEE fp32 division,
  then round half to even). If amax = 0 then s = 0 and q = 0. The value -128
  never occurs.
* The two fp32 divisions define the stored artefact, so they are done in fp32
  here, not fp64.
* Pools are exact integer column sums of the INT8 rows: one per 128-row Q
  block, and per 64-row K block one per 32-row half. The halves of a tail K
  block with n valid rows are rows [0, min(32, n)) and [32, n); an empty half
  sums to zero.
* INT8 V ("FlashVSR Kitchen Sparse Attention", intro: the streaming cache
  keeps K/V as INT8 and the sparse kernel consumes it without rebuilding bf16
  tensors): V uses the K quantiser, 64-row blocks, and its dequantised value
  is x8 * s (fp64 here), the tensor the attention then weights.
"""
import numpy as np

Q_ROWS = 128
K_ROWS = 64


def block_rows(L: int, rows: int):
    """[(start, stop)] of each block of ``rows`` rows over L rows, tail clipped."""
    return [(s, min(L, s + rows)) for s in range(0, L, rows)]


def quantize_blocks(x, rows: int):
    """Quantise one head ``x`` ([L, d], values exactly representable in fp32).

    Returns (q8 int8 [L, d], scale float32 [nB]).
    """
    x = np.asarray(x, dtype=np.float32)
    L, d = x.shape
    spans = block_rows(L, rows)
    q8 = np.zeros((L, d), dtype=np.int8)
    scale = np.zeros(len(spans), dtype=np.float32)
    for b, (r0, r1) in enumerate(spans):
        blk = x[r0:r1]
        amax = np.float32(np.max(np.abs(blk)))
        s = np.float32(amax / np.float32(127.0))
        scale[b] = s
        if s == 0:
            continue
        ratio = blk / s                       # fp32 / fp32 -> fp32, IEEE RN
        q = np.rint(ratio)                    # round half to even
        q8[r0:r1] = np.clip(q, -127, 127).astype(np.int8)
    return q8, scale


def q_pools(q8):
    """Sum-pool of each 128-row Q block, int64 [nQB, d] (values fit int32)."""
    L, d = q8.shape
    spans = block_rows(L, Q_ROWS)
    out = np.zeros((len(spans), d), dtype=np.int64)
    for i, (r0, r1) in enumerate(spans):
        out[i] = q8[r0:r1].astype(np.int64).sum(axis=0)
    return out


def k_half_pools(k8):
    """Sum-pool of each 32-row half of each 64-row K block, int64 [nKB, 2, d]."""
    L, d = k8.shape
    spans = block_rows(L, K_ROWS)
    out = np.zeros((len(spans), 2, d), dtype=np.int64)
    for j, (t0, t1) in enumerate(spans):
        mid = min(t1, t0 + 32)
        out[j, 0] = k8[t0:mid].astype(np.int64).sum(axis=0)
        out[j, 1] = k8[mid:t1].astype(np.int64).sum(axis=0)
    return out


def dequantize_blocks(x8, scale, rows: int):
    """fp64 values x8 * s of a per-block INT8 tensor [L, d] with scales [nBlocks]."""
    x8 = np.asarray(x8)
    out = np.empty(x8.shape, dtype=np.float64)
    for b, (t0, t1) in enumerate(block_rows(x8.shape[0], rows)):
        out[t0:t1] = x8[t0:t1].astype(np.float64) * float(scale[b])
    return out
