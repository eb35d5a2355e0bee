"""INT8 streaming K/V cache in 128-row slabs, and attention over it (oracle; test infrastructure only).

Source: "FlashVSR Kitchen Sparse Attention", intro: in the streaming modes the
node keeps a sliding cache of past K and V as INT8, repacks the cached K and V
into bounded 128-row slabs and hands those straight to the native sparse
kernel, without rebuilding full-precision tensors; *When it bites*: that path
needs an INT8 cache to feed. The mask is FlashVSR's logical 128-query x
128-key block mask ("FlashVSR Sparge Attention", intro and *How it works*).

Readings (the page gives the idea, not the arithmetic):

* A cache of one (batch, head) is a sliding window of at most ``capacity``
  slabs. A slab holds up to 128 consecutive tokens of one appended chunk; a
  chunk of Lc tokens becomes ceil(Lc / 128) new slabs, the last one holding
  Lc - 128 * (ceil(Lc / 128) - 1) rows when Lc is not a multiple of 128.
* Each slab's K and V are quantised with the K quantiser (64-row blocks over
  the slab's valid rows, scale = amax / 127, round half to even; ``quant``).
* When an append would exceed the capacity, the oldest slabs are evicted
  first (first in, first out).
* Attention over the cache: the keys are the valid rows of the live slabs,
  oldest slab first; one logical mask column per live slab (a slab is a
  128-key logical block); exact terms only, as in the mask entry. The logit of
  query row r and cached key t is (sq_i * sk_b * scale) * (q8[r] . k8[t]) with
  sk_b the scale of t's 64-row block, the value is v8[t] * sv_b, and a query
  block with no allowed key gets o = 0 and lse = -inf.
"""
import math

import numpy as np

from .attention import _softmax_rows, resolve_scale
from .quant import Q_ROWS, K_ROWS, block_rows, quantize_blocks

SLAB_ROWS = 128


class KVCache:
    """Sliding INT8 K/V cache of one (batch, head): a list of live slabs, oldest first.

    Each slab is a dict with k8, v8 (int8 [n, d]), k_scale, v_scale (float32, one per
    64-row block of the slab's n valid rows) and n.
    """

    def __init__(self, capacity: int):
        if capacity < 1:
            raise ValueError("capacity must be >= 1 slab")
        self.capacity = capacity
        self.slabs = []
        self.evicted = 0          # slabs dropped so far

    def append(self, k, v):
        """Quantise a chunk (k, v: [Lc, d], values exactly representable in fp32) into new slabs."""
        k = np.asarray(k, dtype=np.float32)
        v = np.asarray(v, dtype=np.float32)
        if k.shape != v.shape or k.ndim != 2 or k.shape[0] < 1:
            raise ValueError("k and v must be non-empty [Lc, d] of the same shape")
        for t0, t1 in block_rows(k.shape[0], SLAB_ROWS):
            k8, ks = quantize_blocks(k[t0:t1], K_ROWS)
            v8, vs = quantize_blocks(v[t0:t1], K_ROWS)
            self.slabs.append(dict(k8=k8, k_scale=ks, v8=v8, v_scale=vs, n=t1 - t0))
        while len(self.slabs) > self.capacity:
            self.slabs.pop(0)
            self.evicted += 1

    @property
    def rows(self):
        """Valid rows of each live slab, oldest first."""
        return [s["n"] for s in self.slabs]

    def keys(self):
        """The live cache as one sequence: (k8, k_scale per row, v8, v_scale per row, slab of each row)."""
        k8 = np.concatenate([s["k8"] for s in self.slabs])
        v8 = np.concatenate([s["v8"] for s in self.slabs])
        ks = np.concatenate([np.repeat(s["k_scale"], [b - a for a, b in block_rows(s["n"], K_ROWS)])
                             for s in self.slabs])
        vs = np.concatenate([np.repeat(s["v_scale"], [b - a for a, b in block_rows(s["n"], K_ROWS)])
                             for s in self.slabs])
        slab = np.concatenate([np.full(s["n"], x) for x, s in enumerate(self.slabs)])
        return k8, ks, v8, vs, slab


def cache_attention_head(q8, q_scale, cache: KVCache, mask, softmax_scale: float = 0.0, q_blocks=None):
    """Attention of one head's quantised queries over its cache.

    mask: [nQB, n_live_slabs] (nonzero = allowed). Returns (O fp64 [Lq, d], lse fp64 [Lq]);
    rows of query blocks outside ``q_blocks`` stay NaN.
    """
    Lq, d = q8.shape
    mask = np.asarray(mask).astype(bool)
    if mask.shape != (-(-Lq // Q_ROWS), len(cache.slabs)):
        raise ValueError("mask must be [query blocks, live slabs]")
    scale = resolve_scale(d, softmax_scale)
    O = np.full((Lq, d), np.nan)
    lse = np.full(Lq, np.nan)
    qspans = block_rows(Lq, Q_ROWS)
    for i in (range(len(qspans)) if q_blocks is None else q_blocks):
        r0, r1 = qspans[i]
        Qi = q8[r0:r1].astype(np.float64)
        logits, values = [], []
        for x, s in enumerate(cache.slabs):
            if not mask[i, x]:
                continue
            for b, (t0, t1) in enumerate(block_rows(s["n"], K_ROWS)):
                dots = Qi @ s["k8"][t0:t1].astype(np.float64).T        # exact integer dots
                logits.append((float(q_scale[i]) * float(s["k_scale"][b]) * scale) * dots)
                values.append(s["v8"][t0:t1].astype(np.float64) * float(s["v_scale"][b]))
        if not logits:
            O[r0:r1] = 0.0
            lse[r0:r1] = -math.inf
            continue
        O[r0:r1], lse[r0:r1] = _softmax_rows(np.concatenate(logits, axis=1), np.concatenate(values, axis=0))
    return O, lse
