"""Seeded synthetic inputs for block-sparse INT8 video attention.

This module is the one piece shared by the CPU oracle (``oracle/``) and the
CUDA path (``block_sparse_video_int8_b200``): it draws Q, K, V and records
each workload's geometry (frame size and window of the LCSA mask), and holds
none of the method's arithmetic (no quantisation, scoring, routing,
attention, and no mask rule: tests build the LCSA mask input with the oracle,
the bench with the library's device builder).

Workload shapes follow the video-diffusion settings the source pages name:
Wan-style self-attention over a frame-major latent video
("Configure Sol Sparse Attention", *How it works*), FlashVSR's LCSA streaming
mask on logical 128x128 blocks ("FlashVSR Sparge Attention", intro and
*How it works*), and an H3-style run whose conditioning prefix stays dense
("Ref2VA VSA", *2-stage attention patch*; "Configure Sol Sparse Attention",
*The inputs that matter*, prefix_policy).

Recipe (every number is a recorded parameter of the workload):

* ``normal``: Q, K, V ~ N(0, 1) in fp32, cast once to bf16 (round to nearest
  even, done by torch).
* ``pe``: video tokens in frame-major order, index ``(t*Hs + y)*Ws + x``;
  Q = 2 * PE(t, y, x) @ W + N(0, 1), K likewise with its own noise, V ~ N(0, 1).
  PE concatenates, per axis, ``[sin(p*w_k), cos(p*w_k)]`` for k = 0..7 with
  ``w_k = 10000**(-k/8)`` (16 dims per axis, 48 in all). W is one 48 x d
  Gaussian matrix with entries N(0, 1/48), seed 7, shared by Q, K and every
  head. An optional prefix of ``n_prefix`` N(0, 1) tokens precedes the video.
* Every (batch, head, tensor) draws from its own ``numpy.random.default_rng``
  stream keyed by ``[seed, b, h, tensor]``, so any single head can be rebuilt
  on its own.
"""
from __future__ import annotations

from dataclasses import dataclass, field
import math

import numpy as np
import torch

__all__ = [
    "Workload", "WORKLOADS", "get", "head_qkv", "batch_qkv", "pe_table", "W_SEED", "source_kv",
]

W_SEED = 7
_Q, _K, _V, _KS, _VS = 0, 1, 2, 3, 4


@dataclass(frozen=True)
class Workload:
    """One synthetic attention problem: shapes, generator and routing knobs."""

    name: str
    B: int
    H: int
    d: int
    Lq: int
    Lk: int
    gen: str = "normal"              # "normal" | "pe"
    grid: tuple | None = None        # (T, Hs, Ws) video latent grid for "pe"
    n_prefix: int = 0                # leading dense-protected tokens
    taus: tuple = (1.0,)             # Sol routing thresholds to run
    centroid_mode: int = 1           # 1 = 1x64, 2 = 2x32, 0 = mask entry
    mask: str | None = None          # "lcsa" for the explicit block-mask entry
    frame_tokens: int = 0            # tokens per latent frame (LCSA)
    lcsa_window: int = 2             # key frames allowed: [f_q - window, f_q]
    slice_tokens: int = 0            # virtual K/V: tokens per latent-time slice
    virtual_map: tuple = ()          # virtual K/V: source slice of each added virtual slice
    n_source_slices: int = 0         # virtual K/V: 0 = the physical K/V is the source,
                                     # else a separate N(0,1) source of this many slices
    seed: int = 0
    notes: str = field(default="", compare=False)

    @property
    def nQB(self) -> int:
        return -(-self.Lq // 128)

    @property
    def nKB(self) -> int:
        return -(-self.Lk // 64)

    @property
    def nLK(self) -> int:
        """Logical 128-key blocks of the mask entry."""
        return -(-self.Lk // 128)

    def dense_flops(self) -> float:
        """Dense-equivalent FLOPs of one attention call, 4*B*H*Lq*Lk*d."""
        return 4.0 * self.B * self.H * self.Lq * self.Lk * self.d


def _video(T, Hs, Ws):
    return T * Hs * Ws


WORKLOADS = {
    # -- the five configurations the method is quoted on --------------------
    "tiny": Workload("tiny", 1, 2, 64, 2048, 2048, "normal", taus=(1.0,),
                     centroid_mode=1, seed=1001,
                     notes="Tiny Sol routing, N(0,1), tau=1.0, 1x64"),
    "lcsa": Workload("lcsa", 1, 12, 128, 12288, 12288, "normal",
                     centroid_mode=0, mask="lcsa", frame_tokens=32 * 48,
                     seed=1002,
                     notes="8 latent frames x 32x48 tokens, LCSA window "
                           "[f_q-2, f_q], no centroids"),
    "wan13b": Workload("wan13b", 1, 12, 128, _video(21, 30, 52),
                       _video(21, 30, 52), "pe", grid=(21, 30, 52),
                       taus=(1.0,), centroid_mode=1, seed=1003,
                       notes="Wan-1.3B-like, 21x30x52, tau=1.0, 1x64"),
    "wan14b": Workload("wan14b", 1, 40, 128, _video(21, 30, 52),
                       _video(21, 30, 52), "pe", grid=(21, 30, 52),
                       taus=(0.5, 1.0, 1.5), centroid_mode=2, seed=1004,
                       notes="Wan-14B-like, 21x30x52, 2x32, tau sweep"),
    "h3": Workload("h3", 1, 40, 128, 1024 + _video(21, 48, 84),
                   1024 + _video(21, 48, 84), "pe", grid=(21, 48, 84),
                   n_prefix=1024, taus=(1.0,), centroid_mode=1, seed=1005,
                   notes="H3-like: 1024 N(0,1) prefix + 21x48x84 video, "
                         "tau=1.0, 1x64"),
    "h3_virtual": Workload("h3_virtual", 1, 40, 128, _video(2, 48, 84),
                           _video(2, 48, 84), "pe", grid=(2, 48, 84),
                           centroid_mode=2, slice_tokens=48 * 84,
                           virtual_map=(0, 0, 1, 1, 1), seed=1006,
                           notes="H3 reference-image path: 2 physical latent "
                                 "slices of 48x84, 5 added virtual slices "
                                 "re-reading them, 2x32 residuals"),
    # -- small parity cases: several tiles and a ragged tail ----------------
    "ragged_pe": Workload("ragged_pe", 2, 3, 128, 1000, 1000, "pe",
                          grid=(5, 10, 20), taus=(0.5, 1.0), centroid_mode=1,
                          seed=2001, notes="1000 = 7*128+104 = 15*64+40"),
    "ragged_pe_2x32": Workload("ragged_pe_2x32", 1, 2, 128, 1000, 1000, "pe",
                               grid=(5, 10, 20), taus=(1.0,),
                               centroid_mode=2, seed=2002),
    "ragged_d64": Workload("ragged_d64", 1, 3, 64, 1304, 1304, "normal",
                           taus=(0.5,), centroid_mode=2, seed=2003,
                           notes="1304 = 10*128+24 = 20*64+24: tail half "
                                 "empty in 2x32"),
    "cross": Workload("cross", 2, 2, 128, 700, 1000, "normal", taus=(1.0,),
                      centroid_mode=1, seed=2004, notes="Lq != Lk"),
    "prefix_small": Workload("prefix_small", 1, 2, 128, 256 + 1000,
                             256 + 1000, "pe", grid=(5, 10, 20), n_prefix=256,
                             taus=(1.0,), centroid_mode=1, seed=2005),
    "lcsa_small": Workload("lcsa_small", 1, 3, 128, 5 * 384 + 100,
                           5 * 384 + 100, "normal", centroid_mode=0,
                           mask="lcsa", frame_tokens=384, seed=2006,
                           notes="5 frames of 3 logical blocks + ragged tail"),
    "virtual_small": Workload("virtual_small", 1, 3, 128, _video(2, 10, 32),
                              _video(2, 10, 32), "pe", grid=(2, 10, 32),
                              centroid_mode=2, slice_tokens=320,
                              virtual_map=(0, 1, 1, 0, 1), seed=2007,
                              notes="2 slices of 320 tokens (5 key blocks)"),
    "virtual_ragged": Workload("virtual_ragged", 2, 2, 64, 600, 1000, "normal",
                               centroid_mode=1, slice_tokens=192,
                               virtual_map=(1, 0, 1, 1), n_source_slices=2,
                               seed=2008,
                               notes="ragged queries and keys, separate "
                                     "2-slice source, 1x64"),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def pe_table(T: int, Hs: int, Ws: int) -> np.ndarray:
    """48-dim sinusoidal (t, y, x) embedding of every video token, fp64 [T*Hs*Ws, 48]."""
    omega = 10000.0 ** (-np.arange(8, dtype=np.float64) / 8.0)

    def axis(p):
        ang = p[:, None] * omega[None, :]
        return np.concatenate([np.sin(ang), np.cos(ang)], axis=1)

    t, y, x = np.meshgrid(np.arange(T, dtype=np.float64),
                          np.arange(Hs, dtype=np.float64),
                          np.arange(Ws, dtype=np.float64), indexing="ij")
    return np.concatenate([axis(t.reshape(-1)), axis(y.reshape(-1)),
                           axis(x.reshape(-1))], axis=1)


_SIGNAL_CACHE: dict = {}


def _signal(w: Workload) -> np.ndarray:
    """2 * PE @ W for the video tokens of a "pe" workload, fp32 [n_video, d]."""
    key = (w.grid, w.d)
    if key not in _SIGNAL_CACHE:
        W = np.random.default_rng(W_SEED).normal(0.0, math.sqrt(1.0 / 48.0),
                                                 (48, w.d))
        _SIGNAL_CACHE[key] = (2.0 * (pe_table(*w.grid) @ W)).astype(np.float32)
    return _SIGNAL_CACHE[key]


def _normal(w: Workload, b: int, h: int, which: int, n: int) -> np.ndarray:
    rng = np.random.default_rng([w.seed, b, h, which])
    return rng.standard_normal((n, w.d), dtype=np.float32)


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16)


def head_qkv(w: Workload, b: int, h: int):
    """(q, k, v) of one (batch, head): torch bf16 CPU tensors [Lq|Lk, d]."""
    q = _normal(w, b, h, _Q, w.Lq)
    k = _normal(w, b, h, _K, w.Lk)
    v = _normal(w, b, h, _V, w.Lk)
    if w.gen == "pe":
        sig = _signal(w)
        n_vid = sig.shape[0]
        assert w.Lq == w.Lk == w.n_prefix + n_vid, "pe workloads are self-attention"
        q[w.n_prefix:] += sig
        k[w.n_prefix:] += sig
    elif w.gen != "normal":
        raise ValueError(f"unknown generator {w.gen!r}")
    return _bf16(q), _bf16(k), _bf16(v)


def source_kv(w: Workload, b: int, h: int):
    """(k_src, v_src) of one (batch, head) for a virtual K/V workload, bf16 CPU.

    ``n_source_slices == 0``: the physical K and V themselves; otherwise a
    separate N(0, 1) source of ``n_source_slices * slice_tokens`` tokens."""
    if w.n_source_slices == 0:
        _, k, v = head_qkv(w, b, h)
        return k, v
    n = w.n_source_slices * w.slice_tokens
    return _bf16(_normal(w, b, h, _KS, n)), _bf16(_normal(w, b, h, _VS, n))


def batch_qkv(w: Workload, heads=None, device="cpu"):
    """Full [B, H, L, d] bf16 tensors (or only the (b, h) pairs in ``heads``)."""
    if heads is None:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    Q = torch.zeros((w.B, w.H, w.Lq, w.d), dtype=torch.bfloat16, device=device)
    K = torch.zeros((w.B, w.H, w.Lk, w.d), dtype=torch.bfloat16, device=device)
    V = torch.zeros((w.B, w.H, w.Lk, w.d), dtype=torch.bfloat16, device=device)
    for b, h in heads:
        q, k, v = head_qkv(w, b, h)
        Q[b, h].copy_(q)
        K[b, h].copy_(k)
        V[b, h].copy_(v)
    return Q, K, V
