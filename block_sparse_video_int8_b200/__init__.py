"""Python binding of ``libbsva.so``, the block-sparse INT8 video attention library.

Argument marshalling only: every step of the method runs in the CUDA kernels
behind the C ABI declared in ``include/bsva.h``. PyTorch supplies device
memory and the current stream. There is no CPU or fallback path: if the
library is missing or was built for another ABI, ``load()`` raises.

Entry points (same names as the C ABI):

* ``quantize_qk(q, k)``                      per-block INT8 Q/K, scales, pools
* ``sparse_attn_route(q, k, tau, n_prefix)`` quantise + proxy score + Sol rule
* ``sparse_attn_route_topk(q, k, sparsity, n_prefix)`` the same with fixed-sparsity top-k selection
* ``sparse_attn_fwd(route, v, mode)``        kept blocks exact + centroids
* ``masked_block_attn_fwd(q8, ..., mask)``   explicit logical 128x128 block mask
* ``build_lcsa_mask(Lq, Lk, frame_tokens, window)`` that mask from frame geometry, on the device
* ``quantize_v(v)``, ``masked_block_attn_fwd_v8(...)`` the mask entry on an INT8 V
* ``virtual_kv_residual_fwd(qk, v, slice_tokens, src_map)`` residual virtual K/V:
  physical keys exact, each added virtual slice as centroid terms
* ``quantize_q(q)``                          per-block INT8 Q alone
* ``KVCache(B, H, d, n_slots)``              the INT8 streaming K/V cache in 128-row slabs:
  ``append(k, v)`` (``bsva_kv_cache_append``) and ``attend(qq, mask)``
  (``masked_block_attn_fwd_kvcache``)
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

__all__ = [
    "BsvaError", "load", "lib_path", "Route", "Shape", "abi_version",
    "workspace_bytes", "route_workspace_bytes", "quantize_qk", "sparse_attn_route",
    "sparse_attn_route_topk", "build_lcsa_mask", "quantize_v", "masked_block_attn_fwd_v8", "sparse_attn_fwd",
    "masked_block_attn_fwd", "check_status", "selftest_timeout", "new_workspace",
    "build_centroids", "sparse_attn_core", "virtual_kv_workspace_bytes", "virtual_kv_residual_fwd",
    "quantize_q", "KVCache",
]

ABI_VERSION = 5
_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None

OUT_DTYPES = {torch.bfloat16: 0, torch.float32: 1}

STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "WORKSPACE", 4: "CUDA",
          5: "DEVICE_TIMEOUT", 6: "DEVICE_BOUNDS"}


class BsvaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"bsva error {code} ({STATUS.get(code, '?')}): {msg}")
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("Lq", ctypes.c_int),
                ("Lk", ctypes.c_int), ("d", ctypes.c_int), ("n_prefix", ctypes.c_int)]


class KVCacheStruct(ctypes.Structure):
    """``bsva_kv_cache``: geometry, device buffers, and the ring state the library updates."""
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int), ("n_slots", ctypes.c_int),
                ("k8", ctypes.c_void_p), ("k_scale", ctypes.c_void_p), ("v8", ctypes.c_void_p),
                ("v_scale", ctypes.c_void_p), ("slab_rows", ctypes.c_void_p),
                ("first", ctypes.c_int), ("count", ctypes.c_int)]


def lib_path() -> str:
    """The library to load: ``libbsva.so``, or the ``BSVA_DEVICE_CHECKS`` build
    ``libbsva_checked.so`` when the environment sets ``BSVA_CHECKED=1``."""
    name = "libbsva_checked.so" if os.environ.get("BSVA_CHECKED") == "1" else "libbsva.so"
    return os.path.join(_HERE, name)


_P = ctypes.c_void_p
_SIGS = {
    "bsva_abi_version": (ctypes.c_int, []),
    "bsva_device_checks": (ctypes.c_int, []),
    "bsva_last_error": (ctypes.c_char_p, []),
    "bsva_workspace_bytes": (ctypes.c_size_t, [Shape, ctypes.c_int]),
    "bsva_quantize_qk": (ctypes.c_int, [Shape, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "bsva_route_workspace_bytes": (ctypes.c_size_t, [Shape]),
    "bsva_build_lcsa_mask": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            _P, _P]),
    "sparse_attn_route_topk": (ctypes.c_int, [Shape, _P, _P, ctypes.c_double, _P, _P, _P, _P, _P, _P,
                                              _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "sparse_attn_route": (ctypes.c_int, [Shape, _P, _P, ctypes.c_double, _P, _P, _P, _P, _P, _P,
                                         _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "sparse_attn_fwd": (ctypes.c_int, [Shape, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int,
                                       ctypes.c_float, ctypes.c_int, _P, _P, _P, ctypes.c_size_t, _P]),
    "masked_block_attn_fwd": (ctypes.c_int, [Shape, _P, _P, _P, _P, _P, _P, ctypes.c_int,
                                             ctypes.c_float, ctypes.c_int, _P, _P, _P, ctypes.c_size_t,
                                             _P]),
    "bsva_build_centroids": (ctypes.c_int, [Shape, _P, _P, _P, ctypes.c_int, _P, ctypes.c_size_t, _P]),
    "bsva_sparse_attn_core": (ctypes.c_int, [Shape, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int,
                                             ctypes.c_float, ctypes.c_int, _P, _P, _P, ctypes.c_size_t, _P]),
    "masked_block_attn_fwd_noalloc": (ctypes.c_int, [Shape, _P, _P, _P, _P, _P, _P, ctypes.c_int,
                                                     ctypes.c_float, ctypes.c_int, _P, _P, _P]),
    "bsva_check_status": (ctypes.c_int, [_P, _P]),
    "bsva_quantize_v": (ctypes.c_int, [Shape, _P, _P, _P, _P]),
    "masked_block_attn_fwd_v8": (ctypes.c_int, [Shape, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int,
                                                ctypes.c_float, ctypes.c_int, _P, _P, _P, ctypes.c_size_t,
                                                _P]),
    "bsva_selftest_timeout": (ctypes.c_int, [_P, ctypes.c_size_t, ctypes.c_longlong, _P]),
    "bsva_quantize_q": (ctypes.c_int, [Shape, _P, _P, _P, _P, _P]),
    "bsva_kv_cache_append": (ctypes.c_int, [ctypes.POINTER(KVCacheStruct), _P, _P, ctypes.c_int, _P]),
    "bsva_kv_cache_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(KVCacheStruct), ctypes.c_int]),
    "masked_block_attn_fwd_kvcache": (ctypes.c_int, [ctypes.POINTER(KVCacheStruct), ctypes.c_int, _P, _P, _P,
                                                     ctypes.c_int, ctypes.c_float, ctypes.c_int, _P, _P, _P,
                                                     ctypes.c_size_t, _P]),
    "bsva_virtual_kv_workspace_bytes": (ctypes.c_size_t, [Shape, ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "virtual_kv_residual_fwd": (ctypes.c_int, [Shape, _P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_int, _P, _P, _P,
                                               ctypes.POINTER(ctypes.c_int), ctypes.c_int, ctypes.c_int,
                                               ctypes.c_float, ctypes.c_int, _P, _P, _P, ctypes.c_size_t, _P]),
}


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the CUDA library (once) and check its ABI version; raise if unavailable."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = path or lib_path()
    if not os.path.exists(path):
        raise FileNotFoundError(
            f"libbsva.so not found at {path}; build it with "
            "`python -m block_sparse_video_int8_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    ver = lib.bsva_abi_version()
    if ver != ABI_VERSION:
        raise RuntimeError(f"{path} has ABI version {ver}, this binding expects {ABI_VERSION}")
    _LIB = lib
    return lib


def abi_version() -> int:
    return load().bsva_abi_version()


def _check(rc: int):
    if rc != 0:
        raise BsvaError(rc, load().bsva_last_error().decode(errors="replace"))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, shape, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _shape_of(q, k, n_prefix=0) -> Shape:
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be [B, H, L, d]")
    B, H, Lq, d = q.shape
    if tuple(k.shape[:2]) != (B, H) or k.shape[3] != d:
        raise ValueError(f"k shape {tuple(k.shape)} does not match q {tuple(q.shape)}")
    return Shape(B, H, Lq, k.shape[2], d, n_prefix)


def workspace_bytes(shape: Shape, centroid_mode: int) -> int:
    n = load().bsva_workspace_bytes(shape, centroid_mode)
    if n == 0:
        raise BsvaError(1, f"bad shape or centroid_mode for a workspace: {_fmt(shape)}, mode {centroid_mode}")
    return n


def _fmt(s: Shape) -> str:
    return f"B={s.B} H={s.H} Lq={s.Lq} Lk={s.Lk} d={s.d} n_prefix={s.n_prefix}"


def new_workspace(shape: Shape, centroid_mode: int, device=None) -> torch.Tensor:
    """A zeroed device workspace (uint8) large enough for ``shape`` and mode."""
    n = workspace_bytes(shape, centroid_mode)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


@dataclass
class Route:
    """Outputs of the routing step (all device tensors)."""
    shape: Shape
    tau: float
    q8: torch.Tensor
    q_scale: torch.Tensor
    k8: torch.Tensor
    k_scale: torch.Tensor
    q_pool: torch.Tensor
    k_pool: torch.Tensor
    kept_mask: torch.Tensor
    kept_idx: torch.Tensor
    kept_cnt: torch.Tensor
    row_stats: torch.Tensor | None
    scratch: torch.Tensor | None = None   # route-only workspace when the caller passes none
    sparsity: float | None = None         # set by the fixed-sparsity top-k rule (tau is then NaN)


def _alloc_quant(s: Shape, dev):
    nQB, nKB = -(-s.Lq // 128), -(-s.Lk // 64)
    return dict(
        q8=torch.empty((s.B, s.H, s.Lq, s.d), dtype=torch.int8, device=dev),
        q_scale=torch.empty((s.B, s.H, nQB), dtype=torch.float32, device=dev),
        k8=torch.empty((s.B, s.H, s.Lk, s.d), dtype=torch.int8, device=dev),
        k_scale=torch.empty((s.B, s.H, nKB), dtype=torch.float32, device=dev),
        q_pool=torch.empty((s.B, s.H, nQB, s.d), dtype=torch.int32, device=dev),
        k_pool=torch.empty((s.B, s.H, nKB, 2, s.d), dtype=torch.int32, device=dev),
    )


def quantize_qk(q: torch.Tensor, k: torch.Tensor, out: dict | None = None, stream=None) -> dict:
    """Per-block INT8 Q/K with scales and sum-pools (C ABI ``bsva_quantize_qk``)."""
    lib = load()
    s = _shape_of(q, k)
    _need(q, torch.bfloat16, None, "q")
    _need(k, torch.bfloat16, None, "k")
    o = out or _alloc_quant(s, q.device)
    _check(lib.bsva_quantize_qk(s, _ptr(q), _ptr(k), _ptr(o["q8"]), _ptr(o["q_scale"]), _ptr(o["k8"]),
                                _ptr(o["k_scale"]), _ptr(o["q_pool"]), _ptr(o["k_pool"]),
                                _stream(stream)))
    return o


def route_workspace_bytes(shape: Shape) -> int:
    n = load().bsva_route_workspace_bytes(shape)
    if n == 0:
        raise BsvaError(1, f"bad shape for a routing workspace: {_fmt(shape)}")
    return n


def _route_call(entry: str, param: float, q, k, n_prefix, row_stats, out, workspace, stream,
                tau: float, sparsity: float | None) -> Route:
    lib = load()
    s = _shape_of(q, k, n_prefix)
    _need(q, torch.bfloat16, None, "q")
    _need(k, torch.bfloat16, None, "k")
    nQB, nKB = -(-s.Lq // 128), -(-s.Lk // 64)
    if out is None:
        dev = q.device
        o = _alloc_quant(s, dev)
        out = Route(shape=s, tau=tau, **o,
                    kept_mask=torch.empty((s.B, s.H, nQB, nKB), dtype=torch.uint8, device=dev),
                    kept_idx=torch.empty((s.B, s.H, nQB, nKB), dtype=torch.int32, device=dev),
                    kept_cnt=torch.empty((s.B, s.H, nQB), dtype=torch.int32, device=dev),
                    row_stats=(torch.empty((s.B, s.H, nQB, 3), dtype=torch.float64, device=dev)
                               if row_stats else None))
    else:
        out.shape, out.tau = s, tau
    out.sparsity = sparsity
    if workspace is None:
        need = lib.bsva_route_workspace_bytes(s)   # 0 on a bad shape: the call below reports it
        if need and (out.scratch is None or out.scratch.numel() < need):
            out.scratch = torch.empty(need, dtype=torch.uint8, device=q.device)
        workspace = out.scratch
    if workspace is not None:
        _need(workspace, torch.uint8, None, "workspace")
    _check(getattr(lib, entry)(s, _ptr(q), _ptr(k), ctypes.c_double(param), _ptr(out.q8),
                               _ptr(out.q_scale), _ptr(out.k8), _ptr(out.k_scale), _ptr(out.q_pool),
                               _ptr(out.k_pool), _ptr(out.kept_mask), _ptr(out.kept_idx),
                               _ptr(out.kept_cnt), _ptr(out.row_stats), _ptr(workspace),
                               0 if workspace is None else workspace.numel(), _stream(stream)))
    return out


def sparse_attn_route(q: torch.Tensor, k: torch.Tensor, tau: float, n_prefix: int = 0,
                      row_stats: bool = False, out: Route | None = None,
                      workspace: torch.Tensor | None = None, stream=None) -> Route:
    """Quantise, score and route by the Sol rule (C ABI ``sparse_attn_route``).

    ``workspace`` is a device uint8 buffer of at least ``route_workspace_bytes``
    (a ``new_workspace`` buffer serves too); without one, a route-only buffer is
    allocated once and kept on the returned ``Route``."""
    return _route_call("sparse_attn_route", tau, q, k, n_prefix, row_stats, out, workspace, stream,
                       tau=tau, sparsity=None)


def sparse_attn_route_topk(q: torch.Tensor, k: torch.Tensor, sparsity: float, n_prefix: int = 0,
                           row_stats: bool = False, out: Route | None = None,
                           workspace: torch.Tensor | None = None, stream=None) -> Route:
    """Quantise, score and keep the top (1 - sparsity) of each row's routed
    blocks (C ABI ``sparse_attn_route_topk``); workspace as for
    ``sparse_attn_route``."""
    return _route_call("sparse_attn_route_topk", sparsity, q, k, n_prefix, row_stats, out, workspace,
                       stream, tau=float("nan"), sparsity=float(sparsity))


def _out(out, shape, out_dtype, device):
    if out_dtype not in OUT_DTYPES:
        raise TypeError(f"out_dtype must be torch.bfloat16 or torch.float32, got {out_dtype}")
    if out is None:
        return torch.empty(shape, dtype=out_dtype, device=device)
    _need(out, out_dtype, shape, "out")
    return out


def sparse_attn_fwd(route: Route, v: torch.Tensor, centroid_mode: int, softmax_scale: float = 0.0,
                    with_lse: bool = False, workspace: torch.Tensor | None = None,
                    out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                    out_dtype=torch.bfloat16, stream=None):
    """Sparse attention over the routed blocks plus centroids (C ABI ``sparse_attn_fwd``).

    Returns ``out`` ([B, H, Lq, d], bf16 or fp32) or ``(out, lse)`` when ``with_lse``.
    """
    lib = load()
    s = route.shape
    _need(v, torch.bfloat16, (s.B, s.H, s.Lk, s.d), "v")
    if workspace is None:
        workspace = new_workspace(s, centroid_mode, v.device)
    out = _out(out, (s.B, s.H, s.Lq, s.d), out_dtype, v.device)
    if with_lse and lse is None:
        lse = torch.empty((s.B, s.H, s.Lq), dtype=torch.float32, device=v.device)
    _check(lib.sparse_attn_fwd(s, _ptr(route.q8), _ptr(route.q_scale), _ptr(route.k8),
                               _ptr(route.k_scale), _ptr(route.k_pool), _ptr(v), _ptr(route.kept_mask),
                               _ptr(route.kept_idx), _ptr(route.kept_cnt), centroid_mode,
                               ctypes.c_float(softmax_scale), OUT_DTYPES[out.dtype], _ptr(out), _ptr(lse),
                               _ptr(workspace),
                               workspace.numel(), _stream(stream)))
    return (out, lse) if with_lse else out


def build_centroids(route: Route, v: torch.Tensor, centroid_mode: int, workspace: torch.Tensor,
                    stream=None):
    """The centroid table of (k_pool, k_scale, v) into ``workspace`` (C ABI ``bsva_build_centroids``)."""
    lib = load()
    s = route.shape
    _need(v, torch.bfloat16, (s.B, s.H, s.Lk, s.d), "v")
    _check(lib.bsva_build_centroids(s, _ptr(route.k_pool), _ptr(route.k_scale), _ptr(v), centroid_mode,
                                    _ptr(workspace), workspace.numel(), _stream(stream)))


def sparse_attn_core(route: Route, v: torch.Tensor, centroid_mode: int, workspace: torch.Tensor,
                     out: torch.Tensor, softmax_scale: float = 0.0, lse: torch.Tensor | None = None,
                     stream=None):
    """The attention kernel alone, on a workspace that holds the centroid table
    (C ABI ``bsva_sparse_attn_core``)."""
    lib = load()
    s = route.shape
    _need(v, torch.bfloat16, (s.B, s.H, s.Lk, s.d), "v")
    if out.dtype not in OUT_DTYPES:
        raise TypeError("out must be bf16 or fp32")
    _need(out, out.dtype, (s.B, s.H, s.Lq, s.d), "out")
    _check(lib.bsva_sparse_attn_core(s, _ptr(route.q8), _ptr(route.q_scale), _ptr(route.k8), _ptr(route.k_scale),
                                     _ptr(v), _ptr(route.kept_mask), _ptr(route.kept_idx), _ptr(route.kept_cnt),
                                     centroid_mode, ctypes.c_float(softmax_scale), OUT_DTYPES[out.dtype],
                                     _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def build_lcsa_mask(Lq: int, Lk: int, frame_tokens: int, window_frames: int, batch: int = 1,
                    out: torch.Tensor | None = None, device=None, stream=None) -> torch.Tensor:
    """The LCSA logical mask from frame geometry, built on the device (C ABI
    ``bsva_build_lcsa_mask``): uint8 [batch, 1, ceil(Lq/128), ceil(Lk/128)]."""
    lib = load()
    shape = (max(batch, 0), 1, -(-Lq // 128) if Lq > 0 else 0, -(-Lk // 128) if Lk > 0 else 0)
    if out is None:
        m = torch.empty(shape, dtype=torch.uint8, device=device or "cuda")
    else:
        _need(out, torch.uint8, shape, "out")
        m = out
    _check(lib.bsva_build_lcsa_mask(Lq, Lk, frame_tokens, window_frames, batch,
                                    _ptr(m) if m.numel() else None, _stream(stream)))
    return m


def _masked_call(entry, q8, q_scale, k8, k_scale, v_args, v_like, block_mask, softmax_scale, with_lse,
                 workspace, out, lse, out_dtype, stream):
    lib = load()
    B, H, Lq, d = q8.shape
    Lk = k8.shape[2]
    s = Shape(B, H, Lq, Lk, d, 0)
    _need(q8, torch.int8, None, "q8")
    _need(k8, torch.int8, (B, H, Lk, d), "k8")
    _need(block_mask, torch.uint8, None, "block_mask")
    if block_mask.dim() != 4 or block_mask.shape[0] != B or block_mask.shape[2:] != (-(-Lq // 128), -(-Lk // 128)):
        raise ValueError(f"block_mask shape {tuple(block_mask.shape)} is not [B, Hm, nQB, nLK]")
    mask_heads = block_mask.shape[1]
    if workspace is None:
        workspace = new_workspace(s, 0, v_like.device)
    out = _out(out, (B, H, Lq, d), out_dtype, v_like.device)
    if with_lse and lse is None:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=v_like.device)
    _check(getattr(lib, entry)(s, _ptr(q8), _ptr(q_scale), _ptr(k8), _ptr(k_scale), *[_ptr(t) for t in v_args],
                               _ptr(block_mask), mask_heads, ctypes.c_float(softmax_scale),
                               OUT_DTYPES[out.dtype], _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
                               _stream(stream)))
    return (out, lse) if with_lse else out


def masked_block_attn_fwd(q8, q_scale, k8, k_scale, v, block_mask, softmax_scale: float = 0.0,
                          with_lse: bool = False, workspace=None, out=None, lse=None,
                          out_dtype=torch.bfloat16, stream=None):
    """Attention over an explicit logical 128x128 block mask (C ABI ``masked_block_attn_fwd``)."""
    B, H, _, d = q8.shape
    _need(v, torch.bfloat16, (B, H, k8.shape[2], d), "v")
    return _masked_call("masked_block_attn_fwd", q8, q_scale, k8, k_scale, (v,), v, block_mask, softmax_scale,
                        with_lse, workspace, out, lse, out_dtype, stream)


def quantize_v(v: torch.Tensor, out: dict | None = None, stream=None) -> dict:
    """Per-64-row-block INT8 V and its scales (C ABI ``bsva_quantize_v``)."""
    lib = load()
    _need(v, torch.bfloat16, None, "v")
    if v.dim() != 4:
        raise ValueError("v must be [B, H, Lk, d]")
    B, H, Lk, d = v.shape
    s = Shape(B, H, Lk, Lk, d, 0)
    o = out or dict(v8=torch.empty(v.shape, dtype=torch.int8, device=v.device),
                    v_scale=torch.empty((B, H, -(-Lk // 64)), dtype=torch.float32, device=v.device))
    _check(lib.bsva_quantize_v(s, _ptr(v), _ptr(o["v8"]), _ptr(o["v_scale"]), _stream(stream)))
    return o


def masked_block_attn_fwd_v8(q8, q_scale, k8, k_scale, v8, v_scale, block_mask, softmax_scale: float = 0.0,
                             with_lse: bool = False, workspace=None, out=None, lse=None,
                             out_dtype=torch.bfloat16, stream=None):
    """The mask entry on an INT8 V (C ABI ``masked_block_attn_fwd_v8``)."""
    B, H, _, d = q8.shape
    Lk = k8.shape[2]
    _need(v8, torch.int8, (B, H, Lk, d), "v8")
    _need(v_scale, torch.float32, (B, H, -(-Lk // 64)), "v_scale")
    return _masked_call("masked_block_attn_fwd_v8", q8, q_scale, k8, k_scale, (v8, v_scale), v8, block_mask,
                        softmax_scale, with_lse, workspace, out, lse, out_dtype, stream)


def virtual_kv_workspace_bytes(shape: Shape, slice_tokens: int, n_src_slices: int, centroid_mode: int = 2) -> int:
    n = load().bsva_virtual_kv_workspace_bytes(shape, slice_tokens, n_src_slices, centroid_mode)
    if n == 0:
        raise BsvaError(1, f"bad shape or geometry for a virtual K/V workspace: {_fmt(shape)}, "
                           f"slice_tokens {slice_tokens}, {n_src_slices} source slices, mode {centroid_mode}")
    return n


def virtual_kv_residual_fwd(qk: dict, v: torch.Tensor, slice_tokens: int, src_map, source: dict | None = None,
                            src_v: torch.Tensor | None = None, centroid_mode: int = 2, softmax_scale: float = 0.0,
                            with_lse: bool = False, workspace: torch.Tensor | None = None, out=None, lse=None,
                            out_dtype=torch.bfloat16, stream=None):
    """Residual virtual K/V attention (C ABI ``virtual_kv_residual_fwd``).

    ``qk`` is the ``quantize_qk`` output of the physical Q and K; ``v`` the
    physical values. Virtual slice l re-reads slice ``src_map[l]`` of the
    source: ``source`` (a ``quantize_qk`` output of the source keys, its
    ``k_scale`` and ``k_pool`` are used) and ``src_v``, by default the
    physical ``qk`` and ``v`` themselves."""
    lib = load()
    B, H, Lq, d = qk["q8"].shape
    Lk = qk["k8"].shape[2]
    s = Shape(B, H, Lq, Lk, d, 0)
    _need(qk["q8"], torch.int8, None, "q8")
    _need(qk["k8"], torch.int8, (B, H, Lk, d), "k8")
    _need(v, torch.bfloat16, (B, H, Lk, d), "v")
    source = qk if source is None else source
    src_v = v if src_v is None else src_v
    _need(src_v, torch.bfloat16, None, "src_v")
    Ls = src_v.shape[2]
    if slice_tokens <= 0 or Ls % slice_tokens:
        raise ValueError(f"src_v holds {Ls} tokens, not a whole number of {slice_tokens}-token slices")
    n_src = Ls // slice_tokens
    _need(src_v, torch.bfloat16, (B, H, Ls, d), "src_v")
    _need(source["k_scale"], torch.float32, (B, H, -(-Ls // 64)), "source k_scale")
    _need(source["k_pool"], torch.int32, (B, H, -(-Ls // 64), 2, d), "source k_pool")
    src_map = [int(x) for x in src_map]
    cmap = (ctypes.c_int * len(src_map))(*src_map) if src_map else None
    if workspace is None:
        workspace = torch.zeros(virtual_kv_workspace_bytes(s, slice_tokens, n_src, centroid_mode),
                                dtype=torch.uint8, device=v.device)
    out = _out(out, (B, H, Lq, d), out_dtype, v.device)
    if with_lse and lse is None:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=v.device)
    _check(lib.virtual_kv_residual_fwd(s, _ptr(qk["q8"]), _ptr(qk["q_scale"]), _ptr(qk["k8"]), _ptr(qk["k_scale"]),
                                       _ptr(v), slice_tokens, n_src, _ptr(source["k_scale"]), _ptr(source["k_pool"]),
                                       _ptr(src_v), cmap, len(src_map), centroid_mode, ctypes.c_float(softmax_scale),
                                       OUT_DTYPES[out.dtype], _ptr(out), _ptr(lse), _ptr(workspace),
                                       workspace.numel(), _stream(stream)))
    return (out, lse) if with_lse else out


def check_status(workspace: torch.Tensor, stream=None):
    """Synchronise and raise BsvaError if a device-side wait timed out."""
    _check(load().bsva_check_status(_ptr(workspace), _stream(stream)))


def selftest_timeout(workspace: torch.Tensor, limit_ns: int, stream=None):
    """Launch the bounded-wait self test (a wait that is meant to run out)."""
    _check(load().bsva_selftest_timeout(_ptr(workspace), workspace.numel(), int(limit_ns),
                                        _stream(stream)))


def quantize_q(q: torch.Tensor, out: dict | None = None, stream=None) -> dict:
    """Per-128-row-block INT8 Q with scales and sum-pools (C ABI ``bsva_quantize_q``)."""
    lib = load()
    _need(q, torch.bfloat16, None, "q")
    if q.dim() != 4:
        raise ValueError("q must be [B, H, Lq, d]")
    B, H, Lq, d = q.shape
    nQB = -(-Lq // 128)
    o = out or dict(q8=torch.empty(q.shape, dtype=torch.int8, device=q.device),
                    q_scale=torch.empty((B, H, nQB), dtype=torch.float32, device=q.device),
                    q_pool=torch.empty((B, H, nQB, d), dtype=torch.int32, device=q.device))
    _check(lib.bsva_quantize_q(Shape(B, H, Lq, Lq, d, 0), _ptr(q), _ptr(o["q8"]), _ptr(o["q_scale"]),
                               _ptr(o["q_pool"]), _stream(stream)))
    return o


class KVCache:
    """The INT8 streaming K/V cache in 128-row slabs (C ABI ``bsva_kv_cache``).

    The device buffers are torch tensors owned by this object; ``append`` and ``attend``
    call the library, which keeps the ring state (oldest slot, live slabs) in the struct."""

    def __init__(self, B: int, H: int, d: int, n_slots: int, device=None):
        dev = device or "cuda"
        rows = n_slots * 128
        self.k8 = torch.zeros((B, H, rows, d), dtype=torch.int8, device=dev)
        self.v8 = torch.zeros((B, H, rows, d), dtype=torch.int8, device=dev)
        self.k_scale = torch.zeros((B, H, 2 * n_slots), dtype=torch.float32, device=dev)
        self.v_scale = torch.zeros((B, H, 2 * n_slots), dtype=torch.float32, device=dev)
        self.slab_rows = torch.zeros((n_slots,), dtype=torch.int32, device=dev)
        self.c = KVCacheStruct(B, H, d, n_slots, self.k8.data_ptr(), self.k_scale.data_ptr(), self.v8.data_ptr(),
                               self.v_scale.data_ptr(), self.slab_rows.data_ptr(), 0, 0)

    @property
    def first(self) -> int:
        return self.c.first

    @property
    def count(self) -> int:
        return self.c.count

    def append(self, k: torch.Tensor, v: torch.Tensor, stream=None):
        """Quantise a chunk of new tokens (bf16 [B, H, Lc, d]) into the next slabs, evicting the oldest."""
        c = self.c
        _need(k, torch.bfloat16, None, "k")
        if k.dim() != 4 or tuple(k.shape[:2]) != (c.B, c.H) or k.shape[3] != c.d:
            raise ValueError(f"k shape {tuple(k.shape)} does not match the cache (B={c.B}, H={c.H}, d={c.d})")
        _need(v, torch.bfloat16, tuple(k.shape), "v")
        _check(load().bsva_kv_cache_append(ctypes.byref(c), _ptr(k), _ptr(v), k.shape[2], _stream(stream)))

    def workspace_bytes(self, Lq: int) -> int:
        n = load().bsva_kv_cache_workspace_bytes(ctypes.byref(self.c), Lq)
        if n == 0:
            raise BsvaError(1, f"bad cache geometry or Lq = {Lq}")
        return n

    def attend(self, qq: dict, block_mask: torch.Tensor, softmax_scale: float = 0.0, with_lse: bool = False,
               workspace=None, out=None, lse=None, out_dtype=torch.bfloat16, stream=None):
        """The mask entry over the live slabs (C ABI ``masked_block_attn_fwd_kvcache``); ``qq`` from
        ``quantize_q``, ``block_mask`` uint8 [B, Hm, nQB, count] over the live slabs, oldest first."""
        c = self.c
        q8, q_scale = qq["q8"], qq["q_scale"]
        _need(q8, torch.int8, None, "q8")
        if q8.dim() != 4 or tuple(q8.shape[:2]) != (c.B, c.H) or q8.shape[3] != c.d:
            raise ValueError(f"q8 shape {tuple(q8.shape)} does not match the cache")
        B, H, Lq, d = q8.shape
        _need(block_mask, torch.uint8, None, "block_mask")
        if block_mask.dim() != 4 or block_mask.shape[0] != B or tuple(block_mask.shape[2:]) != (-(-Lq // 128), c.count):
            raise ValueError(f"block_mask shape {tuple(block_mask.shape)} is not [B, Hm, nQB, live slabs]")
        if workspace is None:
            workspace = torch.zeros(self.workspace_bytes(Lq), dtype=torch.uint8, device=q8.device)
        out = _out(out, (B, H, Lq, d), out_dtype, q8.device)
        if with_lse and lse is None:
            lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q8.device)
        _check(load().masked_block_attn_fwd_kvcache(ctypes.byref(c), Lq, _ptr(q8), _ptr(q_scale), _ptr(block_mask),
                                                    block_mask.shape[1], ctypes.c_float(softmax_scale),
                                                    OUT_DTYPES[out.dtype], _ptr(out), _ptr(lse), _ptr(workspace),
                                                    workspace.numel(), _stream(stream)))
        return (out, lse) if with_lse else out
