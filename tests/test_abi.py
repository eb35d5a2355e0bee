"""The C-ABI library loads, exports every symbol its header declares, and
rejects bad arguments with status codes (CPU only: no kernel is launched)."""
import ctypes
import math
import os
import re

import pytest
import torch

import block_sparse_video_int8_b200 as bsva

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "bsva.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(\w+)\s*\(", src, flags=re.M)))


def test_library_builds_and_exports_every_declared_symbol():
    from block_sparse_video_int8_b200 import build
    build.build()
    lib = ctypes.CDLL(bsva.lib_path())
    names = _declared()
    assert {"sparse_attn_route", "sparse_attn_fwd", "masked_block_attn_fwd", "bsva_quantize_qk",
            "bsva_abi_version", "bsva_last_error", "bsva_workspace_bytes", "bsva_check_status",
            "bsva_selftest_timeout"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_abi_version_matches_binding():
    assert bsva.abi_version() == bsva.ABI_VERSION == 5


def test_checked_build_exports_the_same_symbols_and_says_so():
    # the BSVA_DEVICE_CHECKS build (libbsva_checked.so) is the same ABI with index checks in the
    # kernels; the default build reports that it makes none
    from block_sparse_video_int8_b200 import build
    path = build.build(checked=True)
    lib = ctypes.CDLL(path)
    for n in _declared():
        assert hasattr(lib, n), n
    lib.bsva_abi_version.restype = ctypes.c_int
    lib.bsva_device_checks.restype = ctypes.c_int
    assert lib.bsva_abi_version() == bsva.ABI_VERSION
    assert lib.bsva_device_checks() == 1
    assert bsva.load().bsva_device_checks() == 0


def test_workspace_size_arithmetic():
    s = bsva.Shape(1, 40, 32760, 32760, 128, 0)
    nKB, nQB, BH = 512, 256, 40
    n2 = bsva.workspace_bytes(s, 2)
    nCT = math.ceil(nKB * 2 / 32)
    assert n2 >= BH * nCT * 64 * 128 * 3 + BH * nCT * 32 * 8
    n0 = bsva.workspace_bytes(s, 0)
    assert n0 >= BH * nQB * nKB * 4
    # routing stages its fp64 scores after the 256-byte status word; every full
    # workspace holds that region as well
    nr = bsva.route_workspace_bytes(s)
    assert nr >= 256 + BH * nQB * nKB * 8
    assert min(bsva.workspace_bytes(s, m) for m in (0, 1, 2)) >= nr
    assert n0 >= nr + BH * nQB * nKB * 4
    with pytest.raises(bsva.BsvaError):
        bsva.workspace_bytes(bsva.Shape(1, 1, 100, 100, 96, 0), 1)   # d = 96
    with pytest.raises(bsva.BsvaError):
        bsva.workspace_bytes(s, 3)


def _raw_route(shape, ptr=0, ws_bytes=1 << 30):
    lib = bsva.load()
    P = ctypes.c_void_p(ptr) if ptr else None
    return lib.sparse_attn_route(shape, P, P, ctypes.c_double(1.0), P, P, P, P, P, P, P, P, P, None,
                                 P, ws_bytes, None)


def test_bad_arguments_return_codes_without_launching():
    lib = bsva.load()
    good = bsva.Shape(1, 2, 256, 256, 128, 0)
    assert _raw_route(good) == 1                                   # NULL pointers
    assert b"NULL" in lib.bsva_last_error()
    assert _raw_route(bsva.Shape(1, 2, 256, 256, 80, 0), 0x1000) == 2   # d = 80 unsupported
    assert _raw_route(bsva.Shape(1, 2, 256, 256, 128, 100), 0x1000) == 1  # prefix not /128
    assert _raw_route(bsva.Shape(0, 2, 256, 256, 128, 0), 0x1000) == 1
    assert _raw_route(good, 0x1001) == 1                           # misaligned
    assert b"aligned" in lib.bsva_last_error()
    # NaN / +inf tau are rejected before any device work
    P = ctypes.c_void_p(0x1000)
    rc = lib.sparse_attn_route(good, P, P, ctypes.c_double(float("nan")), P, P, P, P, P, P, P, P, P,
                               None, P, 1 << 30, None)
    assert rc == 1
    # the score workspace: too small, NULL
    assert _raw_route(good, 0x10000, ws_bytes=256) == 3
    assert b"workspace" in lib.bsva_last_error()
    Q = ctypes.c_void_p(0x10000)
    rc = lib.sparse_attn_route(good, Q, Q, ctypes.c_double(1.0), Q, Q, Q, Q, Q, Q, Q, Q, Q, None,
                               None, 1 << 30, None)
    assert rc == 3


def test_topk_route_rejects_bad_sparsity_and_workspace():
    lib = bsva.load()
    good = bsva.Shape(1, 2, 256, 256, 128, 0)
    P = ctypes.c_void_p(0x10000)
    for sp in (-0.1, 1.5, float("nan")):
        rc = lib.sparse_attn_route_topk(good, P, P, ctypes.c_double(sp), P, P, P, P, P, P, P, P, P, None,
                                        P, 1 << 30, None)
        assert rc == 1
        assert b"sparsity" in lib.bsva_last_error()
    rc = lib.sparse_attn_route_topk(good, P, P, ctypes.c_double(0.75), P, P, P, P, P, P, P, P, P, None,
                                    P, 256, None)
    assert rc == 3


def test_lcsa_builder_rejects_bad_geometry():
    lib = bsva.load()
    P = ctypes.c_void_p(0x10000)
    for args in ((0, 100, 64, 1, 1), (100, 100, 0, 1, 1), (100, 100, 64, -1, 1), (100, 100, 64, 1, 0)):
        assert lib.bsva_build_lcsa_mask(*args, P, None) == 1
    assert lib.bsva_build_lcsa_mask(100, 100, 64, 1, 1, None, None) == 1


def test_int8_v_entries_reject_bad_arguments():
    lib = bsva.load()
    s = bsva.Shape(1, 2, 256, 256, 128, 0)
    P = ctypes.c_void_p(0x10000)
    assert lib.bsva_quantize_v(s, P, None, P, None) == 1
    assert lib.bsva_quantize_v(bsva.Shape(1, 2, 256, 256, 96, 0), P, P, P, None) == 2
    rc = lib.masked_block_attn_fwd_v8(s, P, P, P, P, None, P, P, 1, ctypes.c_float(0), 0, P, None, P, 1 << 30,
                                      None)
    assert rc == 1 and b"v8" in lib.bsva_last_error()
    rc = lib.masked_block_attn_fwd_v8(s, P, P, P, P, P, P, P, 3, ctypes.c_float(0), 0, P, None, P, 1 << 30, None)
    assert rc == 1                                                 # mask_heads not in {1, H}
    rc = lib.masked_block_attn_fwd_v8(s, P, P, P, P, P, P, P, 1, ctypes.c_float(0), 0, P, None, P, 16, None)
    assert rc == 3


def test_fwd_rejects_bad_mode_and_small_workspace():
    lib = bsva.load()
    s = bsva.Shape(1, 2, 256, 256, 128, 0)
    P = ctypes.c_void_p(0x10000)
    rc = lib.sparse_attn_fwd(s, P, P, P, P, P, P, P, P, P, 3, ctypes.c_float(0), 0, P, None, P, 1 << 30, None)
    assert rc == 1
    rc = lib.sparse_attn_fwd(s, P, P, P, P, P, P, P, P, P, 1, ctypes.c_float(0), 0, P, None, P, 16, None)
    assert rc == 3
    rc = lib.sparse_attn_fwd(s, P, P, P, P, P, P, P, P, P, 1, ctypes.c_float(0), 7, P, None, P, 1 << 30, None)
    assert rc == 1                                                 # unknown out_dtype
    rc = lib.masked_block_attn_fwd(s, P, P, P, P, P, P, 3, ctypes.c_float(0), 0, P, None, P, 1 << 30, None)
    assert rc == 1                                                 # mask_heads not in {1, H}


def _raw_virtual(s, slice_tokens, n_src, src_map, mode=2, ws_bytes=1 << 30, ptr=0x10000):
    lib = bsva.load()
    P = ctypes.c_void_p(ptr)
    cmap = (ctypes.c_int * len(src_map))(*src_map) if src_map else None
    return lib.virtual_kv_residual_fwd(s, P, P, P, P, P, slice_tokens, n_src, P, P, P, cmap, len(src_map), mode,
                                       ctypes.c_float(0), 0, P, None, P, ws_bytes, None)


def test_virtual_kv_entry_rejects_bad_geometry_and_workspace():
    lib = bsva.load()
    s = bsva.Shape(1, 40, 8064, 8064, 128, 0)
    # workspace: kept lists of every physical block, the virtual tile table and a
    # centroid table over the source groups only
    n = bsva.virtual_kv_workspace_bytes(s, 4032, 2, 2)
    nQB, nKB, BH = 63, 126, 40
    nCT = math.ceil(2 * 63 * 2 / 32)
    assert n >= BH * nQB * nKB * 4 + BH * nCT * 64 * 128 * 3 + BH * nCT * 32 * 8
    assert n < BH * nQB * nKB * 4 + BH * (nCT + 1) * 64 * 128 * 3 + BH * (nCT + 1) * 32 * 8 + 64 * 1024
    for bad in ((100, 2, 2), (0, 2, 2), (4032, 0, 2), (4032, 2, 3)):
        assert lib.bsva_virtual_kv_workspace_bytes(s, *bad) == 0
    assert _raw_virtual(s, 4000, 2, (0, 1)) == 1 and b"slice_tokens" in lib.bsva_last_error()
    assert _raw_virtual(s, 4032, 2, (0, 2)) == 1 and b"src_map[1]" in lib.bsva_last_error()
    assert _raw_virtual(s, 4032, 2, (0, -1)) == 1
    assert _raw_virtual(s, 4032, 2, tuple([0] * 33)) == 1           # more than 32 virtual slices
    assert _raw_virtual(s, 4032, 2, (0, 1), mode=3) == 1
    assert _raw_virtual(s, 4032, 2, (0, 1), ptr=0x10001) == 1       # misaligned
    assert _raw_virtual(s, 4032, 2, (0, 1), ws_bytes=256) == 3
    P = ctypes.c_void_p(0x10000)
    rc = lib.virtual_kv_residual_fwd(s, P, P, P, P, P, 4032, 2, None, P, P, None, 2, 2,
                                     ctypes.c_float(0), 0, P, None, P, 1 << 30, None)
    assert rc == 1                                                  # NULL map with n_virtual > 0


def test_no_device_is_an_error_not_a_fallback():
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    lib = bsva.load()
    s = bsva.Shape(1, 2, 256, 256, 128, 0)
    P = ctypes.c_void_p(0x10000)
    rc = lib.bsva_quantize_qk(s, P, P, P, P, P, P, P, P, None)
    assert rc in (2, 4)
    assert lib.bsva_last_error()
    assert _raw_virtual(bsva.Shape(1, 2, 640, 640, 128, 0), 320, 2, (0, 1, 1)) in (2, 4)


def test_binding_refuses_cpu_tensors():
    q = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        bsva.sparse_attn_route(q, q, 1.0)


def test_binding_signatures_cover_exactly_the_declared_entry_points():
    # every ctypes signature names a declared symbol, and every declared symbol has a signature
    assert set(bsva._SIGS) == set(_declared())


def test_virtual_kv_binding_refuses_cpu_tensors():
    q8 = torch.zeros((1, 1, 640, 128), dtype=torch.int8)
    qk = dict(q8=q8, q_scale=torch.zeros((1, 1, 5)), k8=q8.clone(), k_scale=torch.zeros((1, 1, 10)),
              k_pool=torch.zeros((1, 1, 10, 2, 128), dtype=torch.int32))
    v = torch.zeros((1, 1, 640, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        bsva.virtual_kv_residual_fwd(qk, v, 320, (0, 1))


def _cache(n_slots=4, d=128, B=1, H=2, first=0, count=0, ptr=0x10000):
    P = ptr
    return bsva.KVCacheStruct(B, H, d, n_slots, P, P, P, P, P, first, count)


def test_kv_cache_entries_reject_bad_arguments():
    lib = bsva.load()
    P = ctypes.c_void_p(0x10000)
    c = _cache()
    assert lib.bsva_kv_cache_append(None, P, P, 128, None) == 1
    assert lib.bsva_kv_cache_append(ctypes.byref(c), P, P, 0, None) == 1          # empty chunk
    assert lib.bsva_kv_cache_append(ctypes.byref(c), None, P, 128, None) == 1
    bad_d = _cache(d=96)
    assert lib.bsva_kv_cache_append(ctypes.byref(bad_d), P, P, 128, None) == 2
    bad_ring = _cache(first=4)                                                     # first outside [0, n_slots)
    assert lib.bsva_kv_cache_append(ctypes.byref(bad_ring), P, P, 128, None) == 1
    assert (bad_ring.first, bad_ring.count) == (4, 0)                              # untouched on failure
    misaligned = _cache(ptr=0x10001)
    assert lib.bsva_kv_cache_append(ctypes.byref(misaligned), P, P, 128, None) == 1
    # the attention entry: an empty cache, a wrong mask head count, a small workspace
    rc = lib.masked_block_attn_fwd_kvcache(ctypes.byref(c), 256, P, P, P, 1, ctypes.c_float(0), 0, P, None, P,
                                           1 << 30, None)
    assert rc == 1 and b"no slab" in lib.bsva_last_error()
    live = _cache(count=3, first=2)
    rc = lib.masked_block_attn_fwd_kvcache(ctypes.byref(live), 256, P, P, P, 3, ctypes.c_float(0), 0, P, None, P,
                                           1 << 30, None)
    assert rc == 1
    rc = lib.masked_block_attn_fwd_kvcache(ctypes.byref(live), 256, P, P, P, 1, ctypes.c_float(0), 0, P, None, P,
                                           64, None)
    assert rc == 3
    # workspace: kept lists over the live slabs' 64-row blocks, one row per query block
    n = lib.bsva_kv_cache_workspace_bytes(ctypes.byref(live), 256)
    assert n >= 1 * 2 * 2 * 6 * 4 and lib.bsva_kv_cache_workspace_bytes(ctypes.byref(live), 0) == 0
    assert lib.bsva_quantize_q(bsva.Shape(1, 2, 256, 256, 128, 0), P, None, P, P, None) == 1


def test_kv_cache_binding_refuses_cpu_tensors():
    k = torch.zeros((1, 2, 128, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        bsva.quantize_q(k)
