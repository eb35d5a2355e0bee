// api.cu -- the C ABI (include/bsva.h): argument validation, TMA descriptor
// encoding, workspace carving and kernel launches on the caller's stream.
// No entry point allocates, frees or synchronises device memory (except
// bsva_check_status, whose job is to synchronise), and none falls back to
// another path: a bad argument or an unsupported device returns an error code
// and leaves every output untouched.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

namespace bsva {
}

using namespace bsva;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int ok() {
  g_last_error.clear();
  return BSVA_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(BSVA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// An NVTX range over one entry point (its validation, descriptor encoding and
// launches), named after the entry, so that a profiler timeline shows which
// call issued which kernels. NVTX costs nothing measurable when no tool is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define BSVA_RANGE(name) NvtxRange bsva_nvtx_range_(name)


// ------------------------------------------------------------- device check
int check_device() {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0, minor = 0;
  e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return fail(BSVA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a (B200) only", dev,
                major, minor);
  return BSVA_OK;
}

// ------------------------------------------------------------ validation
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_shape(const bsva_shape& s) {
  if (s.B < 1 || s.H < 1 || s.Lq < 1 || s.Lk < 1)
    return fail(BSVA_ERR_INVALID_ARG, "shape: B, H, Lq, Lk must be >= 1 (got %d, %d, %d, %d)", s.B, s.H, s.Lq, s.Lk);
  if (s.d != 64 && s.d != 128) return fail(BSVA_ERR_UNSUPPORTED, "head dim d = %d; supported: 64, 128", s.d);
  if (s.n_prefix < 0 || s.n_prefix % 128 != 0)
    return fail(BSVA_ERR_INVALID_ARG, "n_prefix = %d must be a non-negative multiple of 128", s.n_prefix);
  if (s.Lq > (1 << 30) || s.Lk > (1 << 30)) return fail(BSVA_ERR_INVALID_ARG, "sequence length too large");
  if (size_t(s.B) * s.H > 65535u) return fail(BSVA_ERR_INVALID_ARG, "B*H must be <= 65535");
  const size_t nQB = (size_t(s.Lq) + 127) / 128;
  if (size_t(s.B) * s.H * nQB > 0x7fffffffu) return fail(BSVA_ERR_INVALID_ARG, "too many query blocks");
  return BSVA_OK;
}

#define REQUIRE_PTR(p, align)                                                                          \
  do {                                                                                                 \
    if ((p) == nullptr) return fail(BSVA_ERR_INVALID_ARG, "%s is NULL", #p);                           \
    if (!aligned((p), (align))) return fail(BSVA_ERR_INVALID_ARG, "%s is not %d-byte aligned", #p, (align)); \
  } while (0)

// ----------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

int get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) return fail(BSVA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  return BSVA_OK;
}

// 3-D map over [heads][rows][inner] with a box of [1][box_rows][box_inner].
int encode_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t inner,
               uint64_t rows, uint64_t heads, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw,
               const char* what) {
  cuuint64_t dims[3] = {inner, rows, heads};
  cuuint64_t strides[2] = {inner * elem_bytes, rows * inner * elem_bytes};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(BSVA_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed with %d", what, int(r));
  return BSVA_OK;
}

int check_workspace(void* ws, size_t bytes, size_t need) {
  if (ws == nullptr) return fail(BSVA_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
  if (!aligned(ws, 256)) return fail(BSVA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (bytes < need) return fail(BSVA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", bytes, need);
  return BSVA_OK;
}

// Shared tail of both attention entry points.
// The INT8 streaming cache as the key side of an attention launch: the K/V maps cover all
// ring slots, key block j lives in slot (first + j / 2) % slots.
struct RingArgs {
  const int32_t* slab_rows = nullptr;
  int first = 0, slots = 0;
};

int run_attention(const bsva_shape& s, const int8_t* q8, const float* q_scale, const int8_t* k8,
                  const float* k_scale, const void* v, const uint8_t* kept_mask, const int32_t* kept_idx,
                  const int32_t* kept_cnt, int centroid_mode, float softmax_scale, int out_dtype, void* out,
                  float* lse, unsigned char* ws, const WsLayout& L, cudaStream_t st,
                  const float* v_scale = nullptr, const int2* vtab = nullptr, const RingArgs& ring = RingArgs()) {
  int rc = get_encoder();
  if (rc) return rc;
  const uint64_t BH = uint64_t(s.B) * s.H;
  const uint64_t krows = ring.slab_rows ? uint64_t(ring.slots) * 128 : uint64_t(s.Lk);   // rows of the K/V maps
  AttnMaps maps;
  const CUtensorMapSwizzle swq = s.d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if ((rc = encode_map(&maps.q8, q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, s.d, s.Lq, BH, s.d, QB, swq, "q8"))) return rc;
  if ((rc = encode_map(&maps.k8, k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, s.d, krows, BH, s.d, KB, swq, "k8"))) return rc;
  if (v_scale) {   // INT8 V: whole rows of d bytes, widened in shared memory by the kernel
    if ((rc = encode_map(&maps.v, v, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, s.d, krows, BH, s.d, KB,
                         CU_TENSOR_MAP_SWIZZLE_NONE, "v8")))
      return rc;
  } else if ((rc = encode_map(&maps.v, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, s.d, s.Lk, BH, 64, KB,
                              CU_TENSOR_MAP_SWIZZLE_128B, "v"))) {
    return rc;
  }
  if (centroid_mode > 0) {
    const uint64_t nCR = uint64_t(L.nCT) * 64;
    if ((rc = encode_map(&maps.ck8, ws + L.ck8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, s.d, nCR, BH, s.d, KB, swq, "ck8")))
      return rc;
    if ((rc = encode_map(&maps.cv, ws + L.cv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, s.d, nCR, BH, 64, KB,
                         CU_TENSOR_MAP_SWIZZLE_128B, "cv")))
      return rc;
  } else {
    maps.ck8 = maps.k8;
    maps.cv = maps.v;
  }
  AttnArgs a{};
  a.B = s.B; a.H = s.H; a.Lq = s.Lq; a.Lk = s.Lk; a.d = s.d; a.n_prefix = s.n_prefix;
  a.nQB = (s.Lq + QB - 1) / QB;
  a.nKB = (s.Lk + KB - 1) / KB;
  a.centroid_mode = centroid_mode;
  a.nCT = L.nCT;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf(float(s.d));
  a.scale_log2e = scale * 1.4426950408889634f;
  a.q_scale = q_scale;
  a.k_scale = k_scale;
  a.kept_idx = kept_idx;
  a.kept_cnt = kept_cnt;
  a.kept_mask = kept_mask;
  a.v_scale = v_scale;
  a.cfac = centroid_mode > 0 ? reinterpret_cast<const float*>(ws + L.cfac) : nullptr;
  a.cbias = centroid_mode > 0 ? reinterpret_cast<const float*>(ws + L.cbias) : nullptr;
  a.vtab = vtab;
  a.n_vtiles = vtab ? L.n_vtiles : 0;
  a.slab_rows = ring.slab_rows;
  a.ring_first = ring.first;
  a.ring_slots = ring.slots;
  a.out = out_dtype == BSVA_OUT_BF16 ? reinterpret_cast<__nv_bfloat16*>(out) : nullptr;
  a.out_f32 = out_dtype == BSVA_OUT_F32 ? reinterpret_cast<float*>(out) : nullptr;
  a.lse = lse;
  a.status = reinterpret_cast<uint32_t*>(ws + L.status);
  a.wait_limit_ns = kWaitLimitNs;
  cudaError_t e = launch_attention(a, maps, st);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return ok();
}

}  // namespace

extern "C" {

int bsva_abi_version(void) { return BSVA_ABI_VERSION; }

const char* bsva_last_error(void) { return g_last_error.c_str(); }

size_t bsva_workspace_bytes(bsva_shape s, int centroid_mode) {
  if (check_shape(s) != BSVA_OK || centroid_mode < 0 || centroid_mode > 2) return 0;
  return ws_layout(s, centroid_mode).total;
}

size_t bsva_route_workspace_bytes(bsva_shape s) {
  if (check_shape(s) != BSVA_OK) return 0;
  return ws_layout(s, 1).route_total;
}

int bsva_quantize_qk(bsva_shape s, const void* q, const void* k, int8_t* q8, float* q_scale, int8_t* k8,
                     float* k_scale, int32_t* q_pool, int32_t* k_pool, bsva_stream_t stream) {
  BSVA_RANGE("bsva_quantize_qk");
  int rc;
  if ((rc = check_shape(s))) return rc;
  REQUIRE_PTR(q, 16); REQUIRE_PTR(k, 16); REQUIRE_PTR(q8, 16); REQUIRE_PTR(k8, 16);
  REQUIRE_PTR(q_scale, 4); REQUIRE_PTR(k_scale, 4); REQUIRE_PTR(q_pool, 16); REQUIRE_PTR(k_pool, 16);
  if ((rc = check_device())) return rc;
  cudaError_t e = launch_quant_pool(s, reinterpret_cast<const __nv_bfloat16*>(q),
                                    reinterpret_cast<const __nv_bfloat16*>(k), q8, q_scale, k8, k_scale, q_pool,
                                    k_pool, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "quant_pool launch");
  return ok();
}

int sparse_attn_route(bsva_shape s, const void* q, const void* k, double tau, int8_t* q8, float* q_scale, int8_t* k8,
                      float* k_scale, int32_t* q_pool, int32_t* k_pool, uint8_t* kept_mask, int32_t* kept_idx,
                      int32_t* kept_cnt, double* row_stats, void* workspace, size_t workspace_bytes,
                      bsva_stream_t stream) {
  BSVA_RANGE("sparse_attn_route");
  int rc;
  if ((rc = check_shape(s))) return rc;
  if (std::isnan(tau)) return fail(BSVA_ERR_INVALID_ARG, "tau is NaN");
  if (std::isinf(tau) && tau > 0) return fail(BSVA_ERR_INVALID_ARG, "tau = +inf is not a routing threshold");
  REQUIRE_PTR(q, 16); REQUIRE_PTR(k, 16); REQUIRE_PTR(q8, 16); REQUIRE_PTR(k8, 16);
  REQUIRE_PTR(q_scale, 4); REQUIRE_PTR(k_scale, 4); REQUIRE_PTR(q_pool, 16); REQUIRE_PTR(k_pool, 16);
  REQUIRE_PTR(kept_mask, 1); REQUIRE_PTR(kept_idx, 4); REQUIRE_PTR(kept_cnt, 4);
  if (row_stats && !aligned(row_stats, 8)) return fail(BSVA_ERR_INVALID_ARG, "row_stats is not 8-byte aligned");
  const WsLayout ws = ws_layout(s, 1);
  if ((rc = check_workspace(workspace, workspace_bytes, ws.route_total))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  double* scores = reinterpret_cast<double*>(static_cast<unsigned char*>(workspace) + ws.scores);
  cudaError_t e = launch_quant_pool(s, reinterpret_cast<const __nv_bfloat16*>(q),
                                    reinterpret_cast<const __nv_bfloat16*>(k), q8, q_scale, k8, k_scale, q_pool,
                                    k_pool, st);
  if (e != cudaSuccess) return cuda_fail(e, "quant_pool launch");
  uint32_t* status = reinterpret_cast<uint32_t*>(static_cast<unsigned char*>(workspace) + ws.status);
  e = launch_route(s, tau, q_pool, k_pool, k_scale, scores, kept_mask, kept_idx, kept_cnt, row_stats, status, st);
  if (e != cudaSuccess) return cuda_fail(e, "route launch");
  return ok();
}

int sparse_attn_route_topk(bsva_shape s, const void* q, const void* k, double sparsity, int8_t* q8,
                           float* q_scale, int8_t* k8, float* k_scale, int32_t* q_pool, int32_t* k_pool,
                           uint8_t* kept_mask, int32_t* kept_idx, int32_t* kept_cnt, double* row_stats,
                           void* workspace, size_t workspace_bytes, bsva_stream_t stream) {
  BSVA_RANGE("sparse_attn_route_topk");
  int rc;
  if ((rc = check_shape(s))) return rc;
  if (!(sparsity >= 0.0 && sparsity <= 1.0)) return fail(BSVA_ERR_INVALID_ARG, "sparsity %g is not in [0, 1]", sparsity);
  REQUIRE_PTR(q, 16); REQUIRE_PTR(k, 16); REQUIRE_PTR(q8, 16); REQUIRE_PTR(k8, 16);
  REQUIRE_PTR(q_scale, 4); REQUIRE_PTR(k_scale, 4); REQUIRE_PTR(q_pool, 16); REQUIRE_PTR(k_pool, 16);
  REQUIRE_PTR(kept_mask, 1); REQUIRE_PTR(kept_idx, 4); REQUIRE_PTR(kept_cnt, 4);
  if (row_stats && !aligned(row_stats, 8)) return fail(BSVA_ERR_INVALID_ARG, "row_stats is not 8-byte aligned");
  const WsLayout ws = ws_layout(s, 1);
  if ((rc = check_workspace(workspace, workspace_bytes, ws.route_total))) return rc;
  if ((rc = check_device())) return rc;
  // kept routed blocks per row: |R| - floor(sparsity * |R|), the product in fp64
  const int nKB = (s.Lk + KB - 1) / KB;
  const int nR = nKB - (s.n_prefix + KB - 1) / KB;
  const int k_keep = nR > 0 ? nR - static_cast<int>(std::floor(sparsity * static_cast<double>(nR))) : 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  double* scores = reinterpret_cast<double*>(static_cast<unsigned char*>(workspace) + ws.scores);
  cudaError_t e = launch_quant_pool(s, reinterpret_cast<const __nv_bfloat16*>(q),
                                    reinterpret_cast<const __nv_bfloat16*>(k), q8, q_scale, k8, k_scale, q_pool,
                                    k_pool, st);
  if (e != cudaSuccess) return cuda_fail(e, "quant_pool launch");
  uint32_t* status = reinterpret_cast<uint32_t*>(static_cast<unsigned char*>(workspace) + ws.status);
  e = launch_route_topk(s, k_keep, q_pool, k_pool, k_scale, scores, kept_mask, kept_idx, kept_cnt, row_stats, status,
                        st);
  if (e != cudaSuccess) return cuda_fail(e, "top-k route launch");
  return ok();
}

int bsva_build_lcsa_mask(int Lq, int Lk, int frame_tokens, int window_frames, int batch, uint8_t* mask,
                         bsva_stream_t stream) {
  BSVA_RANGE("bsva_build_lcsa_mask");
  if (Lq < 1 || Lk < 1 || batch < 1) return fail(BSVA_ERR_INVALID_ARG, "Lq, Lk and batch must be >= 1");
  if (frame_tokens < 1) return fail(BSVA_ERR_INVALID_ARG, "frame_tokens = %d must be >= 1", frame_tokens);
  if (window_frames < 0) return fail(BSVA_ERR_INVALID_ARG, "window_frames = %d must be >= 0", window_frames);
  REQUIRE_PTR(mask, 1);
  int rc;
  if ((rc = check_device())) return rc;
  cudaError_t e = launch_lcsa_mask(Lq, Lk, frame_tokens, window_frames, batch, mask,
                                   reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lcsa mask launch");
  return ok();
}

}  // extern "C"

namespace {

int check_fwd_args(const bsva_shape& s, const int8_t* q8, const float* q_scale, const int8_t* k8,
                   const float* k_scale, const void* v, const uint8_t* kept_mask, const int32_t* kept_idx,
                   const int32_t* kept_cnt, int centroid_mode, float softmax_scale, int out_dtype, void* out,
                   float* lse) {
  int rc;
  if ((rc = check_shape(s))) return rc;
  if (centroid_mode != 1 && centroid_mode != 2)
    return fail(BSVA_ERR_INVALID_ARG, "centroid_mode = %d; use 1 (1x64) or 2 (2x32)", centroid_mode);
  if (std::isnan(softmax_scale) || std::isinf(softmax_scale))
    return fail(BSVA_ERR_INVALID_ARG, "softmax_scale must be finite");
  if (out_dtype != BSVA_OUT_BF16 && out_dtype != BSVA_OUT_F32)
    return fail(BSVA_ERR_INVALID_ARG, "out_dtype = %d; use BSVA_OUT_BF16 (0) or BSVA_OUT_F32 (1)", out_dtype);
  REQUIRE_PTR(q8, 16); REQUIRE_PTR(q_scale, 4); REQUIRE_PTR(k8, 16); REQUIRE_PTR(k_scale, 4);
  REQUIRE_PTR(v, 16); REQUIRE_PTR(kept_mask, 1); REQUIRE_PTR(kept_idx, 4);
  REQUIRE_PTR(kept_cnt, 4); REQUIRE_PTR(out, 16);
  if (lse && !aligned(lse, 4)) return fail(BSVA_ERR_INVALID_ARG, "lse is not 4-byte aligned");
  return BSVA_OK;
}

int check_centroid_args(const bsva_shape& s, const int32_t* k_pool, const float* k_scale, const void* v,
                        int centroid_mode) {
  int rc;
  if ((rc = check_shape(s))) return rc;
  if (centroid_mode != 1 && centroid_mode != 2)
    return fail(BSVA_ERR_INVALID_ARG, "centroid_mode = %d; use 1 (1x64) or 2 (2x32)", centroid_mode);
  REQUIRE_PTR(k_pool, 16); REQUIRE_PTR(k_scale, 4); REQUIRE_PTR(v, 16);
  return BSVA_OK;
}

int build_centroids(const bsva_shape& s, const int32_t* k_pool, const float* k_scale, const void* v,
                    int centroid_mode, unsigned char* ws, const WsLayout& L, cudaStream_t st) {
  cudaError_t e = launch_centroids(s, centroid_mode, L.nCT, k_pool, k_scale, reinterpret_cast<const __nv_bfloat16*>(v),
                                   reinterpret_cast<int8_t*>(ws + L.ck8), reinterpret_cast<__nv_bfloat16*>(ws + L.cv),
                                   reinterpret_cast<float*>(ws + L.cfac), reinterpret_cast<float*>(ws + L.cbias), st);
  if (e != cudaSuccess) return cuda_fail(e, "centroid launch");
  return BSVA_OK;
}

}  // namespace

extern "C" {

int bsva_build_centroids(bsva_shape s, const int32_t* k_pool, const float* k_scale, const void* v,
                         int centroid_mode, void* workspace, size_t workspace_bytes, bsva_stream_t stream) {
  BSVA_RANGE("bsva_build_centroids");
  int rc;
  if ((rc = check_centroid_args(s, k_pool, k_scale, v, centroid_mode))) return rc;
  const WsLayout L = ws_layout(s, centroid_mode);
  if ((rc = check_workspace(workspace, workspace_bytes, L.total))) return rc;
  if ((rc = check_device())) return rc;
  if ((rc = build_centroids(s, k_pool, k_scale, v, centroid_mode, static_cast<unsigned char*>(workspace), L,
                            reinterpret_cast<cudaStream_t>(stream))))
    return rc;
  return ok();
}

int bsva_sparse_attn_core(bsva_shape s, const int8_t* q8, const float* q_scale, const int8_t* k8,
                          const float* k_scale, const void* v, const uint8_t* kept_mask, const int32_t* kept_idx,
                          const int32_t* kept_cnt, int centroid_mode, float softmax_scale, int out_dtype, void* out,
                          float* lse, void* workspace, size_t workspace_bytes, bsva_stream_t stream) {
  BSVA_RANGE("bsva_sparse_attn_core");
  int rc;
  if ((rc = check_fwd_args(s, q8, q_scale, k8, k_scale, v, kept_mask, kept_idx, kept_cnt, centroid_mode,
                           softmax_scale, out_dtype, out, lse)))
    return rc;
  const WsLayout L = ws_layout(s, centroid_mode);
  if ((rc = check_workspace(workspace, workspace_bytes, L.total))) return rc;
  if ((rc = check_device())) return rc;
  return run_attention(s, q8, q_scale, k8, k_scale, v, kept_mask, kept_idx, kept_cnt, centroid_mode, softmax_scale,
                       out_dtype, out, lse, static_cast<unsigned char*>(workspace), L,
                       reinterpret_cast<cudaStream_t>(stream));
}

int sparse_attn_fwd(bsva_shape s, const int8_t* q8, const float* q_scale, const int8_t* k8, const float* k_scale,
                    const int32_t* k_pool, const void* v, const uint8_t* kept_mask, const int32_t* kept_idx,
                    const int32_t* kept_cnt, int centroid_mode, float softmax_scale, int out_dtype, void* out,
                    float* lse, void* workspace, size_t workspace_bytes, bsva_stream_t stream) {
  BSVA_RANGE("sparse_attn_fwd");
  int rc;
  if ((rc = check_fwd_args(s, q8, q_scale, k8, k_scale, v, kept_mask, kept_idx, kept_cnt, centroid_mode,
                           softmax_scale, out_dtype, out, lse)))
    return rc;
  REQUIRE_PTR(k_pool, 16);
  const WsLayout L = ws_layout(s, centroid_mode);
  if ((rc = check_workspace(workspace, workspace_bytes, L.total))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  if ((rc = build_centroids(s, k_pool, k_scale, v, centroid_mode, ws, L, st))) return rc;
  return run_attention(s, q8, q_scale, k8, k_scale, v, kept_mask, kept_idx, kept_cnt, centroid_mode, softmax_scale,
                       out_dtype, out, lse, ws, L, st);
}

int masked_block_attn_fwd(bsva_shape s, const int8_t* q8, const float* q_scale, const int8_t* k8,
                          const float* k_scale, const void* v, const uint8_t* block_mask, int mask_heads,
                          float softmax_scale, int out_dtype, void* out, float* lse, void* workspace,
                          size_t workspace_bytes, bsva_stream_t stream) {
  BSVA_RANGE("masked_block_attn_fwd");
  int rc;
  if ((rc = check_shape(s))) return rc;
  if (mask_heads != 1 && mask_heads != s.H)
    return fail(BSVA_ERR_INVALID_ARG, "mask_heads = %d must be 1 or H = %d", mask_heads, s.H);
  if (std::isnan(softmax_scale) || std::isinf(softmax_scale))
    return fail(BSVA_ERR_INVALID_ARG, "softmax_scale must be finite");
  if (out_dtype != BSVA_OUT_BF16 && out_dtype != BSVA_OUT_F32)
    return fail(BSVA_ERR_INVALID_ARG, "out_dtype = %d; use BSVA_OUT_BF16 (0) or BSVA_OUT_F32 (1)", out_dtype);
  REQUIRE_PTR(q8, 16); REQUIRE_PTR(q_scale, 4); REQUIRE_PTR(k8, 16); REQUIRE_PTR(k_scale, 4);
  REQUIRE_PTR(v, 16); REQUIRE_PTR(block_mask, 1); REQUIRE_PTR(out, 16);
  if (lse && !aligned(lse, 4)) return fail(BSVA_ERR_INVALID_ARG, "lse is not 4-byte aligned");
  const WsLayout L = ws_layout(s, 0);
  if ((rc = check_workspace(workspace, workspace_bytes, L.total))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  int32_t* kidx = reinterpret_cast<int32_t*>(ws + L.kidx);
  int32_t* kcnt = reinterpret_cast<int32_t*>(ws + L.kcnt);
  cudaError_t e = launch_mask_expand(s, block_mask, mask_heads, kidx, kcnt, st);
  if (e != cudaSuccess) return cuda_fail(e, "mask expansion launch");
  return run_attention(s, q8, q_scale, k8, k_scale, v, nullptr, kidx, kcnt, 0, softmax_scale, out_dtype, out, lse,
                       ws, L, st);
}

int bsva_quantize_v(bsva_shape s, const void* v, int8_t* v8, float* v_scale, bsva_stream_t stream) {
  BSVA_RANGE("bsva_quantize_v");
  int rc;
  if ((rc = check_shape(s))) return rc;
  REQUIRE_PTR(v, 16); REQUIRE_PTR(v8, 16); REQUIRE_PTR(v_scale, 4);
  if ((rc = check_device())) return rc;
  cudaError_t e = launch_quant_v(s, reinterpret_cast<const __nv_bfloat16*>(v), v8, v_scale,
                                 reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "V quantiser launch");
  return ok();
}

int masked_block_attn_fwd_v8(bsva_shape s, const int8_t* q8, const float* q_scale, const int8_t* k8,
                             const float* k_scale, const int8_t* v8, const float* v_scale,
                             const uint8_t* block_mask, int mask_heads, float softmax_scale, int out_dtype,
                             void* out, float* lse, void* workspace, size_t workspace_bytes,
                             bsva_stream_t stream) {
  BSVA_RANGE("masked_block_attn_fwd_v8");
  int rc;
  if ((rc = check_shape(s))) return rc;
  if (mask_heads != 1 && mask_heads != s.H)
    return fail(BSVA_ERR_INVALID_ARG, "mask_heads = %d must be 1 or H = %d", mask_heads, s.H);
  if (std::isnan(softmax_scale) || std::isinf(softmax_scale))
    return fail(BSVA_ERR_INVALID_ARG, "softmax_scale must be finite");
  if (out_dtype != BSVA_OUT_BF16 && out_dtype != BSVA_OUT_F32)
    return fail(BSVA_ERR_INVALID_ARG, "out_dtype = %d; use BSVA_OUT_BF16 (0) or BSVA_OUT_F32 (1)", out_dtype);
  REQUIRE_PTR(q8, 16); REQUIRE_PTR(q_scale, 4); REQUIRE_PTR(k8, 16); REQUIRE_PTR(k_scale, 4);
  REQUIRE_PTR(v8, 16); REQUIRE_PTR(v_scale, 4); REQUIRE_PTR(block_mask, 1); REQUIRE_PTR(out, 16);
  if (lse && !aligned(lse, 4)) return fail(BSVA_ERR_INVALID_ARG, "lse is not 4-byte aligned");
  const WsLayout L = ws_layout(s, 0);
  if ((rc = check_workspace(workspace, workspace_bytes, L.total))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  int32_t* kidx = reinterpret_cast<int32_t*>(ws + L.kidx);
  int32_t* kcnt = reinterpret_cast<int32_t*>(ws + L.kcnt);
  cudaError_t e = launch_mask_expand(s, block_mask, mask_heads, kidx, kcnt, st);
  if (e != cudaSuccess) return cuda_fail(e, "mask expansion launch");
  return run_attention(s, q8, q_scale, k8, k_scale, v8, nullptr, kidx, kcnt, 0, softmax_scale, out_dtype, out, lse,
                       ws, L, st, v_scale);
}

int bsva_quantize_q(bsva_shape s, const void* q, int8_t* q8, float* q_scale, int32_t* q_pool, bsva_stream_t stream) {
  BSVA_RANGE("bsva_quantize_q");
  int rc;
  s.Lk = s.Lq;   // not used; keeps the shape check meaningful
  if ((rc = check_shape(s))) return rc;
  REQUIRE_PTR(q, 16); REQUIRE_PTR(q8, 16); REQUIRE_PTR(q_scale, 4); REQUIRE_PTR(q_pool, 16);
  if ((rc = check_device())) return rc;
  cudaError_t e = launch_quant_q(s, reinterpret_cast<const __nv_bfloat16*>(q), q8, q_scale, q_pool,
                                 reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "Q quantiser launch");
  return ok();
}

static int check_kv_cache(const bsva_kv_cache* c) {
  if (c == nullptr) return fail(BSVA_ERR_INVALID_ARG, "cache is NULL");
  if (c->B < 1 || c->H < 1 || size_t(c->B) * c->H > 65535u)
    return fail(BSVA_ERR_INVALID_ARG, "cache: B, H must be >= 1 with B*H <= 65535 (got %d, %d)", c->B, c->H);
  if (c->d != 64 && c->d != 128) return fail(BSVA_ERR_UNSUPPORTED, "cache head dim d = %d; supported: 64, 128", c->d);
  if (c->n_slots < 1 || c->n_slots > (1 << 22)) return fail(BSVA_ERR_INVALID_ARG, "cache n_slots = %d", c->n_slots);
  if (c->first < 0 || c->first >= c->n_slots || c->count < 0 || c->count > c->n_slots)
    return fail(BSVA_ERR_INVALID_ARG, "cache ring state first = %d, count = %d outside [0, %d)", c->first, c->count,
                c->n_slots);
  REQUIRE_PTR(c->k8, 16); REQUIRE_PTR(c->v8, 16); REQUIRE_PTR(c->k_scale, 4); REQUIRE_PTR(c->v_scale, 4);
  REQUIRE_PTR(c->slab_rows, 4);
  return BSVA_OK;
}

int bsva_kv_cache_append(bsva_kv_cache* c, const void* k, const void* v, int Lc, bsva_stream_t stream) {
  BSVA_RANGE("bsva_kv_cache_append");
  int rc;
  if ((rc = check_kv_cache(c))) return rc;
  if (Lc < 1 || Lc > (1 << 30)) return fail(BSVA_ERR_INVALID_ARG, "chunk length %d", Lc);
  REQUIRE_PTR(k, 16); REQUIRE_PTR(v, 16);
  if ((rc = check_device())) return rc;
  const int nslabs = (Lc + 127) / 128;
  const int skip = nslabs > c->n_slots ? nslabs - c->n_slots : 0;   // leading slabs that would be evicted at once
  const int kept = nslabs - skip;
  // evict the oldest slabs to make room, then the chunk's slabs follow the newest one
  const int evict = c->count + kept > c->n_slots ? c->count + kept - c->n_slots : 0;
  const int first = (c->first + evict) % c->n_slots;
  const int count = c->count - evict;
  const int slot0 = (first + count) % c->n_slots;
  cudaError_t e = launch_kv_append(*c, reinterpret_cast<const __nv_bfloat16*>(k),
                                   reinterpret_cast<const __nv_bfloat16*>(v), Lc, skip, slot0,
                                   reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cache append launch");
  c->first = count + kept > 0 ? first : 0;
  c->count = count + kept;
  return ok();
}

static bsva_shape kv_cache_shape(const bsva_kv_cache* c, int Lq) {
  bsva_shape s{};
  s.B = c->B; s.H = c->H; s.Lq = Lq; s.Lk = 128 * (c->count > 0 ? c->count : 1); s.d = c->d; s.n_prefix = 0;
  return s;
}

size_t bsva_kv_cache_workspace_bytes(const bsva_kv_cache* c, int Lq) {
  if (check_kv_cache(c) != BSVA_OK || Lq < 1) return 0;
  const bsva_shape s = kv_cache_shape(c, Lq);
  if (check_shape(s) != BSVA_OK) return 0;
  return ws_layout(s, 0).total;
}

int masked_block_attn_fwd_kvcache(const bsva_kv_cache* c, int Lq, const int8_t* q8, const float* q_scale,
                                  const uint8_t* block_mask, int mask_heads, float softmax_scale, int out_dtype,
                                  void* out, float* lse, void* workspace, size_t workspace_bytes,
                                  bsva_stream_t stream) {
  BSVA_RANGE("masked_block_attn_fwd_kvcache");
  int rc;
  if ((rc = check_kv_cache(c))) return rc;
  if (c->count < 1) return fail(BSVA_ERR_INVALID_ARG, "the cache holds no slab");
  if (Lq < 1) return fail(BSVA_ERR_INVALID_ARG, "Lq = %d", Lq);
  const bsva_shape s = kv_cache_shape(c, Lq);
  if ((rc = check_shape(s))) return rc;
  if (mask_heads != 1 && mask_heads != s.H)
    return fail(BSVA_ERR_INVALID_ARG, "mask_heads = %d must be 1 or H = %d", mask_heads, s.H);
  if (std::isnan(softmax_scale) || std::isinf(softmax_scale))
    return fail(BSVA_ERR_INVALID_ARG, "softmax_scale must be finite");
  if (out_dtype != BSVA_OUT_BF16 && out_dtype != BSVA_OUT_F32)
    return fail(BSVA_ERR_INVALID_ARG, "out_dtype = %d; use BSVA_OUT_BF16 (0) or BSVA_OUT_F32 (1)", out_dtype);
  REQUIRE_PTR(q8, 16); REQUIRE_PTR(q_scale, 4); REQUIRE_PTR(block_mask, 1); REQUIRE_PTR(out, 16);
  if (lse && !aligned(lse, 4)) return fail(BSVA_ERR_INVALID_ARG, "lse is not 4-byte aligned");
  const WsLayout L = ws_layout(s, 0);
  if ((rc = check_workspace(workspace, workspace_bytes, L.total))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  int32_t* kidx = reinterpret_cast<int32_t*>(ws + L.kidx);
  int32_t* kcnt = reinterpret_cast<int32_t*>(ws + L.kcnt);
  const int nQB = (Lq + QB - 1) / QB;
  cudaError_t e = launch_kv_mask_expand(*c, nQB, block_mask, mask_heads, kidx, kcnt, st);
  if (e != cudaSuccess) return cuda_fail(e, "cache mask expansion launch");
  RingArgs ring;
  ring.slab_rows = c->slab_rows;
  ring.first = c->first;
  ring.slots = c->n_slots;
  return run_attention(s, q8, q_scale, c->k8, c->k_scale, c->v8, nullptr, kidx, kcnt, 0, softmax_scale, out_dtype,
                       out, lse, ws, L, st, c->v_scale, nullptr, ring);
}

static int check_virtual_geometry(int slice_tokens, int n_src_slices, int centroid_mode) {
  if (slice_tokens < KB || slice_tokens % KB != 0)
    return fail(BSVA_ERR_INVALID_ARG, "slice_tokens = %d must be a positive multiple of 64", slice_tokens);
  if (n_src_slices < 1) return fail(BSVA_ERR_INVALID_ARG, "n_src_slices = %d must be >= 1", n_src_slices);
  if (size_t(slice_tokens) * size_t(n_src_slices) > (size_t(1) << 30))
    return fail(BSVA_ERR_INVALID_ARG, "source too long: %d slices of %d tokens", n_src_slices, slice_tokens);
  if (centroid_mode != 1 && centroid_mode != 2)
    return fail(BSVA_ERR_INVALID_ARG, "centroid_mode = %d; use 1 (1x64) or 2 (2x32)", centroid_mode);
  return BSVA_OK;
}

size_t bsva_virtual_kv_workspace_bytes(bsva_shape s, int slice_tokens, int n_src_slices, int centroid_mode) {
  if (check_shape(s) != BSVA_OK || check_virtual_geometry(slice_tokens, n_src_slices, centroid_mode) != BSVA_OK)
    return 0;
  return ws_layout_virtual(s, slice_tokens, n_src_slices, 0, centroid_mode).total;
}

int virtual_kv_residual_fwd(bsva_shape s, const int8_t* q8, const float* q_scale, const int8_t* k8,
                            const float* k_scale, const void* v, int slice_tokens, int n_src_slices,
                            const float* src_k_scale, const int32_t* src_k_pool, const void* src_v,
                            const int* src_map, int n_virtual, int centroid_mode, float softmax_scale,
                            int out_dtype, void* out, float* lse, void* workspace, size_t workspace_bytes,
                            bsva_stream_t stream) {
  BSVA_RANGE("virtual_kv_residual_fwd");
  int rc;
  if ((rc = check_shape(s))) return rc;
  if ((rc = check_virtual_geometry(slice_tokens, n_src_slices, centroid_mode))) return rc;
  if (n_virtual < 0 || n_virtual > kMaxVirtualSlices)
    return fail(BSVA_ERR_INVALID_ARG, "n_virtual = %d outside [0, %d]", n_virtual, kMaxVirtualSlices);
  if (n_virtual > 0 && src_map == nullptr) return fail(BSVA_ERR_INVALID_ARG, "src_map is NULL");
  for (int l = 0; l < n_virtual; ++l)
    if (src_map[l] < 0 || src_map[l] >= n_src_slices)
      return fail(BSVA_ERR_INVALID_ARG, "src_map[%d] = %d outside [0, %d)", l, src_map[l], n_src_slices);
  if (std::isnan(softmax_scale) || std::isinf(softmax_scale))
    return fail(BSVA_ERR_INVALID_ARG, "softmax_scale must be finite");
  if (out_dtype != BSVA_OUT_BF16 && out_dtype != BSVA_OUT_F32)
    return fail(BSVA_ERR_INVALID_ARG, "out_dtype = %d; use BSVA_OUT_BF16 (0) or BSVA_OUT_F32 (1)", out_dtype);
  REQUIRE_PTR(q8, 16); REQUIRE_PTR(q_scale, 4); REQUIRE_PTR(k8, 16); REQUIRE_PTR(k_scale, 4);
  REQUIRE_PTR(v, 16); REQUIRE_PTR(out, 16);
  if (n_virtual > 0) {
    REQUIRE_PTR(src_k_scale, 4); REQUIRE_PTR(src_k_pool, 16); REQUIRE_PTR(src_v, 16);
  }
  if (lse && !aligned(lse, 4)) return fail(BSVA_ERR_INVALID_ARG, "lse is not 4-byte aligned");
  const WsLayout L = ws_layout_virtual(s, slice_tokens, n_src_slices, n_virtual, centroid_mode);
  if ((rc = check_workspace(workspace, workspace_bytes, L.total))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  int32_t* kidx = reinterpret_cast<int32_t*>(ws + L.kidx);
  int32_t* kcnt = reinterpret_cast<int32_t*>(ws + L.kcnt);
  cudaError_t e = launch_dense_lists(s, kidx, kcnt, st);
  if (e != cudaSuccess) return cuda_fail(e, "dense list launch");
  if (n_virtual == 0)   // nothing virtual: dense exact attention over the physical keys
    return run_attention(s, q8, q_scale, k8, k_scale, v, nullptr, kidx, kcnt, 0, softmax_scale, out_dtype, out, lse,
                         ws, L, st);
  int2* vtab = reinterpret_cast<int2*>(ws + L.vtab);
  e = launch_virtual_tiles(src_map, n_virtual, slice_tokens / KB * centroid_mode, vtab, st);
  if (e != cudaSuccess) return cuda_fail(e, "virtual tile table launch");
  bsva_shape src = s;
  src.Lk = slice_tokens * n_src_slices;
  if ((rc = build_centroids(src, src_k_pool, src_k_scale, src_v, centroid_mode, ws, L, st))) return rc;
  return run_attention(s, q8, q_scale, k8, k_scale, v, nullptr, kidx, kcnt, centroid_mode, softmax_scale, out_dtype,
                       out, lse, ws, L, st, nullptr, vtab);
}

int bsva_device_checks(void) { return kDeviceChecks ? 1 : 0; }

int bsva_check_status(void* workspace, bsva_stream_t stream) {
  if (workspace == nullptr) return fail(BSVA_ERR_WORKSPACE, "workspace is NULL");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  if (word != 0) {
    e = cudaMemsetAsync(workspace, 0, sizeof(word), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  }
  if (word & kStatusTimeout)
    return fail(BSVA_ERR_DEVICE_TIMEOUT, "a device-side wait ran out of time; outputs of that call are invalid");
  if (word & kStatusBounds)
    return fail(BSVA_ERR_DEVICE_BOUNDS, "a device-side index check failed (kept count, kept list or table row out "
                                        "of range); outputs of that call are invalid");
  return ok();
}

int bsva_selftest_timeout(void* workspace, size_t workspace_bytes, long long limit_ns, bsva_stream_t stream) {
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < 256)
    return fail(BSVA_ERR_WORKSPACE, "workspace must be non-NULL, 256-byte aligned, >= 256 bytes");
  if (limit_ns < 1000 || limit_ns > 1000000000LL)
    return fail(BSVA_ERR_INVALID_ARG, "limit_ns = %lld outside [1e3, 1e9]", limit_ns);
  int rc;
  if ((rc = check_device())) return rc;
  cudaError_t e = launch_selftest_timeout(static_cast<uint32_t*>(workspace), uint64_t(limit_ns),
                                          reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return ok();
}

}  // extern "C"

// --------------------------------------------------- no-allocation variant --
// masked_block_attn_fwd for callers that cannot allocate device memory: the
// kept-block lists live in a scratch array compiled into this library instead
// of a caller workspace. Layout of the array: [0, 256) status word,
// [256, 256 + 4*kNoAllocMaxRows) kept counts, then the kept lists.
namespace {

constexpr size_t kNoAllocMaxRows = size_t(1) << 16;       // B*H*nQB
constexpr size_t kNoAllocMaxEntries = size_t(1) << 21;    // B*H*nQB*nKB
constexpr size_t kNoAllocCntOff = 256;
constexpr size_t kNoAllocIdxOff = kNoAllocCntOff + 4 * kNoAllocMaxRows;
constexpr size_t kNoAllocBytes = kNoAllocIdxOff + 4 * kNoAllocMaxEntries;   // 8,651,008 bytes
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};
unsigned long long g_noalloc_ctx[kNoAllocMaxDevices] = {};   // unique id of the context the address belongs to

using PFN_ctxGetCurrent = CUresult (*)(CUcontext*);
using PFN_ctxGetId = CUresult (*)(CUcontext, unsigned long long*);
PFN_ctxGetCurrent g_ctx_get_current = nullptr;
PFN_ctxGetId g_ctx_get_id = nullptr;
std::once_flag g_ctx_once;

// Unique id of the calling thread's current context, or 0 when none is current
// yet (ids are never reused in a process, unlike context handles).
int current_context_id(unsigned long long* id) {
  std::call_once(g_ctx_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get_current = reinterpret_cast<PFN_ctxGetCurrent>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get_id = reinterpret_cast<PFN_ctxGetId>(fn);
  });
  if (!g_ctx_get_current || !g_ctx_get_id)
    return fail(BSVA_ERR_CUDA, "cuCtxGetCurrent / cuCtxGetId are unavailable from the driver");
  *id = 0;
  CUcontext ctx = nullptr;
  CUresult r = g_ctx_get_current(&ctx);
  if (r != CUDA_SUCCESS) return fail(BSVA_ERR_CUDA, "cuCtxGetCurrent failed with %d", int(r));
  if (ctx == nullptr) return BSVA_OK;
  r = g_ctx_get_id(ctx, id);
  if (r != CUDA_SUCCESS) return fail(BSVA_ERR_CUDA, "cuCtxGetId failed with %d", int(r));
  return BSVA_OK;
}

// Device address of the scratch array in the current device's context. Host
// code cannot use the array's name as a device address, so the address is
// looked up with that device current: on the first call on a device, and
// again whenever the device's context has been recreated (after
// cudaDeviceReset the module can be loaded at another address). The lookup
// itself creates the context when none is current yet.
int noalloc_scratch(unsigned char** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(BSVA_ERR_UNSUPPORTED, "device index %d out of range", dev);
  unsigned long long ctx = 0;
  int rc = current_context_id(&ctx);
  if (rc) return rc;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (ctx == 0 || g_noalloc_ptr[dev] == nullptr || g_noalloc_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    if (ctx == 0 && (rc = current_context_id(&ctx))) return rc;   // the lookup made the context current
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = ctx;
  }
  *out = static_cast<unsigned char*>(g_noalloc_ptr[dev]);
  return BSVA_OK;
}

}  // namespace

extern "C" int masked_block_attn_fwd_noalloc(bsva_shape s, const int8_t* q8, const float* q_scale, const int8_t* k8,
                                             const float* k_scale, const void* v, const uint8_t* block_mask,
                                             int mask_heads, float softmax_scale, int out_dtype, void* out,
                                             float* lse, bsva_stream_t stream) {
  BSVA_RANGE("masked_block_attn_fwd_noalloc");
  int rc;
  if ((rc = check_shape(s))) return rc;
  if (mask_heads != 1 && mask_heads != s.H)
    return fail(BSVA_ERR_INVALID_ARG, "mask_heads = %d must be 1 or H = %d", mask_heads, s.H);
  if (std::isnan(softmax_scale) || std::isinf(softmax_scale))
    return fail(BSVA_ERR_INVALID_ARG, "softmax_scale must be finite");
  if (out_dtype != BSVA_OUT_BF16 && out_dtype != BSVA_OUT_F32)
    return fail(BSVA_ERR_INVALID_ARG, "out_dtype = %d; use BSVA_OUT_BF16 (0) or BSVA_OUT_F32 (1)", out_dtype);
  REQUIRE_PTR(q8, 16); REQUIRE_PTR(q_scale, 4); REQUIRE_PTR(k8, 16); REQUIRE_PTR(k_scale, 4);
  REQUIRE_PTR(v, 16); REQUIRE_PTR(block_mask, 1); REQUIRE_PTR(out, 16);
  if (lse && !aligned(lse, 4)) return fail(BSVA_ERR_INVALID_ARG, "lse is not 4-byte aligned");
  const size_t nQB = (size_t(s.Lq) + QB - 1) / QB, nKB = (size_t(s.Lk) + KB - 1) / KB;
  const size_t rows = size_t(s.B) * s.H * nQB;
  if (rows > kNoAllocMaxRows || rows * nKB > kNoAllocMaxEntries)
    return fail(BSVA_ERR_WORKSPACE,
                "shape needs %zu kept-list rows and %zu entries; the built-in scratch holds at most %zu rows and "
                "%zu entries (use masked_block_attn_fwd with a caller workspace)",
                rows, rows * nKB, kNoAllocMaxRows, kNoAllocMaxEntries);
  if ((rc = check_device())) return rc;
  unsigned char* ws = nullptr;
  if ((rc = noalloc_scratch(&ws))) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the status word must start at zero; the lists are fully rewritten below
  cudaError_t e = cudaMemsetAsync(ws, 0, 256, st);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the scratch status word");
  WsLayout L;
  L.status = 0;
  L.kcnt = kNoAllocCntOff;
  L.kidx = kNoAllocIdxOff;
  L.total = kNoAllocBytes;
  int32_t* kidx = reinterpret_cast<int32_t*>(ws + L.kidx);
  int32_t* kcnt = reinterpret_cast<int32_t*>(ws + L.kcnt);
  e = launch_mask_expand(s, block_mask, mask_heads, kidx, kcnt, st);
  if (e != cudaSuccess) return cuda_fail(e, "mask expansion launch");
  return run_attention(s, q8, q_scale, k8, k_scale, v, nullptr, kidx, kcnt, 0, softmax_scale, out_dtype, out, lse,
                       ws, L, st);
}
