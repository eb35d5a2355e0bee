// common.cuh -- device helpers shared by the sm_100a kernels of the library:
// shared-memory mbarriers with bounded waits, TMA tile loads, tcgen05 (5th-gen
// tensor core) MMA / TMEM wrappers, and the workspace layout.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "bsva.h"

namespace bsva {

constexpr int QB = 128;   // query rows per block (routing granularity)
constexpr int KB = 64;    // key rows per block
constexpr uint32_t kStatusTimeout = 1u;   // workspace status bit: a wait ran out
constexpr uint32_t kStatusBounds = 2u;    // workspace status bit: a device-side index check failed
#ifdef BSVA_DEVICE_CHECKS
constexpr bool kDeviceChecks = true;
#else
constexpr bool kDeviceChecks = false;
#endif

// ---------------------------------------------------------------- workspace --
// Offsets (bytes) of the regions of the caller's workspace. All 256-aligned.
struct WsLayout {
  size_t status = 0;        // uint32 status word (+ padding to 256 B)
  size_t scores = 0;        // fp64  [BH, nQB, nKB] routing scores (first region at a fixed offset)
  size_t route_total = 0;   // bytes a routing call needs (status + scores)
  size_t ck8 = 0;           // int8  [BH, nCR, d]  centroid keys, hi/lo rows
  size_t cv = 0;            // bf16  [BH, nCR, d]  centroid values, hi/lo rows
  size_t cfac = 0;          // fp32  [BH, nCG]     sk_j / |g|
  size_t cbias = 0;         // fp32  [BH, nCG]     log2|g| or -inf
  size_t kidx = 0;          // int32 [BH, nQB, nKB] kept lists (mask entry, virtual K/V)
  size_t kcnt = 0;          // int32 [BH, nQB]
  size_t vtab = 0;          // int2  [n_vtiles] virtual K/V: (first source group, live groups) per tile
  size_t total = 0;
  int nCT = 0;              // centroid tiles per head (64 rows = 32 groups each)
  int n_vtiles = 0;         // virtual K/V: centroid tiles per query block
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout ws_layout(const bsva_shape& s, int centroid_mode) {
  WsLayout w;
  const size_t BH = size_t(s.B) * s.H;
  const int nQB = (s.Lq + QB - 1) / QB, nKB = (s.Lk + KB - 1) / KB;
  size_t off = 256;
  w.scores = off;  off = align256(off + BH * nQB * size_t(nKB) * 8);
  w.route_total = off;
  if (centroid_mode > 0) {
    const int groups = nKB * centroid_mode;
    w.nCT = (groups + 31) / 32;
    const size_t nCR = size_t(w.nCT) * 64, nCG = size_t(w.nCT) * 32;
    w.ck8 = off;   off = align256(off + BH * nCR * s.d);
    w.cv = off;    off = align256(off + BH * nCR * s.d * 2);
    w.cfac = off;  off = align256(off + BH * nCG * 4);
    w.cbias = off; off = align256(off + BH * nCG * 4);
  } else {
    w.kidx = off;  off = align256(off + BH * nQB * size_t(nKB) * 4);
    w.kcnt = off;  off = align256(off + BH * nQB * 4);
  }
  w.total = off;
  return w;
}

// Virtual K/V (residual mode): the physical keys run as dense kept lists, the
// centroid table holds the groups of the source slices, and every added
// virtual slice is ceil(groups per slice / 32) tiles read from its source
// slice's groups.
constexpr int kMaxVirtualSlices = 32;

inline WsLayout ws_layout_virtual(const bsva_shape& s, int slice_tokens, int n_src, int n_virtual,
                                  int centroid_mode) {
  WsLayout w;
  const size_t BH = size_t(s.B) * s.H;
  const int nQB = (s.Lq + QB - 1) / QB, nKB = (s.Lk + KB - 1) / KB;
  const int gps = slice_tokens / KB * centroid_mode;     // groups per slice
  const int tps = (gps + 31) / 32;                       // tiles per virtual slice
  w.nCT = (n_src * gps + 31) / 32;
  w.n_vtiles = n_virtual * tps;
  const size_t nCR = size_t(w.nCT) * 64, nCG = size_t(w.nCT) * 32;
  size_t off = 256;
  w.kidx = off;  off = align256(off + BH * nQB * size_t(nKB) * 4);
  w.kcnt = off;  off = align256(off + BH * nQB * 4);
  w.vtab = off;  off = align256(off + size_t(kMaxVirtualSlices) * tps * 8);
  w.ck8 = off;   off = align256(off + BH * nCR * s.d);
  w.cv = off;    off = align256(off + BH * nCR * s.d * 2);
  w.cfac = off;  off = align256(off + BH * nCG * 4);
  w.cbias = off; off = align256(off + BH * nCG * 4);
  w.total = off;
  return w;
}

// ------------------------------------------------------------------- basics --
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier --
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test for the completion of the phase with the given parity.
// Tests of several barriers issued back to back overlap their latencies.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// BSVA_DEVICE_CHECKS builds: records kStatusBounds when ok is false and returns false, so that
// the caller clamps the value into range; other builds: true, with no code.
__device__ __forceinline__ bool dcheck(bool ok, uint32_t* status) {
  if constexpr (kDeviceChecks) {
    if (!ok) {
      if (status) atomicOr(status, kStatusBounds);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint32_t* status, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort = 1;
      if (status) atomicOr(status, kStatusTimeout);
      return false;
    }
  }
}

// True on exactly one lane of the (converged) warp.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// --------------------------------------------------------------------- TMA --
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ----------------------------------------------------------------- tcgen05 --
__device__ __forceinline__ void tmem_alloc(uint32_t* slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, signed INT8 in, int32 accumulate.
__device__ __forceinline__ void mma_i8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor (kind::i8 / kind::f16, dense, no negate/saturate).
// Bits: [4,6) D format (1 = f32, 2 = s32); [7,10) A format; [10,13) B format
// (i8: 1 = signed; f16: 0 = f16, 1 = bf16); 15 A MN-major; 16 B MN-major;
// [17,23) N >> 3; [24,29) M >> 4.
__host__ __device__ constexpr uint32_t make_idesc(uint32_t d_fmt, uint32_t a_fmt, uint32_t b_fmt, bool a_mn,
                                                  bool b_mn, int M, int N) {
  return (d_fmt << 4) | (a_fmt << 7) | (b_fmt << 10) | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Shared-memory matrix descriptor for tcgen05.mma. Addresses and offsets in
// bytes; the descriptor stores them >> 4. version = 1 (sm_100).
// layout: 0 none, 2 = 128B swizzle, 4 = 64B swizzle, 6 = 32B swizzle.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                               uint32_t layout) {
  uint64_t d = 0;
  d |= uint64_t((smem_addr >> 4) & 0x3FFF);
  d |= uint64_t((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= uint64_t((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(layout & 7) << 61;
  return d;
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Wait for outstanding TMEM loads with the destination registers tied to the
// wait, so that no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
        "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
        "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
        "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
        "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // .x = lo (low 16 bits)
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));   // first source -> upper half
  return r;
}

// Generic-proxy shared-memory stores become visible to the async proxy (tensor core, TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace bsva

// ------------------------------------------------------- host-side launchers --
// Defined next to their kernels; called by api.cu after validation.
namespace bsva {

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per device-side wait

struct AttnArgs {
  int B, H, Lq, Lk, d, n_prefix;
  int nQB, nKB;
  int centroid_mode;        // 0 = exact terms only
  int nCT;                  // centroid tiles per head
  float scale_log2e;        // softmax scale * log2(e)
  const float* q_scale;     // [BH, nQB]
  const float* k_scale;     // [BH, nKB]
  const int32_t* kept_idx;  // [BH, nQB, nKB]
  const int32_t* kept_cnt;  // [BH, nQB]
  const uint8_t* kept_mask; // [BH, nQB, nKB] (centroid exclusion), may be null when mode 0
  const float* v_scale;     // [BH, nKB] per-block scales of an INT8 V (mask entry), null for bf16 V
  const float* cfac;        // [BH, nCT*32]
  const float* cbias;       // [BH, nCT*32]
  const int2* vtab;         // virtual K/V: [n_vtiles] (first source group, live groups); null otherwise
  const int32_t* slab_rows; // INT8 streaming cache: [ring_slots] valid rows per slot; null otherwise
  int ring_first;           // cache: ring slot of the oldest live slab
  int ring_slots;           // cache: slots in the ring
  int n_vtiles;             // virtual K/V: centroid tiles of every query block
  __nv_bfloat16* out;       // [BH, Lq, d] bf16 output, or
  float* out_f32;           // [BH, Lq, d] fp32 output (exactly one is non-null)
  float* lse;               // [BH, Lq] nullable
  uint32_t* status;
  uint64_t wait_limit_ns;
};

struct AttnMaps {
  CUtensorMap q8, k8, v, ck8, cv;
};

cudaError_t launch_quant_pool(const bsva_shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k, int8_t* q8,
                              float* q_scale, int8_t* k8, float* k_scale, int32_t* q_pool, int32_t* k_pool,
                              cudaStream_t st);
// The Q half alone (query codes, scales and pools).
cudaError_t launch_quant_q(const bsva_shape& s, const __nv_bfloat16* q, int8_t* q8, float* q_scale, int32_t* q_pool,
                           cudaStream_t st);
// The K quantiser alone over another [B, H, Lk, d] tensor (INT8 V), no pools.
cudaError_t launch_quant_v(const bsva_shape& s, const __nv_bfloat16* v, int8_t* v8, float* v_scale, cudaStream_t st);
// status: the workspace status word (a score-kernel wait that runs out is recorded there).
cudaError_t launch_route(const bsva_shape& s, double tau, const int32_t* q_pool, const int32_t* k_pool,
                         const float* k_scale, double* scores, uint8_t* kept_mask, int32_t* kept_idx,
                         int32_t* kept_cnt, double* row_stats, uint32_t* status, cudaStream_t st);
cudaError_t launch_route_topk(const bsva_shape& s, int k_keep, const int32_t* q_pool, const int32_t* k_pool,
                              const float* k_scale, double* scores, uint8_t* kept_mask, int32_t* kept_idx,
                              int32_t* kept_cnt, double* row_stats, uint32_t* status, cudaStream_t st);
cudaError_t launch_centroids(const bsva_shape& s, int centroid_mode, int nCT, const int32_t* k_pool,
                             const float* k_scale, const __nv_bfloat16* v, int8_t* ck8, __nv_bfloat16* cv,
                             float* cfac, float* cbias, cudaStream_t st);
cudaError_t launch_lcsa_mask(int Lq, int Lk, int frame_tokens, int window, int batch, uint8_t* mask,
                             cudaStream_t st);
cudaError_t launch_mask_expand(const bsva_shape& s, const uint8_t* block_mask, int mask_heads, int32_t* kept_idx,
                               int32_t* kept_cnt, cudaStream_t st);
// Kept lists with every key block of every query block (virtual K/V: the physical keys stay exact).
cudaError_t launch_dense_lists(const bsva_shape& s, int32_t* kept_idx, int32_t* kept_cnt, cudaStream_t st);
// The virtual-tile table from a source map of n_virtual <= kMaxVirtualSlices host entries.
cudaError_t launch_virtual_tiles(const int* src_map, int n_virtual, int groups_per_slice, int2* vtab,
                                 cudaStream_t st);
cudaError_t launch_attention(const AttnArgs& a, const AttnMaps& maps, cudaStream_t st);
// INT8 streaming cache: quantise a chunk into its slabs (slot0 = slot of the first written
// slab, skip_slabs leading slabs of the chunk dropped), and the kept lists over the live slabs.
cudaError_t launch_kv_append(const bsva_kv_cache& c, const __nv_bfloat16* k, const __nv_bfloat16* v, int Lc,
                             int skip_slabs, int slot0, cudaStream_t st);
cudaError_t launch_kv_mask_expand(const bsva_kv_cache& c, int nQB, const uint8_t* block_mask, int mask_heads,
                                  int32_t* kept_idx, int32_t* kept_cnt, cudaStream_t st);
cudaError_t launch_selftest_timeout(uint32_t* status, uint64_t limit_ns, cudaStream_t st);

}  // namespace bsva
