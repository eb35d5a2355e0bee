// attn_sm100.cu -- block-sparse INT8 attention with centroid terms, sm_100a.
//
// Method ("Configure Sol Sparse Attention", How it works): for each 128-token
// query block, FlashAttention-style online softmax runs over the kept 64-token
// key blocks only; every skipped block still adds its centroid term(s) in the
// same softmax. The mask entry ("FlashVSR Sparge Attention", How it works)
// runs the same loop over the allowed physical blocks with no centroids.
//
// One CTA = one (b, h, query block) work item, 192 threads:
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r). Reads S from
//              TMEM, scales, online max/sum, writes P (bf16) back to TMEM,
//              rescales O in TMEM when the running max grows by more than
//              2^8, and runs the epilogue O / l.
//   warp 4     TMA producer: Q tile once, then K (int8) and V (bf16) tiles of
//              the kept blocks, then the centroid tiles, NS-stage ring.
//   warp 5     TMEM owner (alloc/dealloc) and single-thread MMA issuer:
//              S = Q8 . K8^T with tcgen05.mma kind::i8 (M=128, N=64, int32
//              accumulate) and O += P . V with kind::f16 (A = P from TMEM,
//              B = V from shared memory, fp32 accumulate). S is double
//              buffered so QK of tile n+1 overlaps the softmax of tile n.
// Centroid tiles hold 32 groups as (hi, lo) INT8 row pairs (pool = 128 hi + lo)
// so their dot with q8 is exact in int32; the value rows are (bf16 hi, bf16 lo)
// and share one probability.
// Every wait is bounded: on a timeout the CTA records it in the workspace
// status word, all roles leave their loops, TMEM is freed and the CTA exits.
#include <cmath>

#include "common.cuh"

namespace bsva {
namespace {

constexpr int NS = 3;           // K/V pipeline stages
constexpr int kThreads = 192;
constexpr float kRescaleLog2 = 8.0f;   // lazy O rescale threshold (factor 256)
constexpr uint32_t kTmemCols = 256;

template <int D>
struct __align__(1024) Smem {
  int8_t q[QB * D];
  int8_t k[NS][KB * D];
  __nv_bfloat16 v[NS][KB * D];
  uint64_t q_full;
  uint64_t kv_full[NS];
  uint64_t kv_empty[NS];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done;
  uint64_t o_full;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    attn_kernel(const AttnArgs a, const __grid_constant__ AttnMaps maps) {
  extern __shared__ unsigned char smem_raw[];
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int item = a.order ? a.order[blockIdx.x] : int(blockIdx.x);
  const int bh = item / a.nQB;
  const int i = item % a.nQB;
  const size_t row_item = size_t(bh) * a.nQB + i;

  const int n_exact = a.kept_cnt[row_item];
  const int n_cent = (a.centroid_mode > 0 && n_exact < a.nKB) ? a.nCT : 0;
  const int N = n_exact + n_cent;
  const int q0 = i * QB;

  if (N == 0) {   // nothing to attend: o = 0, lse = -inf
    if (tid < QB && q0 + tid < a.Lq) {
      const size_t orow = (size_t(bh) * a.Lq + q0 + tid) * D;
      uint4* o = a.out_f32 ? reinterpret_cast<uint4*>(a.out_f32 + orow) : reinterpret_cast<uint4*>(a.out + orow);
      const int n16 = a.out_f32 ? D / 4 : D / 8;
      for (int c = 0; c < n16; ++c) o[c] = make_uint4(0, 0, 0, 0);
      if (a.lse) a.lse[size_t(bh) * a.Lq + q0 + tid] = -INFINITY;
    }
    return;
  }

  constexpr uint32_t O_COL = 0;
  constexpr uint32_t S_COL0 = D, S_COL1 = D + 64;

  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.p_full[b], QB);
    }
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.o_full, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;
  const uint64_t lim = a.wait_limit_ns;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&maps.q8);
      tma_prefetch_desc(&maps.k8);
      tma_prefetch_desc(&maps.v);
      mbar_arrive_expect_tx(&sm.q_full, QB * D);
      tma_load_3d(sm.q, &maps.q8, 0, q0, bh, &sm.q_full);
      const int32_t* kidx = a.kept_idx + row_item * a.nKB;
      for (int n = 0; n < N; ++n) {
        const int s = n % NS;
        if (n >= NS && !mbar_wait(&sm.kv_empty[s], ((n / NS) - 1) & 1, abort, a.status, lim)) break;
        mbar_arrive_expect_tx(&sm.kv_full[s], KB * D * 3);
        const CUtensorMap* mk;
        const CUtensorMap* mv;
        int row;
        if (n < n_exact) {
          row = kidx[n] * KB;
          mk = &maps.k8;
          mv = &maps.v;
        } else {
          row = (n - n_exact) * KB;
          mk = &maps.ck8;
          mv = &maps.cv;
        }
        tma_load_3d(sm.k[s], mk, 0, row, bh, &sm.kv_full[s]);
        tma_load_3d(sm.v[s], mv, 0, row, bh, &sm.kv_full[s]);
        if (D == 128) tma_load_3d(sm.v[s] + KB * 64, mv, 64, row, bh, &sm.kv_full[s]);
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      // K-major INT8 tiles: rows of D bytes, 8-row groups of 8*D bytes.
      constexpr uint32_t kLayoutQK = (D == 128) ? 2u : 4u;   // 128B / 64B swizzle
      constexpr uint32_t kSboQK = 8 * D;
      // V tiles, MN-major bf16: 128-byte rows (64 d-values), 8-row groups of
      // 1 KB, the two 64-column halves (D = 128) 8 KB apart.
      constexpr uint32_t kLboV = KB * 128, kSboV = 1024;
      constexpr uint32_t IDESC_QK = make_idesc(2, 1, 1, false, false, 128, 64);
      constexpr uint32_t IDESC_PV = make_idesc(1, 1, 1, false, true, 128, D);
      const uint64_t dq = make_sdesc(smem_u32(sm.q), 16, kSboQK, kLayoutQK);
      bool ok = mbar_wait(&sm.q_full, 0, abort, a.status, lim);
      tc_fence_after();

      auto issue_qk = [&](int n) -> bool {
        const int s = n % NS;
        if (!mbar_wait(&sm.kv_full[s], (n / NS) & 1, abort, a.status, lim)) return false;
        tc_fence_after();
        const uint64_t dk = make_sdesc(smem_u32(sm.k[s]), 16, kSboQK, kLayoutQK);
        const uint32_t dS = tmem + ((n & 1) ? S_COL1 : S_COL0);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)   // K = 32 bytes per MMA
          mma_i8_ss(dS, dq + 2 * kk, dk + 2 * kk, IDESC_QK, kk > 0 ? 1u : 0u);
        tc_commit(&sm.s_full[n & 1]);
        return true;
      };
      auto issue_pv = [&](int n) -> bool {
        if (!mbar_wait(&sm.p_full[n & 1], (n >> 1) & 1, abort, a.status, lim)) return false;
        tc_fence_after();
        const int s = n % NS;
        const uint64_t dv = make_sdesc(smem_u32(sm.v[s]), kLboV, kSboV, 2u);
        const uint32_t aP = tmem + ((n & 1) ? S_COL1 : S_COL0);
#pragma unroll
        for (int kk = 0; kk < KB / 16; ++kk)   // K = 16 keys per MMA: 8 TMEM columns of P, 16 rows of V
          mma_bf16_ts(tmem + O_COL, aP + 8 * kk, dv + (16 * 128 / 16) * kk, IDESC_PV,
                      (n > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&sm.kv_empty[s]);
        tc_commit(&sm.pv_done);
        return true;
      };

      if (ok) ok = issue_qk(0);
      for (int n = 0; ok && n < N; ++n) {
        if (n + 1 < N) ok = issue_qk(n + 1);
        if (ok) ok = issue_pv(n);
      }
      tc_commit(&sm.o_full);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int r = tid;                                   // row within the block
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const float sqs = a.q_scale[row_item] * a.scale_log2e;
    const int32_t* kidx = a.kept_idx + row_item * a.nKB;
    const uint8_t* kmask = a.kept_mask ? a.kept_mask + row_item * a.nKB : nullptr;
    const float* cfac = a.cfac + size_t(bh) * a.nCT * 32;
    const float* cbias = a.cbias + size_t(bh) * a.nCT * 32;
    float m_ref = -INFINITY, l = 0.f, le = 0.f;
    bool alive = true;

    for (int n = 0; n < N; ++n) {
      const bool exact = n < n_exact;
      float f = 0.f;
      int nvalid = 0;
      float gf[32], gb[32];
      if (exact) {
        const int j = kidx[n];
        f = sqs * a.k_scale[size_t(bh) * a.nKB + j];
        nvalid = min(KB, a.Lk - j * KB);
      } else {
        const int t = n - n_exact;
        const float4* fp = reinterpret_cast<const float4*>(cfac + t * 32);
        const float4* bp = reinterpret_cast<const float4*>(cbias + t * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 fv = fp[q], bv = bp[q];
          gf[4 * q] = fv.x; gf[4 * q + 1] = fv.y; gf[4 * q + 2] = fv.z; gf[4 * q + 3] = fv.w;
          gb[4 * q] = bv.x; gb[4 * q + 1] = bv.y; gb[4 * q + 2] = bv.z; gb[4 * q + 3] = bv.w;
        }
#pragma unroll
        for (int g = 0; g < 32; ++g) {
          const int jb = (t * 32 + g) / a.centroid_mode;
          const bool kept = jb < a.nKB && kmask[jb];
          gf[g] *= sqs;
          if (kept) gb[g] = -INFINITY;
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[n & 1], (n >> 1) & 1, abort, a.status, lim))) {
        alive = false;
        break;
      }
      tc_fence_after();
      const uint32_t sc = (n & 1) ? S_COL1 : S_COL0;
      uint32_t sr[64];
      tmem_ld64(tmem + lane_base + sc, sr);
      tmem_wait_ld();

      float x[64];
      float mt = -INFINITY;
      if (exact) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          x[c] = (c < nvalid) ? float(int(sr[c])) * f : -INFINITY;
          mt = fmaxf(mt, x[c]);
        }
      } else {
#pragma unroll
        for (int g = 0; g < 32; ++g) {
          const int dot = 128 * int(sr[2 * g]) + int(sr[2 * g + 1]);
          x[g] = (gb[g] == -INFINITY) ? -INFINITY : fmaf(float(dot), gf[g], gb[g]);
          mt = fmaxf(mt, x[g]);
        }
      }

      // lazy rescale: only when the running max grows by more than 2^8
      const bool need = mt > m_ref + kRescaleLog2;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? mt : m_ref;
        const float alpha = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - m_new);
        if (n > 0) {
          if (!__all_sync(0xffffffffu, mbar_wait(&sm.pv_done, (n - 1) & 1, abort, a.status, lim))) {
            alive = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_base + O_COL + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tmem + lane_base + O_COL + c0, o);
          }
          tmem_wait_st();
        }
        l *= alpha;
        le *= alpha;
        m_ref = m_new;
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;

      uint32_t pk[32];
      float lsum = 0.f;
      // Two row sums: lb adds the bf16-rounded weights that the PV product uses
      // (numerator and denominator then see the same probabilities), le adds
      // the unrounded weights for the log-sum-exp.
      float esum = 0.f;
      if (exact) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float p0 = ex2(x[2 * c] - m_use), p1 = ex2(x[2 * c + 1] - m_use);
          pk[c] = pack_bf16x2(p0, p1);
          lsum += __uint_as_float(pk[c] << 16) + __uint_as_float(pk[c] & 0xFFFF0000u);
          esum += p0 + p1;
        }
      } else {
#pragma unroll
        for (int g = 0; g < 32; ++g) {
          const float p = ex2(x[g] - m_use);
          pk[g] = pack_bf16x2(p, p);
          lsum += __uint_as_float(pk[g] << 16);
          esum += p;
        }
      }
      l += lsum;
      le += esum;
      tmem_st32(tmem + lane_base + sc, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[n & 1]);
    }

    // ------------------------------------------------------------ epilogue
    if (alive && __all_sync(0xffffffffu, mbar_wait(&sm.o_full, 0, abort, a.status, lim))) {
      tc_fence_after();
      const int qr = q0 + r;
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      const size_t orow = (size_t(bh) * a.Lq + qr) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + O_COL + c0, o);
        tmem_wait_ld();
        if (qr < a.Lq) {
          if (a.out_f32) {
            float4* dst = reinterpret_cast<float4*>(a.out_f32 + orow + c0);
#pragma unroll
            for (int c = 0; c < 8; ++c)
              dst[c] = make_float4(__uint_as_float(o[4 * c]) * inv_l, __uint_as_float(o[4 * c + 1]) * inv_l,
                                   __uint_as_float(o[4 * c + 2]) * inv_l, __uint_as_float(o[4 * c + 3]) * inv_l);
          } else {
            uint4 w[4];
            uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
            for (int c = 0; c < 16; ++c)
              wp[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
            uint4* dst = reinterpret_cast<uint4*>(a.out + orow + c0);
#pragma unroll
            for (int c = 0; c < 4; ++c) dst[c] = w[c];
          }
        }
      }
      if (a.lse && qr < a.Lq)
        a.lse[size_t(bh) * a.Lq + qr] = le > 0.f ? (m_ref + __log2f(le)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
cudaError_t launch_attn_d(const AttnArgs& a, const AttnMaps& maps, cudaStream_t st) {
  // At least 100 KB so that no more than two CTAs share an SM: two 256-column
  // TMEM allocations fill the SM's 512 columns.
  const size_t smem = sizeof(Smem<D>) + 1024 > 100 * 1024 ? sizeof(Smem<D>) + 1024 : 100 * 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const unsigned grid = unsigned(a.B) * a.H * a.nQB;
  attn_kernel<D><<<grid, kThreads, smem, st>>>(a, maps);
  return cudaGetLastError();
}

// One CTA waits on a barrier nothing arrives at; the bounded wait runs out.
__global__ void selftest_timeout_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort, status, limit_ns);
  __syncthreads();
}

}  // namespace

cudaError_t launch_attention(const AttnArgs& a, const AttnMaps& maps, cudaStream_t st) {
  return a.d == 128 ? launch_attn_d<128>(a, maps, st) : launch_attn_d<64>(a, maps, st);
}

cudaError_t launch_selftest_timeout(uint32_t* status, uint64_t limit_ns, cudaStream_t st) {
  selftest_timeout_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace bsva
