// route.cu -- proxy block scores and the Sol routing rule.
//
// Method ("Configure Sol Sparse Attention", How it works; The inputs that
// matter): each 128-token query block scores every 64-token key block with a
// cheap proxy on the INT8 tensors and keeps the block exact iff the score is
// at least mean + routing_threshold * std over the row; prefix_policy manual
// keeps the leading tokens dense.
//
// Proxy (reading of the pages; see the header of the public API):
//   dot_ij = sum_c q_pool_i[c] * k_pool_j[c]   (exact: products < 2^27, sums < 2^35, int64)
//   s_ij   = fl64(fl64(dot_ij * sk_j) / n_j)
// Statistics in fp64 over the routed key blocks R_i (start >= n_prefix):
//   mu = sum s / |R|, sigma = sqrt(sum (s - mu)^2 / |R|), T = mu + tau*sigma.
//
// Design: two kernels.
//  score_kernel: per head the dots are a small integer GEMM, [nQB x d] . [d x nKB], run on the
//   tensor core as three INT8 GEMMs over the pools' signed-byte halves (details at the kernel);
//   it writes the fp64 scores to the workspace, [BH, nQB, nKB].
//  select_kernel: one warp per query-block row reduces mu and sigma with shuffles and compacts the
//   kept list with ballots.
//  select_topk_kernel: fixed-sparsity top-k over the same scores ("Ref2VA VSA", 2-stage attention
//   patch: top-k pruning on the generated-video key tiles only). One warp per row finds the k-th
//   largest score by an MSB-first radix select over order-preserving 64-bit keys (8-bit digits,
//   warp-aggregated shared-memory histograms), then keeps every larger score and the lowest-index
//   ties up to k, compacting with ballots.
#include <cmath>

#include "common.cuh"

namespace bsva {
namespace {

constexpr int kThreads = 256;

// ------------------------------------------------------------ proxy scores
// Exact dots on the tensor core. Every pool value is split into two signed bytes,
// x = 128 hi + lo with hi = floor((x + 64) / 128) and lo in [-64, 63]: |q_pool| <= 16256 and
// |k_pool| <= 8128 keep hi in [-127, 127]. Then
//   q . k = 16384 (qh . kh) + 128 (qh . kl + ql . kh) + (ql . kl),
// three INT8 GEMMs with int32 accumulators (each below 127 * 127 * 2 * d < 2^23) combined in
// int64. A CTA owns a tile of 128 query blocks x 64 key blocks: its four byte tiles go to shared
// memory in the K-major swizzled layout tcgen05 reads (128-byte rows with the 128-byte swizzle
// for d = 128, 64-byte rows with the 64-byte swizzle for d = 64), one thread issues the MMAs into
// three 64-column TMEM accumulators, and each warp turns 32 rows x 32 key blocks of dots into
// fp64 scores, fl(fl(dot * sk_j) / n_j) (n_j = 64 is a power of two, so the quotient is the
// product with 1/64, bit for bit), staged through shared memory so that the stores run along
// rows.
constexpr int kSQ = 128;                   // query blocks per CTA (MMA M)
constexpr int kSK = 64;                    // key blocks per CTA (MMA N)
constexpr uint32_t kScoreTmemCols = 256;   // 3 x 64 used; two CTAs per SM
constexpr int kStageLd = 17;               // doubles per staged row (16 + 1 against bank conflicts)

template <int D>
struct __align__(1024) ScoreSmem {
  // the byte tiles; after the MMAs, the same bytes stage each warp's scores
  union {
    struct {
      int8_t qh[kSQ * D];
      int8_t ql[kSQ * D];
      int8_t kh[kSK * D];
      int8_t kl[kSK * D];
    } t;
    double stage[kThreads / 32][32 * kStageLd];
  } u;
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};

// Byte offset of (row r, byte c) of a K-major tile of D-byte rows in the swizzled layout: 8-row
// atoms, the 16-byte chunk index XORed with address bits 7.. (row within the 1024-byte atom for
// 128-byte rows, row / 2 within the 512-byte atom for 64-byte rows).
template <int D>
__device__ __forceinline__ uint32_t swz_offset(int r, int c) {
  if (D == 128) return uint32_t((r >> 3) * 1024 + (r & 7) * 128 + ((((c >> 4) ^ (r & 7)) & 7) << 4) + (c & 15));
  return uint32_t((r >> 3) * 512 + (r & 7) * 64 + ((((c >> 4) ^ ((r >> 1) & 3)) & 3) << 4) + (c & 15));
}

__device__ __forceinline__ void split_bytes(int4 x, uint32_t& hi, uint32_t& lo) {
  const int v[4] = {x.x, x.y, x.z, x.w};
  hi = 0;
  lo = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int h = (v[e] + 64) >> 7;   // arithmetic shift: floor
    const int l = v[e] - (h << 7);
    hi |= uint32_t(h & 0xFF) << (8 * e);
    lo |= uint32_t(l & 0xFF) << (8 * e);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2) score_kernel(const int32_t* __restrict__ q_pool,
                                                            const int32_t* __restrict__ k_pool,
                                                            const float* __restrict__ k_scale,
                                                            double* __restrict__ scores, int Lk, int nQB, int nKB,
                                                            uint32_t* status, uint64_t wait_limit_ns) {
  extern __shared__ unsigned char smem_raw[];
  ScoreSmem<D>& sm =
      *reinterpret_cast<ScoreSmem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int bh = blockIdx.z, i0 = blockIdx.y * kSQ, j0 = blockIdx.x * kSK;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  if (t == 0) {
    mbar_init(&sm.done, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, kScoreTmemCols);
    tmem_relinquish();
  }
  // the byte tiles, four pool values (16 bytes in, 4 bytes out per tile) per step, 8 steps of
  // loads in flight per thread
  constexpr int C4 = D / 4;
  constexpr int kQSteps = kSQ * C4 / kThreads, kKSteps = kSK * C4 / kThreads;
  {
    int4 a[kQSteps];
#pragma unroll
    for (int u = 0; u < kQSteps; ++u) {
      const int idx = t + u * kThreads, r = idx / C4, c4 = idx % C4;
      a[u] = i0 + r < nQB ? __ldg(reinterpret_cast<const int4*>(q_pool + (size_t(bh) * nQB + i0 + r) * D) + c4)
                          : make_int4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kQSteps; ++u) {
      const int idx = t + u * kThreads, r = idx / C4, c4 = idx % C4;
      uint32_t hi, lo;
      split_bytes(a[u], hi, lo);
      const uint32_t off = swz_offset<D>(r, 4 * c4);
      *reinterpret_cast<uint32_t*>(sm.u.t.qh + off) = hi;
      *reinterpret_cast<uint32_t*>(sm.u.t.ql + off) = lo;
    }
    int4 h0[kKSteps], h1[kKSteps];
#pragma unroll
    for (int u = 0; u < kKSteps; ++u) {   // whole key-block pool: the sum of its two 32-row halves
      const int idx = t + u * kThreads, r = idx / C4, c4 = idx % C4;
      h0[u] = h1[u] = make_int4(0, 0, 0, 0);
      if (j0 + r < nKB) {
        const int4* p = reinterpret_cast<const int4*>(k_pool + (size_t(bh) * nKB + j0 + r) * 2 * D);
        h0[u] = __ldg(p + c4);
        h1[u] = __ldg(p + C4 + c4);
      }
    }
#pragma unroll
    for (int u = 0; u < kKSteps; ++u) {
      const int idx = t + u * kThreads, r = idx / C4, c4 = idx % C4;
      uint32_t hi, lo;
      split_bytes(make_int4(h0[u].x + h1[u].x, h0[u].y + h1[u].y, h0[u].z + h1[u].z, h0[u].w + h1[u].w), hi, lo);
      const uint32_t off = swz_offset<D>(r, 4 * c4);
      *reinterpret_cast<uint32_t*>(sm.u.t.kh + off) = hi;
      *reinterpret_cast<uint32_t*>(sm.u.t.kl + off) = lo;
    }
  }
  fence_proxy_async_smem();   // the tensor core reads the tiles
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (t == 0) {
    constexpr uint32_t kLayout = D == 128 ? 2u : 4u;   // 128B / 64B swizzle
    constexpr uint32_t IDESC = make_idesc(2, 1, 1, false, false, kSQ, kSK);
    const uint64_t dqh = make_sdesc(smem_u32(sm.u.t.qh), 16, 8 * D, kLayout);
    const uint64_t dql = make_sdesc(smem_u32(sm.u.t.ql), 16, 8 * D, kLayout);
    const uint64_t dkh = make_sdesc(smem_u32(sm.u.t.kh), 16, 8 * D, kLayout);
    const uint64_t dkl = make_sdesc(smem_u32(sm.u.t.kl), 16, 8 * D, kLayout);
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk) mma_i8_ss(tmem, dqh + 2 * kk, dkh + 2 * kk, IDESC, kk > 0 ? 1u : 0u);
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk) mma_i8_ss(tmem + kSK, dqh + 2 * kk, dkl + 2 * kk, IDESC, kk > 0 ? 1u : 0u);
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk) mma_i8_ss(tmem + kSK, dql + 2 * kk, dkh + 2 * kk, IDESC, 1u);
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk)
      mma_i8_ss(tmem + 2 * kSK, dql + 2 * kk, dkl + 2 * kk, IDESC, kk > 0 ? 1u : 0u);
    tc_commit(&sm.done);
  }
  __syncwarp();
  // once the MMAs are done, their operand bytes are free to stage scores
  if (mbar_wait(&sm.done, 0, &sm.abort, status, wait_limit_ns)) {
    tc_fence_after();
    // warp w: TMEM lanes 32 (w % 4) .. (its 32 query blocks), key-block columns 32 (w / 4) ..
    const int r0 = 32 * (warp & 3), c0 = 32 * (warp >> 2);
    uint32_t d1[32], d2[32], d3[32];
    const uint32_t lane_base = uint32_t(r0) << 16;
    tmem_ld32(tmem + lane_base + c0, d1);
    tmem_ld32(tmem + lane_base + kSK + c0, d2);
    tmem_ld32(tmem + lane_base + 2 * kSK + c0, d3);
    tmem_wait_ld(d1);
    tmem_wait_ld(d2);
    tmem_wait_ld(d3);
    double* stg = sm.u.stage[warp];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      // the row's dots of 16 key blocks into the stage (lane = row)
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int cc = 16 * half + c;
        stg[lane * kStageLd + c] = double(16384ll * int(d1[cc]) + 128ll * int(d2[cc]) + int(d3[cc]));
      }
      __syncwarp();
      // two rows per store: lanes 0-15 and 16-31 each write one row's 16 key blocks
      const int j = j0 + c0 + 16 * half + (lane & 15);
      if (j < nKB) {
        const double skj = double(k_scale[size_t(bh) * nKB + j]);
        const int nj = min(KB, Lk - j * KB);
#pragma unroll 4
        for (int rr = 0; rr < 32; rr += 2) {
          const int row = rr + (lane >> 4);
          const int i = i0 + r0 + row;
          if (i < nQB) {
            const double prod = __dmul_rn(stg[row * kStageLd + (lane & 15)], skj);
            scores[(size_t(bh) * nQB + i) * nKB + j] =
                nj == KB ? __dmul_rn(prod, 1.0 / KB) : __ddiv_rn(prod, double(nj));
          }
        }
      }
      __syncwarp();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kScoreTmemCols);
  }
}

__global__ void __launch_bounds__(kThreads) select_kernel(const double* __restrict__ scores,
                                                          uint8_t* __restrict__ kept_mask,
                                                          int32_t* __restrict__ kept_idx,
                                                          int32_t* __restrict__ kept_cnt,
                                                          double* __restrict__ row_stats, int nQB, int nKB,
                                                          double tau, int tau_is_neginf, int n_prefix) {
  const int bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * (kThreads / 32) + warp;
  if (i >= nQB) return;
  const int jr0 = (n_prefix + KB - 1) / KB;   // first routed key block
  const int nR = nKB - jr0;
  const size_t rowoff = (size_t(bh) * nQB + i) * nKB;
  const double* srow = scores + rowoff;

  double sum = 0.0, mx = -INFINITY, mn = INFINITY;
  for (int j = jr0 + lane; j < nKB; j += 32) {
    const double v = srow[j];
    sum += v;
    mx = fmax(mx, v);
    mn = fmin(mn, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  const double mu = nR > 0 ? sum / nR : 0.0;
  double ss = 0.0;
  for (int j = jr0 + lane; j < nKB; j += 32) {
    const double dv = srow[j] - mu;
    ss += dv * dv;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const double sigma = nR > 0 ? sqrt(ss / nR) : 0.0;
  const bool all_kept = tau_is_neginf || nR <= 0 || i * QB < n_prefix || mx == mn;
  const double T = all_kept ? -INFINITY : __dadd_rn(mu, __dmul_rn(tau, sigma));

  int base = 0;
  for (int j0 = 0; j0 < nKB; j0 += 32) {
    const int j = j0 + lane;
    bool keep = false;
    if (j < nKB) keep = all_kept || j < jr0 || srow[j] >= T;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (j < nKB) {
      kept_mask[rowoff + j] = keep ? 1 : 0;
      if (keep) kept_idx[rowoff + base + __popc(bal & ((1u << lane) - 1u))] = j;
    }
    base += __popc(bal);
  }
  if (lane == 0) {
    kept_cnt[size_t(bh) * nQB + i] = base;
    if (row_stats) {
      double* st = row_stats + (size_t(bh) * nQB + i) * 3;
      st[0] = mu;
      st[1] = sigma;
      st[2] = T;
    }
  }
}

// Order-preserving map of an fp64 score to a uint64 key (larger score, larger key); -0.0 folds to +0.0.
__device__ __forceinline__ unsigned long long score_key(double x) {
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(x + 0.0));
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

__device__ __forceinline__ double key_score(unsigned long long k) {
  const unsigned long long b = (k >> 63) ? (k & 0x7FFFFFFFFFFFFFFFull) : ~k;
  return __longlong_as_double(static_cast<long long>(b));
}

__global__ void __launch_bounds__(kThreads) select_topk_kernel(const double* __restrict__ scores,
                                                               uint8_t* __restrict__ kept_mask,
                                                               int32_t* __restrict__ kept_idx,
                                                               int32_t* __restrict__ kept_cnt,
                                                               double* __restrict__ row_stats, int nQB, int nKB,
                                                               int k_keep, int n_prefix) {
  __shared__ unsigned int hist[kThreads / 32][256];
  const int bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * (kThreads / 32) + warp;
  if (i >= nQB) return;   // whole warps only
  const int jr0 = (n_prefix + KB - 1) / KB;   // first routed key block
  const int nR = nKB - jr0;
  const size_t rowoff = (size_t(bh) * nQB + i) * nKB;
  const double* srow = scores + rowoff;
  const unsigned lt = (1u << lane) - 1u;

  // mu and sigma of the routed scores (diagnostics, as for the Sol rule)
  double sum = 0.0;
  for (int j = jr0 + lane; j < nKB; j += 32) sum += srow[j];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const double mu = nR > 0 ? sum / nR : 0.0;
  double ss = 0.0;
  for (int j = jr0 + lane; j < nKB; j += 32) {
    const double dv = srow[j] - mu;
    ss += dv * dv;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const double sigma = nR > 0 ? sqrt(ss / nR) : 0.0;

  const bool all_kept = nR <= 0 || i * QB < n_prefix || k_keep >= nR;
  unsigned long long tkey = ~0ull;   // keep keys above tkey ...
  int take_eq = 0;                   // ... and the first take_eq keys equal to it, by index
  double T = all_kept ? -INFINITY : INFINITY;
  if (!all_kept && k_keep > 0) {
    unsigned int* h = hist[warp];
    unsigned long long prefix = 0, mask = 0;
    int kr = k_keep;   // rank, from the top, of the wanted key among those matching the prefix
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int b = lane; b < 256; b += 32) h[b] = 0;
      __syncwarp();
      for (int j0 = jr0; j0 < nKB; j0 += 32) {
        const int j = j0 + lane;
        int bin = -1;
        if (j < nKB) {
          const unsigned long long key = score_key(srow[j]);
          if ((key & mask) == prefix) bin = int((key >> shift) & 255u);
        }
        const unsigned same = __match_any_sync(0xffffffffu, bin);
        if (bin >= 0 && lane == __ffs(same) - 1) atomicAdd(&h[bin], unsigned(__popc(same)));
      }
      __syncwarp();
      // lane l owns bins [8l, 8l+8); count the matching keys in higher bins
      unsigned int c[8], tot = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        c[e] = h[8 * lane + e];
        tot += c[e];
      }
      unsigned int incl = tot;   // keys in the bins of lanes >= this lane
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned int v = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += v;
      }
      unsigned int cum = incl - tot;   // keys in bins above this lane's
      int digit = -1;
      unsigned int above = 0;
#pragma unroll
      for (int e = 7; e >= 0; --e) {
        if (digit < 0 && cum < unsigned(kr) && cum + c[e] >= unsigned(kr)) {
          digit = 8 * lane + e;
          above = cum;
        }
        cum += c[e];
      }
      const unsigned who = __ballot_sync(0xffffffffu, digit >= 0);
      const int src = __ffs(who) - 1;   // exactly one lane holds the k-th key's digit
      digit = __shfl_sync(0xffffffffu, digit, src);
      above = __shfl_sync(0xffffffffu, above, src);
      kr -= int(above);
      prefix |= static_cast<unsigned long long>(digit) << shift;
      mask |= 255ull << shift;
      __syncwarp();
    }
    tkey = prefix;
    take_eq = kr;
    T = key_score(tkey);
  }

  int base = 0, eq_seen = 0;
  for (int j0 = 0; j0 < nKB; j0 += 32) {
    const int j = j0 + lane;
    const bool valid = j < nKB;
    bool keep = valid && (all_kept || j < jr0);
    bool eq = false;
    if (valid && !all_kept && j >= jr0 && k_keep > 0) {
      const unsigned long long key = score_key(srow[j]);
      keep = key > tkey;
      eq = key == tkey;
    }
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    if (eq) keep = eq_seen + __popc(eqb & lt) < take_eq;
    eq_seen += __popc(eqb);
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (valid) {
      kept_mask[rowoff + j] = keep ? 1 : 0;
      if (keep) kept_idx[rowoff + base + __popc(bal & lt)] = j;
    }
    base += __popc(bal);
  }
  if (lane == 0) {
    kept_cnt[size_t(bh) * nQB + i] = base;
    if (row_stats) {
      double* st = row_stats + (size_t(bh) * nQB + i) * 3;
      st[0] = mu;
      st[1] = sigma;
      st[2] = T;
    }
  }
}

}  // namespace

static cudaError_t launch_scores(const bsva_shape& s, const int32_t* q_pool, const int32_t* k_pool,
                                 const float* k_scale, double* scores, uint32_t* status, cudaStream_t st) {
  const int nQB = (s.Lq + QB - 1) / QB, nKB = (s.Lk + KB - 1) / KB;
  dim3 g1((nKB + kSK - 1) / kSK, (nQB + kSQ - 1) / kSQ, s.B * s.H);
  // more than a third of an SM's shared memory: at most two CTAs per SM, so that their
  // 256-column TMEM allocations always fit
  const size_t need = (s.d == 128 ? sizeof(ScoreSmem<128>) : sizeof(ScoreSmem<64>)) + 1024;
  const size_t smem = need > 80 * 1024 ? need : 80 * 1024;
  cudaError_t e;
  if (s.d == 128) {
    e = cudaFuncSetAttribute(score_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    score_kernel<128><<<g1, kThreads, smem, st>>>(q_pool, k_pool, k_scale, scores, s.Lk, nQB, nKB, status,
                                                  kWaitLimitNs);
  } else {
    e = cudaFuncSetAttribute(score_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    score_kernel<64><<<g1, kThreads, smem, st>>>(q_pool, k_pool, k_scale, scores, s.Lk, nQB, nKB, status,
                                                 kWaitLimitNs);
  }
  return cudaGetLastError();
}

cudaError_t launch_route_topk(const bsva_shape& s, int k_keep, const int32_t* q_pool, const int32_t* k_pool,
                              const float* k_scale, double* scores, uint8_t* kept_mask, int32_t* kept_idx,
                              int32_t* kept_cnt, double* row_stats, uint32_t* status, cudaStream_t st) {
  const int nQB = (s.Lq + QB - 1) / QB, nKB = (s.Lk + KB - 1) / KB;
  cudaError_t e = launch_scores(s, q_pool, k_pool, k_scale, scores, status, st);
  if (e != cudaSuccess) return e;
  dim3 g2((nQB + kThreads / 32 - 1) / (kThreads / 32), s.B * s.H);
  select_topk_kernel<<<g2, kThreads, 0, st>>>(scores, kept_mask, kept_idx, kept_cnt, row_stats, nQB, nKB, k_keep,
                                              s.n_prefix);
  return cudaGetLastError();
}

cudaError_t launch_route(const bsva_shape& s, double tau, const int32_t* q_pool, const int32_t* k_pool,
                         const float* k_scale, double* scores, uint8_t* kept_mask, int32_t* kept_idx,
                         int32_t* kept_cnt, double* row_stats, uint32_t* status, cudaStream_t st) {
  const int nQB = (s.Lq + QB - 1) / QB, nKB = (s.Lk + KB - 1) / KB;
  cudaError_t e = launch_scores(s, q_pool, k_pool, k_scale, scores, status, st);
  if (e != cudaSuccess) return e;
  const int neginf = std::isinf(tau) && tau < 0;
  dim3 g2((nQB + kThreads / 32 - 1) / (kThreads / 32), s.B * s.H);
  select_kernel<<<g2, kThreads, 0, st>>>(scores, kept_mask, kept_idx, kept_cnt, row_stats, nQB, nKB, tau, neginf,
                                         s.n_prefix);
  return cudaGetLastError();
}

}  // namespace bsva
