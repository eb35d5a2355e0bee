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
//  score_kernel: per head the dots are a small integer GEMM, [nQB x d] . [d x nKB]. A CTA of 256
//   threads owns a 64 x 64 tile of (query block, key block); both pool tiles are staged in shared
//   memory (rows padded to d+4 words: conflict-free 16-byte loads), each thread accumulates a 4 x 4
//   block of dots (query blocks ty+16a, key blocks tx+16b) in int32 over 16 dims at a time (|q_pool|
//   <= 16256 and |k_pool| <= 8128, so 16 products stay below 2^31) and in int64 across them, and
//   writes the fp64 scores to the workspace, [BH, nQB, nKB].
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
constexpr int kTile = 64;

template <int D>
__global__ void __launch_bounds__(kThreads, 2) score_kernel(const int32_t* __restrict__ q_pool,
                                                            const int32_t* __restrict__ k_pool,
                                                            const float* __restrict__ k_scale,
                                                            double* __restrict__ scores, int Lk, int nQB,
                                                            int nKB) {
  constexpr int KS = D + 4;
  constexpr int C4 = D / 4;
  extern __shared__ __align__(16) int32_t sm[];
  int32_t* sq = sm;                 // [kTile][KS] query-block pools
  int32_t* sk = sm + kTile * KS;    // [kTile][KS] whole key-block pools (sum of the two halves)
  const int bh = blockIdx.z, i0 = blockIdx.y * kTile, j0 = blockIdx.x * kTile;
  const int t = threadIdx.x;

  for (int idx = t; idx < kTile * C4; idx += kThreads) {
    const int r = idx / C4, c4 = idx % C4;
    int4 a = make_int4(0, 0, 0, 0), b = make_int4(0, 0, 0, 0);
    if (i0 + r < nQB) a = __ldg(reinterpret_cast<const int4*>(q_pool + (size_t(bh) * nQB + i0 + r) * D) + c4);
    if (j0 + r < nKB) {
      const int4* p = reinterpret_cast<const int4*>(k_pool + (size_t(bh) * nKB + j0 + r) * 2 * D);
      const int4 h0 = __ldg(p + c4), h1 = __ldg(p + C4 + c4);
      b = make_int4(h0.x + h1.x, h0.y + h1.y, h0.z + h1.z, h0.w + h1.w);
    }
    *reinterpret_cast<int4*>(sq + r * KS + 4 * c4) = a;
    *reinterpret_cast<int4*>(sk + r * KS + 4 * c4) = b;
  }
  __syncthreads();

  const int tx = t & 15, ty = t >> 4;
  long long acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0;
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += 16) {
    int part[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) part[a][b] = 0;
#pragma unroll
    for (int c = c0; c < c0 + 16; c += 4) {
      int4 x[4], y[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) x[a] = *reinterpret_cast<const int4*>(sq + (ty + 16 * a) * KS + c);
#pragma unroll
      for (int b = 0; b < 4; ++b) y[b] = *reinterpret_cast<const int4*>(sk + (tx + 16 * b) * KS + c);
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
          part[a][b] += x[a].x * y[b].x + x[a].y * y[b].y + x[a].z * y[b].z + x[a].w * y[b].w;
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] += part[a][b];
  }

#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const int j = j0 + tx + 16 * b;
    if (j >= nKB) continue;
    const double skj = (double)k_scale[size_t(bh) * nKB + j];
    const double nj = (double)min(KB, Lk - j * KB);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int i = i0 + ty + 16 * a;
      if (i < nQB) scores[(size_t(bh) * nQB + i) * nKB + j] = __ddiv_rn(__dmul_rn((double)acc[a][b], skj), nj);
    }
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
                                 const float* k_scale, double* scores, cudaStream_t st) {
  const int nQB = (s.Lq + QB - 1) / QB, nKB = (s.Lk + KB - 1) / KB;
  const size_t smem = size_t(2) * kTile * (s.d + 4) * 4;
  dim3 g1((nKB + kTile - 1) / kTile, (nQB + kTile - 1) / kTile, s.B * s.H);
  cudaError_t e;
  if (s.d == 128) {
    e = cudaFuncSetAttribute(score_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    score_kernel<128><<<g1, kThreads, smem, st>>>(q_pool, k_pool, k_scale, scores, s.Lk, nQB, nKB);
  } else {
    e = cudaFuncSetAttribute(score_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    score_kernel<64><<<g1, kThreads, smem, st>>>(q_pool, k_pool, k_scale, scores, s.Lk, nQB, nKB);
  }
  return cudaGetLastError();
}

cudaError_t launch_route_topk(const bsva_shape& s, int k_keep, const int32_t* q_pool, const int32_t* k_pool,
                              const float* k_scale, double* scores, uint8_t* kept_mask, int32_t* kept_idx,
                              int32_t* kept_cnt, double* row_stats, cudaStream_t st) {
  const int nQB = (s.Lq + QB - 1) / QB, nKB = (s.Lk + KB - 1) / KB;
  cudaError_t e = launch_scores(s, q_pool, k_pool, k_scale, scores, st);
  if (e != cudaSuccess) return e;
  dim3 g2((nQB + kThreads / 32 - 1) / (kThreads / 32), s.B * s.H);
  select_topk_kernel<<<g2, kThreads, 0, st>>>(scores, kept_mask, kept_idx, kept_cnt, row_stats, nQB, nKB, k_keep,
                                              s.n_prefix);
  return cudaGetLastError();
}

cudaError_t launch_route(const bsva_shape& s, double tau, const int32_t* q_pool, const int32_t* k_pool,
                         const float* k_scale, double* scores, uint8_t* kept_mask, int32_t* kept_idx,
                         int32_t* kept_cnt, double* row_stats, cudaStream_t st) {
  const int nQB = (s.Lq + QB - 1) / QB, nKB = (s.Lk + KB - 1) / KB;
  cudaError_t e = launch_scores(s, q_pool, k_pool, k_scale, scores, st);
  if (e != cudaSuccess) return e;
  const int neginf = std::isinf(tau) && tau < 0;
  dim3 g2((nQB + kThreads / 32 - 1) / (kThreads / 32), s.B * s.H);
  select_kernel<<<g2, kThreads, 0, st>>>(scores, kept_mask, kept_idx, kept_cnt, row_stats, nQB, nKB, tau, neginf,
                                         s.n_prefix);
  return cudaGetLastError();
}

}  // namespace bsva
