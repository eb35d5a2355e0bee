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

}  // namespace

cudaError_t launch_route(const bsva_shape& s, double tau, const int32_t* q_pool, const int32_t* k_pool,
                         const float* k_scale, double* scores, uint8_t* kept_mask, int32_t* kept_idx,
                         int32_t* kept_cnt, double* row_stats, cudaStream_t st) {
  const int nQB = (s.Lq + QB - 1) / QB, nKB = (s.Lk + KB - 1) / KB;
  const int BH = s.B * s.H;
  const size_t smem = size_t(2) * kTile * (s.d + 4) * 4;
  dim3 g1((nKB + kTile - 1) / kTile, (nQB + kTile - 1) / kTile, BH);
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
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int neginf = std::isinf(tau) && tau < 0;
  dim3 g2((nQB + kThreads / 32 - 1) / (kThreads / 32), BH);
  select_kernel<<<g2, kThreads, 0, st>>>(scores, kept_mask, kept_idx, kept_cnt, row_stats, nQB, nKB, tau, neginf,
                                         s.n_prefix);
  return cudaGetLastError();
}

}  // namespace bsva
