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
// Design: one CTA of 256 threads owns TQ query-block rows of one (b, h). The
// head's whole-block K pools stream through shared memory in tiles of 32 key
// blocks (rows padded to d+1 words: conflict-free), each thread computes one
// (row, key block) dot per tile, and the fp64 scores of the CTA's rows stay in
// shared memory (TQ x nKB x 8 bytes). Then one warp per row reduces mu and
// sigma with warp shuffles and compacts the kept list with ballots.
#include <cmath>

#include "common.cuh"

namespace bsva {
namespace {

constexpr int kThreads = 256;
constexpr int kTileJ = 32;
constexpr int kMaxSmem = 200 * 1024;

template <int D>
__global__ void __launch_bounds__(kThreads) route_kernel(const int32_t* __restrict__ q_pool,
                                                         const int32_t* __restrict__ k_pool,
                                                         const float* __restrict__ k_scale,
                                                         uint8_t* __restrict__ kept_mask,
                                                         int32_t* __restrict__ kept_idx,
                                                         int32_t* __restrict__ kept_cnt,
                                                         double* __restrict__ row_stats, int Lk, int nQB,
                                                         int nKB, int TQ, double tau, int tau_is_neginf,
                                                         int n_prefix) {
  extern __shared__ __align__(16) unsigned char smem[];
  double* s_score = reinterpret_cast<double*>(smem);                        // [TQ][nKB]
  int32_t* s_q = reinterpret_cast<int32_t*>(s_score + size_t(TQ) * nKB);    // [TQ][D]
  int32_t* s_k = s_q + TQ * D;                                              // [kTileJ][D+1]

  const int bh = blockIdx.y;
  const int i0 = blockIdx.x * TQ;
  const int nrows = min(TQ, nQB - i0);
  const int t = threadIdx.x;

  for (int idx = t; idx < nrows * D; idx += kThreads)
    s_q[idx] = q_pool[(size_t(bh) * nQB + i0) * D + idx];

  // ---- scores
  for (int j0 = 0; j0 < nKB; j0 += kTileJ) {
    __syncthreads();
    const int nj = min(kTileJ, nKB - j0);
    for (int idx = t; idx < nj * D; idx += kThreads) {
      const int jj = idx / D, c = idx % D;
      const int32_t* p = k_pool + (size_t(bh) * nKB + j0 + jj) * 2 * D;
      s_k[jj * (D + 1) + c] = p[c] + p[D + c];
    }
    __syncthreads();
    for (int w = t; w < nrows * kTileJ; w += kThreads) {
      const int r = w / kTileJ, jj = w % kTileJ;
      if (jj >= nj) continue;
      const int32_t* a = s_q + r * D;
      const int32_t* b = s_k + jj * (D + 1);
      long long acc = 0;
#pragma unroll 16
      for (int c = 0; c < D; ++c) acc += (long long)a[c] * b[c];
      const int j = j0 + jj;
      const int nj_rows = min(KB, Lk - j * KB);
      const double prod = __dmul_rn((double)acc, (double)k_scale[size_t(bh) * nKB + j]);
      s_score[size_t(r) * nKB + j] = __ddiv_rn(prod, (double)nj_rows);
    }
  }
  __syncthreads();

  // ---- statistics and compaction: one warp per row
  const int warp = t >> 5, lane = t & 31;
  const int jr0 = (n_prefix + KB - 1) / KB;   // first routed key block
  const int nR = nKB - jr0;
  for (int r = warp; r < nrows; r += kThreads / 32) {
    const int i = i0 + r;
    const double* srow = s_score + size_t(r) * nKB;
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

    const size_t rowoff = (size_t(bh) * nQB + i) * nKB;
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
}

}  // namespace

// Rows per CTA so that the fp64 score rows fit the shared-memory budget.
static int route_rows_per_cta(int nKB, int d) {
  const int fixed = kTileJ * (d + 1) * 4;
  for (int tq = 8; tq >= 1; --tq)
    if (size_t(tq) * nKB * 8 + size_t(tq) * d * 4 + fixed <= size_t(kMaxSmem)) return tq;
  return 0;
}

bool route_supported(int nKB, int d) { return route_rows_per_cta(nKB, d) > 0; }

cudaError_t launch_route(const bsva_shape& s, double tau, const int32_t* q_pool, const int32_t* k_pool,
                         const float* k_scale, uint8_t* kept_mask, int32_t* kept_idx, int32_t* kept_cnt,
                         double* row_stats, cudaStream_t st) {
  const int nQB = (s.Lq + QB - 1) / QB, nKB = (s.Lk + KB - 1) / KB;
  const int TQ = route_rows_per_cta(nKB, s.d);
  if (TQ == 0) return cudaErrorInvalidValue;
  const size_t smem = size_t(TQ) * nKB * 8 + size_t(TQ) * s.d * 4 + size_t(kTileJ) * (s.d + 1) * 4;
  dim3 grid((nQB + TQ - 1) / TQ, s.B * s.H);
  const int neginf = std::isinf(tau) && tau < 0;
  cudaError_t e;
  if (s.d == 128) {
    e = cudaFuncSetAttribute(route_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e != cudaSuccess) return e;
    route_kernel<128><<<grid, kThreads, smem, st>>>(q_pool, k_pool, k_scale, kept_mask, kept_idx, kept_cnt,
                                                    row_stats, s.Lk, nQB, nKB, TQ, tau, neginf, s.n_prefix);
  } else {
    e = cudaFuncSetAttribute(route_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e != cudaSuccess) return e;
    route_kernel<64><<<grid, kThreads, smem, st>>>(q_pool, k_pool, k_scale, kept_mask, kept_idx, kept_cnt,
                                                   row_stats, s.Lk, nQB, nKB, TQ, tau, neginf, s.n_prefix);
  }
  return cudaGetLastError();
}

}  // namespace bsva
