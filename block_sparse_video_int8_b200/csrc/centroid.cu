// centroid.cu -- per-head centroid table for the skipped-block correction.
//
// Method ("Configure Sol Sparse Attention", How it works): a skipped 64-token
// key block is replaced by one centroid (1x64) or two 32-token centroids
// (2x32) that still enter the online softmax. For group g of key block j:
//   kbar_g = sk_j * pool_g / |g|        (pool_g: int32 column sums of the INT8 K rows)
//   logit  = sq_i * scale * (q8_r . kbar_g) + ln|g|,   value vbar_g = mean of V over g.
//
// Layout written here (consumed by the attention kernel as extra 64-row tiles):
//   ck8 [BH, nCT*64, d] int8 : row 2G = hi, row 2G+1 = lo with pool = 128*hi + lo,
//        hi = pool >> 7 in [-64, 63], lo = pool & 127 in [0, 127], so the tensor
//        core computes q8 . pool exactly as 128*(q8 . hi) + (q8 . lo) in int32.
//   cv  [BH, nCT*64, d] bf16 : row 2G = bf16(vbar), row 2G+1 = bf16(vbar - bf16(vbar));
//        the attention kernel weights both rows by the same probability.
//   cfac  [BH, nCT*32] fp32  : sk_j / |g|          (0 for padding groups)
//   cbias [BH, nCT*32] fp32  : log2 |g|            (-inf for empty or padding groups)
// Group G = j*c + h (c = 1 or 2 centroids per block).
#include <cmath>

#include "common.cuh"

namespace bsva {
namespace {

// Eight columns per thread (16-byte loads and stores), d/8 threads per key
// block, 256/(d/8) key blocks per CTA.
template <int D>
__global__ void __launch_bounds__(256) centroid_kernel(const int32_t* __restrict__ k_pool,
                                                       const float* __restrict__ k_scale,
                                                       const __nv_bfloat16* __restrict__ v,
                                                       int8_t* __restrict__ ck8, __nv_bfloat16* __restrict__ cv,
                                                       float* __restrict__ cfac, float* __restrict__ cbias,
                                                       int Lk, int nKB, int mode, int nCT) {
  constexpr int TPB = D / 8;                 // threads per key block
  constexpr int BPC = 256 / TPB;             // key blocks per CTA
  const int bh = blockIdx.y;
  const int slot = threadIdx.x / TPB;
  const int c8 = threadIdx.x % TPB;          // column group: columns 8*c8 .. 8*c8+7
  const int j = blockIdx.x * BPC + slot;     // key block (may be padding)
  const int nG = nCT * 32;                   // groups per head incl. padding
  if (j >= nG / mode) return;
  const size_t nCR = size_t(nCT) * 64;
  const int nj = (j < nKB) ? min(KB, Lk - j * KB) : 0;

  // V column sums over each 32-row half of the block (fp32)
  float sum[2][8];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int e = 0; e < 8; ++e) sum[h][e] = 0.f;
  if (nj > 0) {
    const uint4* vp = reinterpret_cast<const uint4*>(v + (size_t(bh) * Lk + size_t(j) * KB) * D) + c8;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int rend = min(32 * (h + 1), nj);
#pragma unroll 4
      for (int r = 32 * h; r < rend; ++r) {
        const uint4 w = __ldg(vp + size_t(r) * (D / 8));
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(b2[e]);
          sum[h][2 * e] += f.x;
          sum[h][2 * e + 1] += f.y;
        }
      }
    }
  }
  const float skj = (j < nKB) ? k_scale[size_t(bh) * nKB + j] : 0.f;
  const int32_t* kp = (j < nKB) ? k_pool + (size_t(bh) * nKB + j) * 2 * D + 8 * c8 : nullptr;

  for (int g = 0; g < mode; ++g) {
    const int G = j * mode + g;
    // group rows [g0, g1) of the block: 1x64 the whole block, 2x32 its halves
    const int g0 = (mode == 1) ? 0 : (g == 0 ? 0 : min(32, nj));
    const int g1 = (mode == 1) ? nj : (g == 0 ? min(32, nj) : nj);
    const int n = g1 - g0;
    int32_t p[8];
    float m[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      p[e] = 0;
      if (n > 0) p[e] = (mode == 1) ? kp[e] + kp[D + e] : kp[g * D + e];
      const float tot = (mode == 1) ? sum[0][e] + sum[1][e] : (g == 0 ? sum[0][e] : sum[1][e]);
      m[e] = n > 0 ? tot / (float)n : 0.f;
    }
    const size_t rhi = (size_t(bh) * nCR + 2 * size_t(G)) * D + 8 * c8;
    const size_t rlo = rhi + D;
    // key rows: pool = 128*hi + lo, hi = pool >> 7 in [-64, 63], lo = pool & 127
    uint32_t hw[2] = {0, 0}, lw[2] = {0, 0};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      hw[e >> 2] |= (uint32_t(p[e] >> 7) & 0xFF) << (8 * (e & 3));
      lw[e >> 2] |= (uint32_t(p[e] & 127) & 0xFF) << (8 * (e & 3));
    }
    *reinterpret_cast<uint2*>(ck8 + rhi) = make_uint2(hw[0], hw[1]);
    *reinterpret_cast<uint2*>(ck8 + rlo) = make_uint2(lw[0], lw[1]);
    // value rows: vbar as bf16 hi + bf16 lo
    uint32_t vh[4], vl[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(m[2 * e], m[2 * e + 1]);
      const float2 hf = __bfloat1622float2(h2);
      const __nv_bfloat162 l2 = __floats2bfloat162_rn(m[2 * e] - hf.x, m[2 * e + 1] - hf.y);
      vh[e] = *reinterpret_cast<const uint32_t*>(&h2);
      vl[e] = *reinterpret_cast<const uint32_t*>(&l2);
    }
    *reinterpret_cast<uint4*>(cv + rhi) = make_uint4(vh[0], vh[1], vh[2], vh[3]);
    *reinterpret_cast<uint4*>(cv + rlo) = make_uint4(vl[0], vl[1], vl[2], vl[3]);
    if (c8 == 0) {
      cfac[size_t(bh) * nG + G] = n > 0 ? skj / (float)n : 0.f;
      cbias[size_t(bh) * nG + G] = n > 0 ? log2f((float)n) : -INFINITY;
    }
  }
}

}  // namespace

cudaError_t launch_centroids(const bsva_shape& s, int centroid_mode, int nCT, const int32_t* k_pool,
                             const float* k_scale, const __nv_bfloat16* v, int8_t* ck8, __nv_bfloat16* cv,
                             float* cfac, float* cbias, cudaStream_t st) {
  const int nKB = (s.Lk + KB - 1) / KB;
  const int nblk_virtual = nCT * 32 / centroid_mode;
  const int bpc = 256 / (s.d / 8);
  dim3 grid((nblk_virtual + bpc - 1) / bpc, s.B * s.H);
  if (s.d == 128)
    centroid_kernel<128><<<grid, 256, 0, st>>>(k_pool, k_scale, v, ck8, cv, cfac, cbias, s.Lk, nKB,
                                               centroid_mode, nCT);
  else
    centroid_kernel<64><<<grid, 256, 0, st>>>(k_pool, k_scale, v, ck8, cv, cfac, cbias, s.Lk, nKB,
                                              centroid_mode, nCT);
  return cudaGetLastError();
}

}  // namespace bsva
