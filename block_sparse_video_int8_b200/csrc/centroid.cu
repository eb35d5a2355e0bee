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

// One thread per pair of columns, one "slot" of d/2 threads per key block.
template <int D>
__global__ void __launch_bounds__(256) centroid_kernel(const int32_t* __restrict__ k_pool,
                                                       const float* __restrict__ k_scale,
                                                       const __nv_bfloat16* __restrict__ v,
                                                       int8_t* __restrict__ ck8, __nv_bfloat16* __restrict__ cv,
                                                       float* __restrict__ cfac, float* __restrict__ cbias,
                                                       int Lk, int nKB, int mode, int nCT) {
  constexpr int TPB = D / 2;                 // threads per key block
  constexpr int BPC = 256 / TPB;             // key blocks per CTA
  const int bh = blockIdx.y;
  const int slot = threadIdx.x / TPB;
  const int cp = threadIdx.x % TPB;          // column pair
  const int j = blockIdx.x * BPC + slot;     // key block (may be padding)
  const int nG = nCT * 32;                   // groups per head incl. padding
  const int nblk_virtual = nG / mode;
  if (j >= nblk_virtual) return;
  const size_t nCR = size_t(nCT) * 64;

  const int nj = (j < nKB) ? min(KB, Lk - j * KB) : 0;
  // group spans (relative rows) and sizes
  int g0[2], g1[2];
  if (mode == 1) {
    g0[0] = 0; g1[0] = nj; g0[1] = 0; g1[1] = 0;
  } else {
    g0[0] = 0; g1[0] = min(32, nj); g0[1] = min(32, nj); g1[1] = nj;
  }

  // V sums over each half of the block (fp32)
  float sx[2] = {0.f, 0.f}, sy[2] = {0.f, 0.f};
  if (nj > 0) {
    const __nv_bfloat162* vp =
        reinterpret_cast<const __nv_bfloat162*>(v + (size_t(bh) * Lk + size_t(j) * KB) * D) + cp;
    for (int r = 0; r < nj; ++r) {
      const float2 f = __bfloat1622float2(vp[size_t(r) * (D / 2)]);
      const int h = (mode == 2 && r >= 32) ? 1 : 0;
      sx[h] += f.x;
      sy[h] += f.y;
    }
  }
  const float skj = (j < nKB) ? k_scale[size_t(bh) * nKB + j] : 0.f;
  const int32_t* kp = (j < nKB) ? k_pool + (size_t(bh) * nKB + j) * 2 * D : nullptr;

  for (int g = 0; g < mode; ++g) {
    const int G = j * mode + g;
    const int n = g1[g] - g0[g];
    // pool of the group
    int32_t p0 = 0, p1 = 0;
    if (n > 0) {
      if (mode == 1) {
        p0 = kp[2 * cp] + kp[D + 2 * cp];
        p1 = kp[2 * cp + 1] + kp[D + 2 * cp + 1];
      } else {
        p0 = kp[g * D + 2 * cp];
        p1 = kp[g * D + 2 * cp + 1];
      }
    }
    const size_t rhi = (size_t(bh) * nCR + 2 * size_t(G)) * D;
    const size_t rlo = rhi + D;
    // key rows: pool = 128*hi + lo
    char2 hi, lo;
    hi.x = (char)(p0 >> 7); lo.x = (char)(p0 & 127);
    hi.y = (char)(p1 >> 7); lo.y = (char)(p1 & 127);
    *reinterpret_cast<char2*>(ck8 + rhi + 2 * cp) = hi;
    *reinterpret_cast<char2*>(ck8 + rlo + 2 * cp) = lo;
    // value rows: vbar split into bf16 hi + bf16 lo
    float mx = 0.f, my = 0.f;
    if (n > 0) {
      mx = sx[g] / (float)n;
      my = sy[g] / (float)n;
    }
    const __nv_bfloat162 vh = __floats2bfloat162_rn(mx, my);
    const float2 vhf = __bfloat1622float2(vh);
    const __nv_bfloat162 vl = __floats2bfloat162_rn(mx - vhf.x, my - vhf.y);
    *reinterpret_cast<__nv_bfloat162*>(cv + rhi + 2 * cp) = vh;
    *reinterpret_cast<__nv_bfloat162*>(cv + rlo + 2 * cp) = vl;
    if (cp == 0) {
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
  const int bpc = 256 / (s.d / 2);
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
