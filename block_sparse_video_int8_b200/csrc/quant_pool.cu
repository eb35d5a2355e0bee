// quant_pool.cu -- per-block symmetric INT8 quantisation of Q and K plus their
// integer sum-pools, in one HBM pass.
//
// Method ("Configure Sol Sparse Attention", How it works): the routing proxy
// and the exact path read the same prequantized INT8 Q/K. Per block the scale
// is s = fl32(amax/127) and x8 = clamp(rint_half_even(fl32(x/s)), -127, 127),
// both divisions IEEE round-to-nearest; Q blocks hold 128 rows, K blocks 64.
//
// Design: one CTA of 256 threads owns a 128-row slab of one (b, h) of Q
// (blockIdx.z = 0, one quant block) or of K (blockIdx.z = 1, two 64-row
// blocks). Each thread loads its 16-byte chunks once into registers (a slab is
// 32 KB of bf16 at d = 128), the CTA reduces amax, then the same registers are
// quantised and written as 8-byte int8 chunks; column sums for the pools go
// through shared memory. Every byte of Q and K is read once and every INT8
// byte written once: 3 bytes of HBM traffic per element.
#include "common.cuh"

namespace bsva {
namespace {

constexpr int kThreads = 256;

template <int D>
__global__ void __launch_bounds__(kThreads) quant_pool_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, int8_t* __restrict__ q8,
    float* __restrict__ q_scale, int8_t* __restrict__ k8, float* __restrict__ k_scale,
    int32_t* __restrict__ q_pool, int32_t* __restrict__ k_pool, int Lq, int Lk) {
  constexpr int CPR = D / 8;                 // 16-byte chunks per row
  constexpr int NC = QB * CPR / kThreads;    // chunks per thread (8 for d=128)
  constexpr int RSTEP = kThreads / CPR;      // row step between a thread's chunks
  const bool isK = blockIdx.z == 1;
  const int L = isK ? Lk : Lq;
  const int slab = blockIdx.x;
  const int r0 = slab * QB;
  if (r0 >= L) return;
  const int bh = blockIdx.y;
  const int nvalid = min(QB, L - r0);
  const __nv_bfloat16* src = (isK ? k : q) + (size_t(bh) * L + r0) * D;
  int8_t* dst = (isK ? k8 : q8) + (size_t(bh) * L + r0) * D;

  const int t = threadIdx.x;
  const int col8 = t % CPR;
  const int rbase = t / CPR;

  // ---- load (16 B per chunk) and per-thread amax, per 64-row half of the slab
  uint4 v[NC];
  float amax[2] = {0.f, 0.f};
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int row = rbase + RSTEP * c;
    if (row < nvalid) {
      v[c] = __ldg(reinterpret_cast<const uint4*>(src + size_t(row) * D) + col8);
    } else {
      v[c] = make_uint4(0, 0, 0, 0);
    }
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[c]);
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __bfloat1622float2(h[e]);
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    amax[row >= 64] = fmaxf(amax[row >= 64], m);
  }

  // ---- CTA reduction of amax (two halves; Q uses their max)
  __shared__ float s_amax[2][kThreads / 32];
  __shared__ float s_scale[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float m = amax[h];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((t & 31) == 0) s_amax[h][t >> 5] = m;
  }
  __syncthreads();
  if (t < 2) {
    float m = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) m = fmaxf(m, s_amax[t][w]);
    s_amax[t][0] = m;
  }
  __syncthreads();
  if (t == 0) {
    if (isK) {
      s_scale[0] = __fdiv_rn(s_amax[0][0], 127.0f);
      s_scale[1] = __fdiv_rn(s_amax[1][0], 127.0f);
    } else {
      const float s = __fdiv_rn(fmaxf(s_amax[0][0], s_amax[1][0]), 127.0f);
      s_scale[0] = s;
      s_scale[1] = s;
    }
  }
  __syncthreads();

  // ---- quantise, store, and per-thread column sums (4 halves of 32 rows)
  int32_t part[4][8];
#pragma unroll
  for (int h = 0; h < 4; ++h)
#pragma unroll
    for (int e = 0; e < 8; ++e) part[h][e] = 0;

#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int row = rbase + RSTEP * c;
    const float s = s_scale[row >= 64];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[c]);
    int qv[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __bfloat1622float2(h[e]);
      int a = 0, b = 0;
      if (s != 0.f) {
        a = __float2int_rn(__fdiv_rn(f.x, s));
        b = __float2int_rn(__fdiv_rn(f.y, s));
        a = max(-127, min(127, a));
        b = max(-127, min(127, b));
      }
      qv[2 * e] = a;
      qv[2 * e + 1] = b;
    }
    if (row < nvalid) {
      uint32_t lo = (uint32_t(qv[0]) & 0xFF) | ((uint32_t(qv[1]) & 0xFF) << 8) | ((uint32_t(qv[2]) & 0xFF) << 16) |
                    ((uint32_t(qv[3]) & 0xFF) << 24);
      uint32_t hi = (uint32_t(qv[4]) & 0xFF) | ((uint32_t(qv[5]) & 0xFF) << 8) | ((uint32_t(qv[6]) & 0xFF) << 16) |
                    ((uint32_t(qv[7]) & 0xFF) << 24);
      *(reinterpret_cast<uint2*>(dst + size_t(row) * D) + col8) = make_uint2(lo, hi);
    }
    const int hsel = row >> 5;   // 32-row half index within the slab (0..3); rows >= nvalid hold 0
#pragma unroll
    for (int e = 0; e < 8; ++e) part[hsel][e] += qv[e];
  }

  // ---- pools: reduce the RSTEP threads sharing a column group through smem
  __shared__ int32_t s_part[4][RSTEP][D];
#pragma unroll
  for (int h = 0; h < 4; ++h)
#pragma unroll
    for (int e = 0; e < 8; ++e) s_part[h][rbase][col8 * 8 + e] = part[h][e];
  __syncthreads();

  const int nQB = (Lq + QB - 1) / QB, nKB = (Lk + KB - 1) / KB;
  for (int idx = t; idx < 4 * D; idx += kThreads) {
    const int h = idx / D, col = idx % D;
    int32_t sum = 0;
#pragma unroll 4
    for (int r = 0; r < RSTEP; ++r) sum += s_part[h][r][col];
    s_part[h][0][col] = sum;
  }
  __syncthreads();
  if (!isK) {
    for (int col = t; col < D; col += kThreads) {
      const int32_t tot = s_part[0][0][col] + s_part[1][0][col] + s_part[2][0][col] + s_part[3][0][col];
      q_pool[(size_t(bh) * nQB + slab) * D + col] = tot;
    }
    if (t == 0) q_scale[size_t(bh) * nQB + slab] = s_scale[0];
  } else {
    for (int idx = t; idx < 4 * D; idx += kThreads) {
      const int h = idx / D, col = idx % D;
      const int kb = 2 * slab + (h >> 1);
      if (kb < nKB) k_pool[((size_t(bh) * nKB + kb) * 2 + (h & 1)) * D + col] = s_part[h][0][col];
    }
    if (t < 2) {
      const int kb = 2 * slab + t;
      if (kb < nKB) k_scale[size_t(bh) * nKB + kb] = s_scale[t];
    }
  }
}

}  // namespace

cudaError_t launch_quant_pool(const bsva_shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k, int8_t* q8,
                              float* q_scale, int8_t* k8, float* k_scale, int32_t* q_pool, int32_t* k_pool,
                              cudaStream_t st) {
  const int slabs = (max(s.Lq, s.Lk) + QB - 1) / QB;
  dim3 grid(slabs, s.B * s.H, 2);
  if (s.d == 128) {
    quant_pool_kernel<128><<<grid, kThreads, 0, st>>>(q, k, q8, q_scale, k8, k_scale, q_pool, k_pool, s.Lq, s.Lk);
  } else {
    quant_pool_kernel<64><<<grid, kThreads, 0, st>>>(q, k, q8, q_scale, k8, k_scale, q_pool, k_pool, s.Lq, s.Lk);
  }
  return cudaGetLastError();
}

}  // namespace bsva
