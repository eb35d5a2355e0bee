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
#ifndef BSVA_QP_MINB
#define BSVA_QP_MINB 4   // resident CTAs per SM the register budget is sized for (4 beat 3 on B200)
#endif
constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23: q + kMagic rounds q to an integer, half to even
// Half-integer guard band. With rcp = fl(1/s) and q = fl(x * rcp), |x/s| <= 127 + 2^-16 gives
// |q - x/s| <= 127.0001 * (2^-23 + 2^-48) < 1.52e-5, and the IEEE quotient fl(x/s) lies within
// 2^-18 < 3.9e-6 of x/s, so q and fl(x/s) round to the same integer unless q is within 1.9e-5 of
// a half-integer (ties of fl(x/s) included). Chunks with such an element take the exact division.
constexpr float kBand = 0.5f - 4e-5f;

// |a| max of two bf16x2 words (sign bits of the result are meaningless and masked later).
__device__ __forceinline__ uint32_t bmax_abs(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ float bmax_fold(uint32_t m) {
  return fmaxf(__uint_as_float((m & 0x7FFFu) << 16), __uint_as_float(m & 0x7FFF0000u));
}

// Exact step for one element: code n of rint_half_even(fl32(x / s)), returned as the float
// kMagic + n (the bit pattern the fast path produces; its low byte is n as int8).
__device__ __forceinline__ float quant_exact(float x, float s) {
  const int n = (s == 0.f) ? 0 : __float2int_rn(__fdiv_rn(x, s));
  return __int_as_float(0x4B400000 + n);
}

template <int D>
__global__ void __launch_bounds__(kThreads, BSVA_QP_MINB) quant_pool_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, int8_t* __restrict__ q8,
    float* __restrict__ q_scale, int8_t* __restrict__ k8, float* __restrict__ k_scale,
    int32_t* __restrict__ q_pool, int32_t* __restrict__ k_pool, int Lq, int Lk, int z0) {
  constexpr int CPR = D / 8;                 // 16-byte chunks per row
  constexpr int NC = QB * CPR / kThreads;    // chunks per thread (8 for d=128)
  constexpr int RSTEP = kThreads / CPR;      // row step between a thread's chunks
  constexpr int CPQ = 32 / RSTEP;            // chunks per 32-row quarter
  static_assert(RSTEP <= 32 && 32 % RSTEP == 0 && NC == 4 * CPQ, "slab tiling");
  const bool isK = blockIdx.z + z0 == 1;   // z0 = 1: K part only (the INT8 V entry)
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

  // ---- load (16 B per chunk) and |x| max per 64-row half of the slab, in bf16x2
  uint4 v[NC];
  uint32_t m2[2] = {0u, 0u};
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int row = rbase + RSTEP * c;
    v[c] = (row < nvalid) ? __ldg(reinterpret_cast<const uint4*>(src + size_t(row) * D) + col8)
                          : make_uint4(0, 0, 0, 0);
    const int hh = (RSTEP * c >= 64) ? 1 : 0;
    m2[hh] = bmax_abs(bmax_abs(m2[hh], v[c].x), bmax_abs(v[c].y, bmax_abs(v[c].z, v[c].w)));
  }

  // ---- CTA reduction of amax (two halves; Q uses their max)
  __shared__ float s_amax[2][kThreads / 32];
  __shared__ float s_scale[2];
  __shared__ float s_rcp[2];
  __shared__ int s_slow[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float m = bmax_fold(m2[h]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((t & 31) == 0) s_amax[h][t >> 5] = m;
  }
  __syncthreads();
  if (t < 2) {
    float m0 = 0.f, m1 = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) {
      m0 = fmaxf(m0, s_amax[0][w]);
      m1 = fmaxf(m1, s_amax[1][w]);
    }
    const float a = isK ? (t == 0 ? m0 : m1) : fmaxf(m0, m1);
    const float sc = __fdiv_rn(a, 127.0f);
    s_scale[t] = sc;
    // s == 0 quantises to 0 on the fast path; scales below 2^-120 (1/s could overflow) go exact
    s_rcp[t] = sc >= 0x1p-120f ? __frcp_rn(sc) : 0.f;
    s_slow[t] = (sc > 0.f && sc < 0x1p-120f) ? 1 : 0;
  }
  __syncthreads();

  // ---- quantise and store; per-thread column sums per 32-row quarter go to shared memory as
  // s_red[quarter][rbase][k][col8][4] (column 8*col8 + 4*k + e): conflict-free float4 stores.
  __shared__ __align__(16) float s_red[4 * RSTEP * D];
  const float2 mg = make_float2(kMagic, kMagic);
  const float2 nmg = make_float2(-kMagic, -kMagic);
  float2 acc[4];
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int row = rbase + RSTEP * c;
    const int hh = (RSTEP * c >= 64) ? 1 : 0;   // rbase < RSTEP and 64 % RSTEP == 0
    const float sc = s_scale[hh];
    const float2 rc = make_float2(s_rcp[hh], s_rcp[hh]);
    const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
    float2 tq[4], rr[4];
    float dm = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
      const float2 qq = __fmul2_rn(x, rc);
      tq[e] = __fadd2_rn(qq, mg);
      rr[e] = __fadd2_rn(tq[e], nmg);
      const float2 dd = __fadd2_rn(qq, make_float2(-rr[e].x, -rr[e].y));   // exact
      dm = fmaxf(dm, fmaxf(fabsf(dd.x), fabsf(dd.y)));
    }
    if (dm >= kBand || s_slow[hh]) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        tq[e].x = quant_exact(__uint_as_float(w[e] << 16), sc);
        tq[e].y = quant_exact(__uint_as_float(w[e] & 0xFFFF0000u), sc);
        rr[e] = __fadd2_rn(tq[e], nmg);
      }
    }
    // |x| <= amax keeps |code| <= 127 without a clamp: fl(x/s) <= 127 + 2^-16 and q < 127.5.
    if (row < nvalid) {
      const uint32_t b01 = __byte_perm(__float_as_uint(tq[0].x), __float_as_uint(tq[0].y), 0x0040);
      const uint32_t b23 = __byte_perm(__float_as_uint(tq[1].x), __float_as_uint(tq[1].y), 0x0040);
      const uint32_t b45 = __byte_perm(__float_as_uint(tq[2].x), __float_as_uint(tq[2].y), 0x0040);
      const uint32_t b67 = __byte_perm(__float_as_uint(tq[3].x), __float_as_uint(tq[3].y), 0x0040);
      *(reinterpret_cast<uint2*>(dst + size_t(row) * D) + col8) =
          make_uint2(__byte_perm(b01, b23, 0x5410), __byte_perm(b45, b67, 0x5410));
    }
    // rows >= nvalid hold 0 and add nothing
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = (c % CPQ == 0) ? rr[e] : __fadd2_rn(acc[e], rr[e]);
    if (c % CPQ == CPQ - 1) {
      float* base = s_red + size_t((c / CPQ) * RSTEP + rbase) * D + col8 * 4;
      *reinterpret_cast<float4*>(base) = make_float4(acc[0].x, acc[0].y, acc[1].x, acc[1].y);
      *reinterpret_cast<float4*>(base + CPR * 4) = make_float4(acc[2].x, acc[2].y, acc[3].x, acc[3].y);
    }
  }
  __syncthreads();

  // ---- pools: sums over the row slots (exact: integers below 2^14 in fp32)
  const int nQB = (Lq + QB - 1) / QB, nKB = (Lk + KB - 1) / KB;
  if (!isK) {
    for (int rem = t; rem < D; rem += kThreads) {
      float tot = 0.f;
#pragma unroll 4
      for (int r = 0; r < 4 * RSTEP; ++r) tot += s_red[r * D + rem];
      const int col = 8 * ((rem / 4) % CPR) + 4 * (rem / (4 * CPR)) + (rem % 4);
      q_pool[(size_t(bh) * nQB + slab) * D + col] = __float2int_rn(tot);
    }
    if (t == 0) q_scale[size_t(bh) * nQB + slab] = s_scale[0];
  } else {
    for (int idx = t; idx < 4 * D; idx += kThreads) {
      const int hq = idx / D, rem = idx % D;
      float tot = 0.f;
#pragma unroll 4
      for (int r = 0; r < RSTEP; ++r) tot += s_red[(hq * RSTEP + r) * D + rem];
      const int col = 8 * ((rem / 4) % CPR) + 4 * (rem / (4 * CPR)) + (rem % 4);
      const int kb = 2 * slab + (hq >> 1);
      if (kb < nKB && k_pool) k_pool[((size_t(bh) * nKB + kb) * 2 + (hq & 1)) * D + col] = __float2int_rn(tot);
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
    quant_pool_kernel<128><<<grid, kThreads, 0, st>>>(q, k, q8, q_scale, k8, k_scale, q_pool, k_pool, s.Lq, s.Lk, 0);
  } else {
    quant_pool_kernel<64><<<grid, kThreads, 0, st>>>(q, k, q8, q_scale, k8, k_scale, q_pool, k_pool, s.Lq, s.Lk, 0);
  }
  return cudaGetLastError();
}

cudaError_t launch_quant_q(const bsva_shape& s, const __nv_bfloat16* q, int8_t* q8, float* q_scale, int32_t* q_pool,
                           cudaStream_t st) {
  dim3 grid((s.Lq + QB - 1) / QB, s.B * s.H, 1);
  if (s.d == 128)
    quant_pool_kernel<128><<<grid, kThreads, 0, st>>>(q, nullptr, q8, q_scale, nullptr, nullptr, q_pool, nullptr,
                                                      s.Lq, s.Lk, 0);
  else
    quant_pool_kernel<64><<<grid, kThreads, 0, st>>>(q, nullptr, q8, q_scale, nullptr, nullptr, q_pool, nullptr,
                                                     s.Lq, s.Lk, 0);
  return cudaGetLastError();
}

cudaError_t launch_quant_v(const bsva_shape& s, const __nv_bfloat16* v, int8_t* v8, float* v_scale, cudaStream_t st) {
  dim3 grid((s.Lk + QB - 1) / QB, s.B * s.H, 1);
  if (s.d == 128)
    quant_pool_kernel<128><<<grid, kThreads, 0, st>>>(nullptr, v, nullptr, nullptr, v8, v_scale, nullptr, nullptr,
                                                      s.Lq, s.Lk, 1);
  else
    quant_pool_kernel<64><<<grid, kThreads, 0, st>>>(nullptr, v, nullptr, nullptr, v8, v_scale, nullptr, nullptr,
                                                     s.Lq, s.Lk, 1);
  return cudaGetLastError();
}

}  // namespace bsva
