// kv_cache.cu -- the INT8 streaming K/V cache in 128-row slabs: quantising an
// appended chunk into its slabs, and the kept lists of the mask entry over the
// live slabs.
//
// Method ("FlashVSR Kitchen Sparse Attention", intro and When it bites): the
// streaming modes keep a sliding cache of past K and V as INT8, held as
// bounded 128-row slabs that the sparse kernel reads directly, with no
// full-precision rebuild. Layout (per (b, h), n_slots slabs in a ring):
//   k8, v8       [BH, n_slots * 128, d] int8
//   k_scale,
//   v_scale      [BH, n_slots * 2] fp32, one per 64-row block of a slot
//   slab_rows    [n_slots] int32, valid rows of the slab in each slot
// Logical slab x (0 = oldest live slab) sits in slot (first + x) % n_slots;
// logical key block j is 64-row block j % 2 of logical slab j / 2.
// Each 64-row block is quantised like K (s = fl32(amax / 127), codes
// rint_half_even(fl32(x / s)) clamped to [-127, 127], both IEEE divisions),
// over its valid rows.
#include "common.cuh"

namespace bsva {
namespace {

constexpr int kAppendThreads = 256;

// One CTA per (64-row block of the chunk, b*h, K or V). Writes the block's codes and scale
// into its slot; the CTA of a slab's first block also records the slab's valid rows.
template <int D>
__global__ void __launch_bounds__(kAppendThreads) kv_append_kernel(const __nv_bfloat16* __restrict__ k,
                                                                   const __nv_bfloat16* __restrict__ v, int Lc,
                                                                   int skip_slabs, int slot0, int n_slots,
                                                                   int8_t* __restrict__ k8, float* __restrict__ k_scale,
                                                                   int8_t* __restrict__ v8, float* __restrict__ v_scale,
                                                                   int32_t* __restrict__ slab_rows) {
  const int blk = blockIdx.x + 2 * skip_slabs;   // 64-row block of the chunk
  const int bh = blockIdx.y;
  const bool isV = blockIdx.z == 1;
  const int r0 = blk * KB;
  if (r0 >= Lc) return;
  const int n = min(KB, Lc - r0);
  const int slab = blk / 2;
  const int slot = (slot0 + slab - skip_slabs) % n_slots;
  const __nv_bfloat16* src = (isV ? v : k) + (size_t(bh) * Lc + r0) * D;
  int8_t* dst = (isV ? v8 : k8) + (size_t(bh) * n_slots * 128 + size_t(slot) * 128 + (blk & 1) * KB) * D;
  float* sc = (isV ? v_scale : k_scale) + size_t(bh) * n_slots * 2 + slot * 2 + (blk & 1);

  // amax over the block's valid rows
  constexpr int EPT = KB * D / kAppendThreads;   // elements per thread
  float x[EPT];
  float m = 0.f;
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    const int idx = threadIdx.x + e * kAppendThreads;   // row idx / D, column idx % D
    x[e] = (idx / D < n) ? __bfloat162float(src[idx]) : 0.f;
    m = fmaxf(m, fabsf(x[e]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float s_m[kAppendThreads / 32];
  __shared__ float s_scale;
  if ((threadIdx.x & 31) == 0) s_m[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = 0.f;
    for (int w = 0; w < kAppendThreads / 32; ++w) a = fmaxf(a, s_m[w]);
    s_scale = __fdiv_rn(a, 127.0f);
    *sc = s_scale;
    if (!isV && (blk & 1) == 0 && bh == 0) slab_rows[slot] = min(128, Lc - r0);
  }
  __syncthreads();
  const float s = s_scale;
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    const int idx = threadIdx.x + e * kAppendThreads;
    int q = 0;
    if (s > 0.f) q = max(-127, min(127, __float2int_rn(__fdiv_rn(x[e], s))));
    dst[idx] = int8_t(idx / D < n ? q : 0);
  }
}

// Kept lists of the mask entry over the cache: physical key block j of query block i (logical
// slab j / 2, its 64-row block j % 2) runs iff mask[b, h mod Hm, i, j / 2] and the block holds
// at least one valid row. One warp per (b*h, query block) row, ballot compaction.
__global__ void __launch_bounds__(256) kv_mask_expand_kernel(const uint8_t* __restrict__ mask, int mask_heads, int H,
                                                             int nQB, int count, int first, int n_slots,
                                                             const int32_t* __restrict__ slab_rows, int rows,
                                                             int32_t* __restrict__ kept_idx,
                                                             int32_t* __restrict__ kept_cnt) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int i = row % nQB;
  const int bh = row / nQB;
  const int b = bh / H, h = bh % H;
  const uint8_t* mrow = mask + ((size_t(b) * mask_heads + (h % mask_heads)) * nQB + i) * count;
  const int nKB = 2 * count;
  int base = 0;
  for (int j0 = 0; j0 < nKB; j0 += 32) {
    const int j = j0 + lane;
    bool keep = false;
    if (j < nKB) {
      const int x = j >> 1;
      const int slot = (first + x) % n_slots;
      keep = mrow[x] != 0 && slab_rows[slot] > (j & 1) * KB;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) kept_idx[size_t(row) * nKB + base + __popc(bal & ((1u << lane) - 1u))] = j;
    base += __popc(bal);
  }
  if (lane == 0) kept_cnt[row] = base;
}

}  // namespace

cudaError_t launch_kv_append(const bsva_kv_cache& c, const __nv_bfloat16* k, const __nv_bfloat16* v, int Lc,
                             int skip_slabs, int slot0, cudaStream_t st) {
  const int blocks = (Lc + KB - 1) / KB - 2 * skip_slabs;
  if (blocks <= 0) return cudaSuccess;
  const dim3 grid(blocks, unsigned(c.B) * c.H, 2);
  if (c.d == 128)
    kv_append_kernel<128><<<grid, kAppendThreads, 0, st>>>(k, v, Lc, skip_slabs, slot0, c.n_slots, c.k8, c.k_scale,
                                                           c.v8, c.v_scale, c.slab_rows);
  else
    kv_append_kernel<64><<<grid, kAppendThreads, 0, st>>>(k, v, Lc, skip_slabs, slot0, c.n_slots, c.k8, c.k_scale,
                                                          c.v8, c.v_scale, c.slab_rows);
  return cudaGetLastError();
}

cudaError_t launch_kv_mask_expand(const bsva_kv_cache& c, int nQB, const uint8_t* block_mask, int mask_heads,
                                  int32_t* kept_idx, int32_t* kept_cnt, cudaStream_t st) {
  const int rows = c.B * c.H * nQB;
  kv_mask_expand_kernel<<<(rows + 7) / 8, 256, 0, st>>>(block_mask, mask_heads, c.H, nQB, c.count, c.first,
                                                        c.n_slots, c.slab_rows, rows, kept_idx, kept_cnt);
  return cudaGetLastError();
}

}  // namespace bsva
