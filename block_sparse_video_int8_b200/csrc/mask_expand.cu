// mask_expand.cu -- logical 128x128 block mask -> physical kept-block lists.
//
// Method ("FlashVSR Sparge Attention", How it works): routing happens on
// logical 128-query x 128-key blocks and the mask is converted to the
// kernel's physical block geometry after routing, then the complete compact
// mask runs in one sparse call. Physical 64-key block j of query block i is
// allowed iff mask[b, h % mask_heads, i, j / 2] != 0.
//
// One warp per (b, h, query block) row; ballots compact the allowed indices
// in ascending order.
#include "common.cuh"

namespace bsva {
namespace {

__global__ void __launch_bounds__(256) mask_expand_kernel(const uint8_t* __restrict__ mask, int mask_heads, int H,
                                                          int nQB, int nKB, int nLK, int rows,
                                                          int32_t* __restrict__ kidx, int32_t* __restrict__ kcnt) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int i = row % nQB;
  const int bh = row / nQB;
  const int b = bh / H, h = bh % H;
  const uint8_t* m = mask + ((size_t(b) * mask_heads + (h % mask_heads)) * nQB + i) * nLK;
  int32_t* out = kidx + size_t(row) * nKB;
  int base = 0;
  for (int j0 = 0; j0 < nKB; j0 += 32) {
    const int j = j0 + lane;
    const bool on = j < nKB && m[j >> 1] != 0;
    const unsigned bal = __ballot_sync(0xffffffffu, on);
    if (on) out[base + __popc(bal & ((1u << lane) - 1u))] = j;
    base += __popc(bal);
  }
  if (lane == 0) kcnt[row] = base;
}

}  // namespace

cudaError_t launch_mask_expand(const bsva_shape& s, const uint8_t* block_mask, int mask_heads, int32_t* kept_idx,
                               int32_t* kept_cnt, cudaStream_t st) {
  const int nQB = (s.Lq + QB - 1) / QB, nKB = (s.Lk + KB - 1) / KB, nLK = (s.Lk + 127) / 128;
  const int rows = s.B * s.H * nQB;
  mask_expand_kernel<<<(rows + 7) / 8, 256, 0, st>>>(block_mask, mask_heads, s.H, nQB, nKB, nLK, rows, kept_idx,
                                                     kept_cnt);
  return cudaGetLastError();
}

}  // namespace bsva
