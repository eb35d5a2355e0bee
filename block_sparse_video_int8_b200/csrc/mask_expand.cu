// mask_expand.cu -- logical 128x128 block mask -> physical kept-block lists,
// and the kept lists and centroid-tile table of the virtual K/V mode.
//
// Method ("FlashVSR Sparge Attention", How it works): routing happens on
// logical 128-query x 128-key blocks and the mask is converted to the
// kernel's physical block geometry after routing, then the complete compact
// mask runs in one sparse call. Physical 64-key block j of query block i is
// allowed iff mask[b, h % mask_heads, i, j / 2] != 0.
//
// One warp per (b, h, query block) row; ballots compact the allowed indices
// in ascending order.
//
// lcsa_mask_kernel builds the logical mask itself from frame geometry
// ("FlashVSR Sparge Attention", intro: each query block attends only to a
// small, locally causal set of key blocks): a 128-token block belongs to the
// frame of its first token, floor(128 x / frame_tokens), and key block x_k is
// allowed for query block x_q iff f_q - window <= f_k <= f_q.
//
// Virtual K/V, residual mode ("Configure H3 Static Virtual KV", the mode
// list): the two real slices stay dense, so dense_lists_kernel writes kept
// lists holding every key block; virtual_tiles_kernel turns the logical
// source map (virtual slice l re-reads source slice src[l]) into one entry per
// centroid tile: the tile's first source group and how many of its 32 groups
// belong to the slice.
#include <algorithm>

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

__global__ void __launch_bounds__(256) lcsa_mask_kernel(uint8_t* __restrict__ mask, int nQB, int nLK, int frame_tokens,
                                                        int window, size_t total) {
  for (size_t idx = size_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < total; idx += size_t(gridDim.x) * blockDim.x) {
    const int xk = int(idx % nLK);
    const int xq = int((idx / nLK) % nQB);
    const long long fq = (128LL * xq) / frame_tokens, fk = (128LL * xk) / frame_tokens;
    mask[idx] = (fk <= fq && fq - fk <= window) ? 1 : 0;
  }
}

__global__ void __launch_bounds__(256) dense_lists_kernel(int32_t* __restrict__ kidx, int32_t* __restrict__ kcnt,
                                                          int nKB, size_t total) {
  for (size_t idx = size_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < total; idx += size_t(gridDim.x) * blockDim.x) {
    const int j = int(idx % nKB);
    kidx[idx] = j;
    if (j == 0) kcnt[idx / nKB] = nKB;
  }
}

// The map travels by value; it is read with compile-time indices only.
struct VirtualMap {
  int src[kMaxVirtualSlices];
};

__global__ void __launch_bounds__(128) virtual_tiles_kernel(VirtualMap m, int n_virtual, int gps, int2* __restrict__ vtab) {
  const int tps = (gps + 31) / 32;
#pragma unroll
  for (int l = 0; l < kMaxVirtualSlices; ++l) {
    if (l < n_virtual) {
      for (int lt = threadIdx.x; lt < tps; lt += blockDim.x)
        vtab[l * tps + lt] = make_int2(m.src[l] * gps + 32 * lt, min(32, gps - 32 * lt));
    }
  }
}

}  // namespace

cudaError_t launch_dense_lists(const bsva_shape& s, int32_t* kept_idx, int32_t* kept_cnt, cudaStream_t st) {
  const int nQB = (s.Lq + QB - 1) / QB, nKB = (s.Lk + KB - 1) / KB;
  const size_t total = size_t(s.B) * s.H * nQB * nKB;
  const unsigned grid = unsigned(std::min<size_t>((total + 255) / 256, 148 * 16));
  dense_lists_kernel<<<grid, 256, 0, st>>>(kept_idx, kept_cnt, nKB, total);
  return cudaGetLastError();
}

cudaError_t launch_virtual_tiles(const int* src_map, int n_virtual, int groups_per_slice, int2* vtab,
                                 cudaStream_t st) {
  VirtualMap m{};
  for (int l = 0; l < n_virtual && l < kMaxVirtualSlices; ++l) m.src[l] = src_map[l];
  virtual_tiles_kernel<<<1, 128, 0, st>>>(m, n_virtual, groups_per_slice, vtab);
  return cudaGetLastError();
}

cudaError_t launch_lcsa_mask(int Lq, int Lk, int frame_tokens, int window, int batch, uint8_t* mask,
                             cudaStream_t st) {
  const int nQB = (Lq + QB - 1) / QB, nLK = (Lk + 127) / 128;
  const size_t total = size_t(batch) * nQB * nLK;
  const unsigned grid = unsigned(std::min<size_t>((total + 255) / 256, 148 * 16));
  lcsa_mask_kernel<<<grid, 256, 0, st>>>(mask, nQB, nLK, frame_tokens, window, total);
  return cudaGetLastError();
}

cudaError_t launch_mask_expand(const bsva_shape& s, const uint8_t* block_mask, int mask_heads, int32_t* kept_idx,
                               int32_t* kept_cnt, cudaStream_t st) {
  const int nQB = (s.Lq + QB - 1) / QB, nKB = (s.Lk + KB - 1) / KB, nLK = (s.Lk + 127) / 128;
  const int rows = s.B * s.H * nQB;
  mask_expand_kernel<<<(rows + 7) / 8, 256, 0, st>>>(block_mask, mask_heads, s.H, nQB, nKB, nLK, rows, kept_idx,
                                                     kept_cnt);
  return cudaGetLastError();
}

}  // namespace bsva
