// attn_sm100.cu -- block-sparse INT8 attention with centroid terms, sm_100a.
//
// Method ("Configure Sol Sparse Attention", How it works): for each 128-token
// query block, FlashAttention-style online softmax runs over the kept 64-token
// key blocks only; every skipped block still adds its centroid term(s) in the
// same softmax. The mask entry ("FlashVSR Sparge Attention", How it works)
// runs the same loop over the allowed physical blocks with no centroids.
//
// One CTA = one (b, h, query block) work item, 192 threads:
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r). Reads S from
//              TMEM, scales, online max/sum, writes P (bf16) back to TMEM,
//              rescales O in TMEM when the running max grows by more than
//              2^8, and runs the epilogue O / l. The weights are computed
//              against the running max first; the tile max is taken only
//              when some row's weights sum to more than 2^8.
//   warp 4     TMA producer: Q tile once, then K (int8) tiles with their
//              per-tile metadata into a 4-stage ring (freed by the softmax
//              warps once they are done with the tile), first the kept
//              blocks, starting at the query block's own keys and wrapping
//              round, then the centroid tiles.
//   warp 5     TMEM owner (alloc/dealloc) and MMA issuer (the warp runs the
//              schedule, one elected lane issues); it also loads the V
//              (bf16) tiles into a 3-stage ring, two tiles ahead of PV, as
//              soon as a stage's last PV has landed, so that K and V loads
//              (about 1.5 us each here) never wait for one another:
//              S = Q8 . K8^T with tcgen05.mma kind::i8 (M=128, N=64, int32
//              accumulate) and O += P . V with kind::f16 (A = P from TMEM,
//              B = V from shared memory, fp32 accumulate). S is double
//              buffered so QK of tile n+1 overlaps the softmax of tile n.
// INT8 V (mask entry; "FlashVSR Kitchen Sparse Attention", intro: the
// streaming cache keeps K/V as INT8 and the kernel eats it without rebuilding
// bf16 tensors; the kV8 instantiation): the V tile lands in the upper half of
// its stage and the MMA warp widens it in place to f16 integers (exact,
// |v8| <= 127) before its PV, which then runs as f16 x f16 with P packed as
// f16; the block scale s_j is folded into the exponent, P' = 2^(y + log2 s_j),
// and the row sums take the rounded P' times 2^-log2 s_j, so numerator and
// denominator weight each key alike.
// The same instantiation reads the INT8 streaming cache: key block j of the
// cache is 64-row block j mod 2 of the slab in ring slot (first + j / 2) mod
// n_slots (a.slab_rows non-null).
// Centroid tiles hold 32 groups as (hi, lo) INT8 row pairs (pool = 128 hi + lo)
// so their dot with q8 is exact in int32; the value rows are (bf16 hi, bf16 lo)
// and share one probability.
// Virtual K/V, residual mode ("Configure H3 Static Virtual KV", the mode
// list): the kept lists hold every physical block, and the centroid tiles are
// those of the added virtual slices, each re-reading its source slice's groups
// through a per-tile table (a.vtab) instead of a skipped-block mask.
// Every wait is bounded: on a timeout the CTA records it in the workspace
// status word, all roles leave their loops, TMEM is freed and the CTA exits.
#include <cmath>

#include "common.cuh"

namespace bsva {
namespace {

constexpr int NK = 4;           // K tile + metadata stages (freed once the softmax is done with the tile)
constexpr int NV = 3;           // V tile stages (freed once PV is done)
constexpr int NR = 8;           // V row slots passed from the producer to the V loads
constexpr int kThreads = 192;
constexpr float kRescaleLog2 = 8.0f;   // lazy O rescale threshold (factor 256)
constexpr uint32_t kTmemCols = 256;

// Per-stage tile description, written by the producer warp before it arms
// the K stage's barrier and read by the softmax warps after QK of that tile.
struct TileMeta {
  float fac[32];    // centroid tiles: logit factor per group (sq*scale*log2e*sk/|g|)
  float bias[32];   // centroid tiles: log2|g|, or -inf (kept block / no group)
  float f;          // kept tiles: sq*sk*scale*log2e
  int nvalid;       // kept tiles: valid key columns (64 except a tail block)
  int centroid;     // 1 = centroid tile
  float vlog2;      // INT8 V: log2 of the V block scale (0 for a zero block); unused for bf16 V
};

template <int D>
struct __align__(1024) Smem {
  int8_t q[QB * D];
  int8_t k[NK][KB * D];
  __nv_bfloat16 v[NV][KB * D];
  TileMeta meta[NK];
  int vrow[NR];         // first V row of tile t at [t % NR], written before K(t)'s barrier is armed
  uint64_t q_full;
  uint64_t k_full[NK];
  uint64_t k_empty[NK];
  uint64_t v_full[NV];
  uint64_t v_empty[NV];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float y;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Physical 64-row block of logical key block j: itself, or in the INT8 streaming cache the
// block of the slab in ring slot (first + j / 2) mod n_slots.
__device__ __forceinline__ int phys_block(const AttnArgs& a, int j) {
  if (a.slab_rows == nullptr) return j;
  return ((a.ring_first + (j >> 1)) % a.ring_slots) * 2 + (j & 1);
}

// kV8: V is INT8 with per-block scales (a.v_scale), P and V enter PV as f16.
// kVirt: the centroid tiles are the virtual slices' (a.vtab), not the skipped blocks'.
template <int D, bool kV8, bool kVirt>
__global__ void __launch_bounds__(kThreads, 2)
    attn_kernel(const AttnArgs a, const __grid_constant__ AttnMaps maps) {
  extern __shared__ unsigned char smem_raw[];
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int item = int(blockIdx.x);
  const int bh = item / a.nQB;
  const int i = item % a.nQB;
  const size_t row_item = size_t(bh) * a.nQB + i;

  // a kept count comes from the caller's route: checked in BSVA_DEVICE_CHECKS builds
  const int n_exact_in = a.kept_cnt[row_item];
  const int n_exact = dcheck(n_exact_in >= 0 && n_exact_in <= a.nKB, a.status) ? n_exact_in
                      : n_exact_in < 0                                     ? 0
                                                                           : a.nKB;
  // Sol: the whole centroid table once some block is skipped; virtual K/V: the virtual slices' tiles
  const int n_cent = kVirt ? a.n_vtiles : (a.centroid_mode > 0 && n_exact < a.nKB) ? a.nCT : 0;
  const int N = n_exact + n_cent;
  const int q0 = i * QB;

  if (N == 0) {   // nothing to attend: o = 0, lse = -inf
    if (tid < QB && q0 + tid < a.Lq) {
      const size_t orow = (size_t(bh) * a.Lq + q0 + tid) * D;
      uint4* o = a.out_f32 ? reinterpret_cast<uint4*>(a.out_f32 + orow) : reinterpret_cast<uint4*>(a.out + orow);
      const int n16 = a.out_f32 ? D / 4 : D / 8;
      for (int c = 0; c < n16; ++c) o[c] = make_uint4(0, 0, 0, 0);
      if (a.lse) a.lse[size_t(bh) * a.Lq + q0 + tid] = -INFINITY;
    }
    return;
  }

  constexpr uint32_t O_COL = 0;
  constexpr uint32_t S_COL0 = D, S_COL1 = D + 64;

  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < NK; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 4);   // released by the 4 softmax warps
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.p_full[b], QB);
    }
    mbar_init(&sm.o_full, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;
  const uint64_t lim = a.wait_limit_ns;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    // K tiles (and metadata) as soon as their stage is free. Kept indices and
    // their scales are fetched 32 tiles at a time, one per lane; centroid
    // metadata is fetched a tile ahead, one group per lane. Lane 0 issues TMA.
    const float sqs = a.q_scale[row_item] * a.scale_log2e;
    const int scale_stride = a.slab_rows ? 2 * a.ring_slots : a.nKB;   // per-head count of K/V block scales
    const int32_t* kidx = a.kept_idx + row_item * a.nKB;
    const uint8_t* kmask = a.kept_mask ? a.kept_mask + row_item * a.nKB : nullptr;
    const float* cfac = a.cfac ? a.cfac + size_t(bh) * a.nCT * 32 : nullptr;
    const float* cbias = a.cbias ? a.cbias + size_t(bh) * a.nCT * 32 : nullptr;
    if (lane == 0) {
      tma_prefetch_desc(&maps.q8);
      tma_prefetch_desc(&maps.k8);
      tma_prefetch_desc(&maps.v);
      mbar_arrive_expect_tx(&sm.q_full, QB * D);
      tma_load_3d(sm.q, &maps.q8, 0, q0, bh, &sm.q_full);
    }
    // The kept tiles run from the first kept block at or after the query block's own keys (the
    // key block at the middle of its rows, the ends of the two sequences aligned), wrapping round:
    // the largest logits of a row then come first, so the running max seldom has to grow later.
    int rot = 0;
    if (n_exact > 1) {
      const int jstar = min(max((q0 + QB / 2 + a.Lk - a.Lq) / KB, 0), a.nKB - 1);
      // count the kept indices below jstar (the list ascends): narrow with 32 probes per round
      int lo = 0, len = n_exact;   // every index before lo is below jstar; the count is in [lo, lo + len]
      while (len > 32) {
        const int step = (len + 31) / 32;
        const int x = lo + lane * step;
        const bool below = x < lo + len && kidx[x] < jstar;
        const int c = __popc(__ballot_sync(0xffffffffu, below));
        if (c == 0) {
          len = 0;
        } else {
          const int nlo = lo + (c - 1) * step + 1;
          len = min(step - 1, lo + len - nlo);
          lo = nlo;
        }
      }
      const bool below = lane < len && kidx[lo + lane] < jstar;
      rot = lo + __popc(__ballot_sync(0xffffffffu, below));
      if (rot >= n_exact) rot = n_exact - 1;
    }
    int chunk_j = 0;          // kept index of tile (32*c + lane) of the current chunk
    float chunk_f = 0.f;
    int j_next = 0;              // key block of the K step's tile
    float cf_next = 0.f, cb_next = 0.f;   // centroid metadata of the next centroid tile
    int cr_next = 0;                      // and its first table row
    bool ok = true;

    // group metadata of centroid tile t for this lane, and the tile's first table row
    auto cent_meta = [&](int t, float& fac, float& bias, int& row) {
      if constexpr (kVirt) {   // virtual slice: 32 source groups from e.x, the first e.y of them live
        int2 e = a.vtab[t];
        if (!dcheck(e.x >= 0 && e.x <= (a.nCT - 1) * 32 && e.y >= 0 && e.y <= 32, a.status)) e = make_int2(0, 0);
        const bool live = lane < e.y;
        const int G = e.x + (live ? lane : 0);   // dead lanes re-read a live entry, never past the table
        fac = sqs * cfac[G];
        bias = live ? cbias[G] : -INFINITY;
        row = 2 * e.x;
      } else {        // Sol: groups 32t .. 32t+31, live where their block was skipped
        const int G = t * 32 + lane;
        const int jb = G / a.centroid_mode;
        const bool kept = jb >= a.nKB || kmask[jb];
        fac = sqs * cfac[G];
        bias = kept ? -INFINITY : cbias[G];
        row = t * KB;
      }
    };
    auto k_step = [&](int t) -> bool {
      const int sk = t % NK;
      if (t >= NK && !__all_sync(0xffffffffu, mbar_wait(&sm.k_empty[sk], ((t / NK) - 1) & 1, abort, a.status, lim)))
        return false;
      TileMeta& mt = sm.meta[sk];
      int row;
      if (t < n_exact) {
        if ((t & 31) == 0) {
          const int nn = t + lane;
          const int pos = nn + rot < n_exact ? nn + rot : nn + rot - n_exact;
          int jk = nn < n_exact ? kidx[pos] : 0;
          if (!dcheck(jk >= 0 && jk < a.nKB, a.status)) jk = 0;   // a kept block of the caller's list
          chunk_j = phys_block(a, jk);
          chunk_f = nn < n_exact ? sqs * a.k_scale[size_t(bh) * scale_stride + chunk_j] : 0.f;
        }
        j_next = __shfl_sync(0xffffffffu, chunk_j, t & 31);
        const float f_next = __shfl_sync(0xffffffffu, chunk_f, t & 31);
        row = j_next * KB;
        if (lane == 0) {
          mt.f = f_next;
          mt.nvalid = a.slab_rows ? min(KB, a.slab_rows[j_next >> 1] - (j_next & 1) * KB) : min(KB, a.Lk - row);
          mt.centroid = 0;
          if constexpr (kV8) {
            const float sv = a.v_scale[size_t(bh) * scale_stride + j_next];
            mt.vlog2 = sv > 0.f ? __log2f(sv) : 0.f;
          }
        }
      } else {
        const int tc = t - n_exact;
        float fac, bias;
        if (tc == 0) cent_meta(0, fac, bias, row);
        else { fac = cf_next; bias = cb_next; row = cr_next; }
        if constexpr (!kVirt) row = tc * KB;   // Sol: the table in order
        mt.fac[lane] = fac;
        mt.bias[lane] = bias;
        if (lane == 0) mt.centroid = 1;
        if (t + 1 < N) cent_meta(tc + 1, cf_next, cb_next, cr_next);   // prefetch the next centroid tile
      }
      if (lane == 0) sm.vrow[t % NR] = row;
      __syncwarp();   // the metadata is published by lane 0's arrive on the stage's barrier
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.k_full[sk], KB * D);
        tma_load_3d(sm.k[sk], t < n_exact ? &maps.k8 : &maps.ck8, 0, row, bh, &sm.k_full[sk]);
      }
      return true;
    };
    for (int t = 0; ok && t < N; ++t) ok = k_step(t);
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    // K-major INT8 tiles: rows of D bytes, 8-row groups of 8*D bytes.
    constexpr uint32_t kLayoutQK = (D == 128) ? 2u : 4u;   // 128B / 64B swizzle
    constexpr uint32_t kSboQK = 8 * D;
    // V tiles, MN-major bf16: 128-byte rows (64 d-values), 8-row groups of
    // 1 KB, the two 64-column halves (D = 128) 8 KB apart.
    constexpr uint32_t kLboV = KB * 128, kSboV = 1024;
    constexpr uint32_t IDESC_QK = make_idesc(2, 1, 1, false, false, 128, 64);
    constexpr uint32_t kFmtPV = kV8 ? 0u : 1u;   // f16 (INT8 V widened) or bf16
    constexpr uint32_t IDESC_PV = make_idesc(1, kFmtPV, kFmtPV, false, true, 128, D);
    constexpr uint32_t kStrideK = (KB * D) >> 4, kStrideV = (KB * D * 2) >> 4;   // stage strides, 16 B units
    const uint64_t dq = make_sdesc(smem_u32(sm.q), 16, kSboQK, kLayoutQK);
    const uint64_t dk0 = make_sdesc(smem_u32(sm.k[0]), 16, kSboQK, kLayoutQK);
    const uint64_t dv0 = make_sdesc(smem_u32(sm.v[0]), kLboV, kSboV, 2u);
    // The whole warp runs the schedule (all values warp-uniform); one elected
    // lane issues each group of MMAs and its commit (whole-warp issue with
    // elect.sync measured faster than a single issuing thread).
    // QK(n) into S buffer n&1: int8, K = 32 per MMA.
    auto do_qk = [&](int n) {
      const int sk = n % NK;
      const uint64_t dk = dk0 + uint64_t(sk * kStrideK);
      const uint32_t dS = tmem + ((n & 1) ? S_COL1 : S_COL0);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          mma_i8_ss(dS, dq + 2 * kk, dk + 2 * kk, IDESC_QK, kk > 0 ? 1u : 0u);
        tc_commit(&sm.s_full[n & 1]);
      }
      __syncwarp();
    };
    // PV(n): O += P(n) . V(n), A = P from TMEM (aliases S buffer n&1), K = 16 per MMA.
    auto do_pv = [&](int n) {
      const int sv = n % NV;
      const uint64_t dv = dv0 + uint64_t(sv * kStrideV);
      const uint32_t aP = tmem + ((n & 1) ? S_COL1 : S_COL0);
      const uint32_t acc0 = n > 0 ? 1u : 0u;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < KB / 16; ++kk)
          mma_bf16_ts(tmem + O_COL, aP + 8 * kk, dv + (16 * 128 / 16) * kk, IDESC_PV, kk > 0 ? 1u : acc0);
        tc_commit(&sm.v_empty[sv]);   // also tells the softmax warps that PV(n) has landed
      }
      __syncwarp();
    };
    auto wait = [&](uint64_t* bar, uint32_t par) { return __all_sync(0xffffffffu, mbar_wait(bar, par, abort, a.status, lim)); };
    // V(t) into stage t % NV once PV(t - NV) has landed; its row was published
    // with K(t)'s barrier, which this warp has already waited on.
    auto v_load = [&](int t, bool stage_free) -> bool {
      const int sv = t % NV;
      if (t >= NV && !stage_free && !wait(&sm.v_empty[sv], ((t / NV) - 1) & 1)) return false;
      if (lane == 0) {
        const int row = sm.vrow[t % NR];
        if constexpr (kV8) {
          // INT8 rows of D bytes into the upper half of the stage; widened before its PV
          mbar_arrive_expect_tx(&sm.v_full[sv], KB * D);
          tma_load_3d(reinterpret_cast<unsigned char*>(sm.v[sv]) + KB * D, &maps.v, 0, row, bh, &sm.v_full[sv]);
        } else {
          const CUtensorMap* mv = t < n_exact ? &maps.v : &maps.cv;
          mbar_arrive_expect_tx(&sm.v_full[sv], KB * D * 2);
          tma_load_3d(sm.v[sv], mv, 0, row, bh, &sm.v_full[sv]);
          if (D == 128) tma_load_3d(sm.v[sv] + KB * 64, mv, 64, row, bh, &sm.v_full[sv]);
        }
      }
      __syncwarp();
      return true;
    };
    // INT8 V: widen tile t in place to the f16 layout PV reads (MN-major rows of 64 values,
    // 128 bytes, 128-byte swizzle; the two 64-column halves 8 KB apart). Every INT8 byte is
    // read into registers before the first store, since the f16 tile overwrites them.
    // x in [-127, 127] -> f16 bits 0x6400 | (x + 128) = 1024 + x + 128, minus 1152: exact.
    auto v_widen = [&](int t) -> bool {
      const int sv = t % NV;
      if (!wait(&sm.v_full[sv], (t / NV) & 1)) return false;
      unsigned char* stage = reinterpret_cast<unsigned char*>(sm.v[sv]);
      const unsigned char* src = stage + KB * D;
      constexpr int CPR = D / 16;              // 16-byte INT8 chunks per row
      constexpr int NCH = KB * CPR / 32;       // chunks per lane
      uint4 in[NCH];
#pragma unroll
      for (int i = 0; i < NCH; ++i) in[i] = *reinterpret_cast<const uint4*>(src + (lane + 32 * i) * 16);
      __syncwarp();
      const __half2 k1152 = __floats2half2_rn(1152.f, 1152.f);
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        const int q = lane + 32 * i;
        const int r = q / CPR, c16 = q % CPR;   // key row; INT8 columns 16*c16 .. 16*c16+15
        const int j0 = (2 * c16) % 8;           // first 16-byte f16 chunk in the half's row
        unsigned char* rowp = stage + ((16 * c16) / 64) * (KB * 128) + r * 128;
        const uint32_t w[4] = {in[i].x ^ 0x80808080u, in[i].y ^ 0x80808080u, in[i].z ^ 0x80808080u,
                               in[i].w ^ 0x80808080u};
        uint32_t o[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint32_t lo = __byte_perm(w[e], 0x64646464u, 0x5140), hi = __byte_perm(w[e], 0x64646464u, 0x5342);
          __half2 hl = __hsub2(*reinterpret_cast<__half2*>(&lo), k1152);
          __half2 hh = __hsub2(*reinterpret_cast<__half2*>(&hi), k1152);
          o[2 * e] = *reinterpret_cast<uint32_t*>(&hl);
          o[2 * e + 1] = *reinterpret_cast<uint32_t*>(&hh);
        }
        *reinterpret_cast<uint4*>(rowp + ((j0 ^ (r & 7)) * 16)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(rowp + (((j0 + 1) ^ (r & 7)) * 16)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
      fence_proxy_async_smem();   // the tensor core reads the widened tile
      __syncwarp();
      return true;
    };
    bool ok = wait(&sm.q_full, 0);
    tc_fence_after();
    // Blocking waits in the order events occur: QK(0), QK(1), then PV(n)
    // (frees S buffer n&1) followed by QK(n+2). This order measured faster
    // than an event loop polling both queues.
    for (int n = 0; ok && n < 2 && n < N; ++n) {
      ok = wait(&sm.k_full[n % NK], (n / NK) & 1);
      if (ok) { tc_fence_after(); do_qk(n); }
      if (ok) ok = v_load(n, true);
    }
    if constexpr (kV8) {
      if (ok) ok = v_widen(0);
    }
    for (int n = 0; ok && n < N; ++n) {
      // The barriers of this step that are usually complete already are tested
      // together, so their round trips overlap instead of adding up.
      const bool v_in = mbar_test_wait(&sm.v_full[n % NV], (n / NV) & 1);
      const bool k_in = n + 2 >= N || mbar_test_wait(&sm.k_full[(n + 2) % NK], ((n + 2) / NK) & 1);
      const bool e_in = n + 2 >= N || n + 2 < NV ||
                        mbar_test_wait(&sm.v_empty[(n + 2) % NV], (((n + 2) / NV) - 1) & 1);
      ok = wait(&sm.p_full[n & 1], (n >> 1) & 1) &&
           (__all_sync(0xffffffffu, v_in) || wait(&sm.v_full[n % NV], (n / NV) & 1));
      if (!ok) break;
      tc_fence_after();
      do_pv(n);
      if (n + 2 < N) {
        ok = __all_sync(0xffffffffu, k_in) || wait(&sm.k_full[(n + 2) % NK], ((n + 2) / NK) & 1);
        // no second fence: the one after the p_full wait above already orders this
        // QK's S writes after the softmax warps' loads of that buffer, and the K
        // tile arrives by TMA under its own barrier
        if (ok) do_qk(n + 2);
        if (ok) ok = v_load(n + 2, __all_sync(0xffffffffu, e_in));   // needs PV(n - 1), issued one step ago
      }
      if constexpr (kV8) {
        if (ok && n + 1 < N) ok = v_widen(n + 1);   // while the softmax works on tile n + 1
      }
    }
    if (elect_one()) tc_commit(&sm.o_full);
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax
    const int r = tid;                                   // row within the block
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const bool want_lse = a.lse != nullptr;
    float m_ref = -INFINITY, l = 0.f, le = 0.f;
    bool alive = true;
    int n_cur = 0;
    // O *= alpha in TMEM once the PV product of the previous tile has landed.
    auto rescale_o = [&](float alpha) -> bool {
      // PV of the previous tile has landed once it released its V stage
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.v_empty[(n_cur - 1) % NV], ((n_cur - 1) / NV) & 1, abort,
                                             a.status, lim)))
        return false;
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + O_COL + c0, o);
        tmem_wait_ld(o);
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
        tmem_st32(tmem + lane_base + O_COL + c0, o);
      }
      tmem_wait_st();
      return true;
    };

    for (int n = 0; n < N; ++n) {
      n_cur = n;
      const int sk = n % NK;
      // the tile's metadata is published with its K stage's barrier (long complete once S
      // is in); testing it first overlaps the two round trips
      const bool meta_in = mbar_test_wait(&sm.k_full[sk], (n / NK) & 1);
      bool ok = mbar_wait(&sm.s_full[n & 1], (n >> 1) & 1, abort, a.status, lim);
      ok = ok && (meta_in || mbar_wait(&sm.k_full[sk], (n / NK) & 1, abort, a.status, lim));
      if (!__all_sync(0xffffffffu, ok)) {
        alive = false;
        break;
      }
      tc_fence_after();
      const TileMeta& mt = sm.meta[sk];
      const bool cent = mt.centroid != 0;
      const uint32_t sc = (n & 1) ? S_COL1 : S_COL0;
      uint32_t pk[32];
      float lsum = 0.f, esum = 0.f;

      if (!cent) {
        // ---- kept tile: logits x = S * f (log2 units), 64 keys per row.
        // f = 0 (an all-zero Q or K block) would turn a masked -inf into NaN;
        // 1e-30 keeps every valid logit within 1e-23 of 0 and masked ones at -inf.
        const float f = fmaxf(mt.f, 1e-30f);
        const int nvalid = mt.nvalid;
        float xs[64];
        uint32_t sa[32], sb[32];
        tmem_ld32(tmem + lane_base + sc, sa);
        tmem_wait_ld(sa);
        tmem_ld32(tmem + lane_base + sc + 32, sb);    // in flight while the first half converts
#pragma unroll
        for (int c = 0; c < 32; ++c) xs[c] = float(int(sa[c]));
        tmem_wait_ld(sb);
#pragma unroll
        for (int c = 0; c < 32; ++c) xs[32 + c] = float(int(sb[c]));
        if (nvalid < KB) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= nvalid) xs[c] = -INFINITY;
        }
        // P = 2^(x*f - m) as bf16 pairs; lsum adds the fp32 weights before rounding (the
        // bf16 rounding of each weight, at most 2^-9 relative and unbiased, stays in the
        // numerator only), and the log-sum-exp uses the same sum.
        // INT8 V: the weights carry the V block scale, P' = 2^(y + log2 s_j), and lsum takes the
        // f16-rounded P' * 2^-(log2 s_j) (esum the unrounded weights, log-sum-exp only).
        const float vlog2 = kV8 ? mt.vlog2 : 0.f;
        const float vinv = kV8 ? ex2(-vlog2) : 1.f;
        auto exps = [&](float m_use) {
          const float2 f2 = make_float2(f, f);
          const float nm = kV8 ? vlog2 - m_use : -m_use;
          const float2 nm2 = make_float2(nm, nm);
          float2 la = make_float2(0.f, 0.f), ea = make_float2(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float2 y = __ffma2_rn(make_float2(xs[2 * c], xs[2 * c + 1]), f2, nm2);
            const float p0 = ex2(y.x), p1 = ex2(y.y);
            if constexpr (kV8) {
              pk[c] = pack_f16x2(p0, p1);
              const __half2 h = *reinterpret_cast<const __half2*>(&pk[c]);
              la = __fadd2_rn(la, __half22float2(h));
              if (want_lse) ea = __fadd2_rn(ea, make_float2(p0, p1));
            } else {
              pk[c] = pack_bf16x2(p0, p1);
              la = __fadd2_rn(la, make_float2(p0, p1));
            }
          }
          lsum = la.x + la.y;
          esum = kV8 ? ea.x + ea.y : lsum;
          if constexpr (kV8) {
            lsum *= vinv;
            esum *= vinv;
          }
        };
        // Speculate that the running max still holds (it nearly always does
        // after the first tiles), so the exps need not wait for this tile's max.
        // The tile max is needed only where some weight may exceed 2^8 (a logit
        // above m_ref + 8): a row whose weights sum to at most 2^8 has none.
        const bool first = __all_sync(0xffffffffu, m_ref == -INFINITY);
        bool check = first;
        if (!first) {
          exps(m_ref);
          check = __any_sync(0xffffffffu, !(lsum <= 256.f));
        }
        if (check) {
          float m8[22];
#pragma unroll
          for (int c = 0; c < 21; ++c) m8[c] = fmax3(xs[3 * c], xs[3 * c + 1], xs[3 * c + 2]);
          m8[21] = xs[63];
#pragma unroll
          for (int c = 0; c < 7; ++c) m8[c] = fmax3(m8[3 * c], m8[3 * c + 1], m8[3 * c + 2]);
          m8[0] = fmax3(m8[0], m8[1], m8[2]);
          m8[1] = fmax3(m8[3], m8[4], m8[5]);
          m8[2] = fmax3(m8[6], m8[21], m8[0]);
          const float mt_max = fmaxf(m8[1], m8[2]) * f;   // f > 0: the max commutes with the scale
          const bool need = mt_max > m_ref + kRescaleLog2;
          if (first || __any_sync(0xffffffffu, need)) {
            const float m_new = need ? mt_max : m_ref;
            const float alpha = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - m_new);
            if (n > 0 && !rescale_o(alpha)) {
              alive = false;
              break;
            }
            l *= alpha;
            le *= alpha;
            m_ref = m_new;
            exps(m_ref == -INFINITY ? 0.f : m_ref);
          }
        }
      } else {
        // ---- centroid tile: 32 groups, each an exact int dot from its (hi, lo) rows
        uint32_t sa[32], sb[32];
        tmem_ld32(tmem + lane_base + sc, sa);
        tmem_wait_ld(sa);
        tmem_ld32(tmem + lane_base + sc + 32, sb);
        float xs[32];
#pragma unroll
        for (int g = 0; g < 16; ++g) {
          const int dot = 128 * int(sa[2 * g]) + int(sa[2 * g + 1]);
          xs[g] = fmaf(float(dot), mt.fac[g], mt.bias[g]);   // bias -inf masks the group
        }
        tmem_wait_ld(sb);
#pragma unroll
        for (int g = 0; g < 16; ++g) {
          const int dot = 128 * int(sb[2 * g]) + int(sb[2 * g + 1]);
          xs[16 + g] = fmaf(float(dot), mt.fac[16 + g], mt.bias[16 + g]);
        }
        auto cexps = [&](float m_use) {
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int g = 0; g < 32; g += 2) {
            const float p0 = ex2(xs[g] - m_use), p1 = ex2(xs[g + 1] - m_use);
            pk[g] = pack_bf16x2(p0, p0);
            pk[g + 1] = pack_bf16x2(p1, p1);
            s0 += p0;
            s1 += p1;
          }
          lsum = s0 + s1;
        };
        // as for kept tiles: speculate on the running max, take the tile max only where the
        // weights of some row sum to more than 2^8
        const bool first = __all_sync(0xffffffffu, m_ref == -INFINITY);
        bool check = first;
        if (!first) {
          cexps(m_ref);
          check = __any_sync(0xffffffffu, !(lsum <= 256.f));
        }
        if (check) {
          float m8[11];
#pragma unroll
          for (int c = 0; c < 10; ++c) m8[c] = fmax3(xs[3 * c], xs[3 * c + 1], xs[3 * c + 2]);
          m8[10] = fmaxf(xs[30], xs[31]);
          m8[0] = fmax3(m8[0], m8[1], m8[2]);
          m8[1] = fmax3(m8[3], m8[4], m8[5]);
          m8[2] = fmax3(m8[6], m8[7], m8[8]);
          const float mt_max = fmax3(fmax3(m8[0], m8[1], m8[2]), m8[9], m8[10]);
          const bool need = mt_max > m_ref + kRescaleLog2;
          const bool any_need = __any_sync(0xffffffffu, need);
          if (any_need) {
            const float m_new = need ? mt_max : m_ref;
            const float alpha = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - m_new);
            if (n > 0 && !rescale_o(alpha)) {
              alive = false;
              break;
            }
            l *= alpha;
            le *= alpha;
            m_ref = m_new;
          }
          if (first || any_need) cexps(m_ref == -INFINITY ? 0.f : m_ref);
        }
        esum = lsum;
      }
      l += lsum;
      le += esum;
      tmem_st32(tmem + lane_base + sc, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[n & 1]);
      if (lane == 0) mbar_arrive(&sm.k_empty[sk]);   // done with the tile's K stage and metadata
    }

    // ------------------------------------------------------------ epilogue
    if (alive && __all_sync(0xffffffffu, mbar_wait(&sm.o_full, 0, abort, a.status, lim))) {
      tc_fence_after();
      const int qr = q0 + r;
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      const size_t orow = (size_t(bh) * a.Lq + qr) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + O_COL + c0, o);
        tmem_wait_ld();
        if (qr < a.Lq) {
          if (a.out_f32) {
            float4* dst = reinterpret_cast<float4*>(a.out_f32 + orow + c0);
#pragma unroll
            for (int c = 0; c < 8; ++c)
              dst[c] = make_float4(__uint_as_float(o[4 * c]) * inv_l, __uint_as_float(o[4 * c + 1]) * inv_l,
                                   __uint_as_float(o[4 * c + 2]) * inv_l, __uint_as_float(o[4 * c + 3]) * inv_l);
          } else {
            uint4 w[4];
            uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
            for (int c = 0; c < 16; ++c)
              wp[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
            uint4* dst = reinterpret_cast<uint4*>(a.out + orow + c0);
#pragma unroll
            for (int c = 0; c < 4; ++c) dst[c] = w[c];
          }
        }
      }
      if (a.lse && qr < a.Lq)
        a.lse[size_t(bh) * a.Lq + qr] = le > 0.f ? (m_ref + __log2f(le)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool kV8, bool kVirt>
cudaError_t launch_attn_dv(const AttnArgs& a, const AttnMaps& maps, cudaStream_t st) {
  // At least 100 KB so that no more than two CTAs share an SM: two 256-column
  // TMEM allocations fill the SM's 512 columns.
  const size_t smem = sizeof(Smem<D>) + 1024 > 100 * 1024 ? sizeof(Smem<D>) + 1024 : 100 * 1024;
  cudaError_t e =
      cudaFuncSetAttribute(attn_kernel<D, kV8, kVirt>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const unsigned grid = unsigned(a.B) * a.H * a.nQB;
  attn_kernel<D, kV8, kVirt><<<grid, kThreads, smem, st>>>(a, maps);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_attn_d(const AttnArgs& a, const AttnMaps& maps, cudaStream_t st) {
  // no entry point combines an INT8 V with virtual slices
  if (a.vtab) return launch_attn_dv<D, false, true>(a, maps, st);
  return a.v_scale ? launch_attn_dv<D, true, false>(a, maps, st) : launch_attn_dv<D, false, false>(a, maps, st);
}

// One CTA waits on a barrier nothing arrives at; the bounded wait runs out.
__global__ void selftest_timeout_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort, status, limit_ns);
  __syncthreads();
}

}  // namespace

cudaError_t launch_attention(const AttnArgs& a, const AttnMaps& maps, cudaStream_t st) {
  return a.d == 128 ? launch_attn_d<128>(a, maps, st) : launch_attn_d<64>(a, maps, st);
}

cudaError_t launch_selftest_timeout(uint32_t* status, uint64_t limit_ns, cudaStream_t st) {
  selftest_timeout_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace bsva
