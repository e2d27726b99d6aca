// decode_tc.cuh — split-KV MLA decode on the tcgen05 tensor cores, one CTA pair per
// (sequence, split).
//
// What it computes (《DeepSeek-V2》深度解读报告 §2.3 Absorption, §2.4 Decoupled RoPE): for every
// head h the score of cached token t is  s = scale * q_full[h] . row_t  over the 576-wide row
// [c (512) | RoPE(k^R) (64)] (content plus position channel), an online softmax over the split's
// tokens, and  O[h] = sum_t e^{s - m} c_t  over the 512-wide latent.  Every latent row is read from
// HBM once and shared by all 128 heads, which is what makes QK^T and PV dense contractions.
//
// B200 mapping.  The two CTAs of a cluster run "pair" MMAs (tcgen05 cta_group::2, M = 128): CTA r
// owns heads [64r, 64r+64) (its half of the A operand: Q for QK^T, P for PV) and each CTA's TMEM
// receives a 64-head slice of the accumulator folded over all 128 lanes, so
//   S tile (64 heads x 128 tokens, fp32)  = 64 TMEM columns per CTA (two buffers, and two
//                                           partial sums over disjoint dims: 256 columns),
//   O      (64 heads x 512 latent, fp32)  = 256 TMEM columns per CTA.
// Per 128-token tile the B operand of QK^T is split by tokens: CTA r holds tokens [64r, 64r+64)
// with all 576 dims, as 9 swizzled slabs of 64 dims.  The B operand of PV is split by latent
// columns: CTA r holds latent [256n + 128r, +128) of all 128 tokens (slabs of 32 tokens), a
// second read of the tile's rows that hits L2 because the pair reads them within microseconds.
//
// Staging.  The TMA unit of a CTA works through its tensor copies one at a time at a roughly
// fixed cost per copy (measured: ~0.35 us for anything from 8 KB to 72 KB from L2), so every copy
// is large: a CTA's K rows of a tile (from HBM) come as one 3-D box of all 9 dim-slabs (72 KB),
// and V rows (the L2 re-read) as 4-D boxes of 64 tokens x both 64-wide latent chunks x both
// latent halves (32 KB, 2 copies per tile) into a 2-slot V ring.  K tiles a few steps ahead are
// pulled into L2 with bulk prefetches.  Separate K and V buffers let the K copy of the next tile
// proceed while V of the current tile waits for its softmax.
// V rows past the split end are zeroed in shared memory before PV (rows past a sequence's end may
// hold anything, and 0 * NaN would poison the sum).
//
// Warp roles (416 threads): warps 0-7 softmax / O correction / epilogue (two warps per TMEM lane
// quadrant, each owning half of the S columns), warp 8 TMA producer and L2 prefetcher, and in the
// even CTA only: warp 9 QK^T part A (warp 9 also allocates TMEM in both CTAs), warp 11 QK^T part
// B, warps 10 and 12 PV for the two latent halves.
#pragma once

#include <cuda_bf16.h>

#include <climits>

#include "decode_common.cuh"

namespace mla {

constexpr int kTcTile = 128;                 // tokens per tile
constexpr int kTcSlab = 8192;                // 64 rows x 128 bytes
// QK^T of a tile is split along the 576 dims into two parts with their own K slot, issuing warp
// and S accumulator (the softmax adds the two): part A = dim-slabs [0, 5), part B = [5, 9).
constexpr int kTcKSlabsA = 5;
constexpr int kTcKSlabsB = 4;
__host__ __device__ constexpr int tc_part_slab0(int part) { return part ? kTcKSlabsA : 0; }
__host__ __device__ constexpr int tc_part_slabs(int part) { return part ? kTcKSlabsB : kTcKSlabsA; }
constexpr int kTcVSlots = 2;
constexpr int kTcPrefetchTiles = 4;          // K tiles pulled into L2 ahead of their load
constexpr int kTcVBox = 4 * kTcSlab;         // 64 tokens x 2 chunks x 2 latent halves
constexpr int kTcQBytes = 9 * kTcSlab;
constexpr int kTcPBytes = 2 * kTcSlab;       // 64 heads x 128 tokens bf16, two 64-token K chunks
constexpr float kTcRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows > 2^8

constexpr int kTcOffQ = 0;
constexpr int kTcOffP = kTcOffQ + kTcQBytes;
constexpr int kTcOffK = kTcOffP + kTcPBytes;  // slot of part A, then slot of part B: 9 slabs in dim order
constexpr int kTcOffV = kTcOffK + 9 * kTcSlab;
constexpr int kTcOffBar = kTcOffV + kTcVSlots * kTcVBox;
constexpr int kTcOffMisc = kTcOffBar + 256;
constexpr int kTcSmemBytes = kTcOffMisc + 64 + 2 * 256 * 4;   // the dynamic base is 1024-aligned (checked)

// TMEM columns of each CTA (512 allocated): S part A (2 buffers x 64), S part B (2 x 64), O (256).
constexpr uint32_t kTcColSA = 0;
constexpr uint32_t kTcColSB = 128;
constexpr uint32_t kTcColO = 256;

constexpr int kTcSoftmaxWarps = 8;
constexpr int kTcProducerWarp = 8;
constexpr int kTcMmaWarp = 9;     // TMEM allocation (both CTAs); QK^T part A issue (even CTA)
constexpr int kTcPvWarp = 10;     // PV issue, first latent half (even CTA)
constexpr int kTcMmaBWarp = 11;   // QK^T part B issue (even CTA)
constexpr int kTcPv1Warp = 12;    // PV issue, second latent half (even CTA)
constexpr int kTcThreads = 32 * (kTcSoftmaxWarps + 5);

struct DecodeTcArgs {
  CacheView v;
  const uint8_t* cache;   // cache rows (for L2 prefetches)
  const int32_t* seq_lens;
  int batch;
  int capacity;        // tokens a sequence can hold (lengths are clamped to it)
  int P;               // work ranges (CTA pairs)
  float scale_log2;    // softmax_scale * log2(e)
  Workspace ws;
  __nv_bfloat16* out_lat;
  float* lse;
};

// This CTA pair's work range, computed once per CTA at entry (the cursor's starting state).
struct TcPlan {
  int start, end;   // tiles [start, end): global (balanced plan) or of sequence b0 (per sequence)
  int b0, off0;     // the first sequence of the range and its tile offset in the same frame
  int b_end;        // sequences [b0, b_end) may hold segments
  int len0;         // length of sequence b0
};

struct TcBars {
  uint64_t k_full[2];            // even CTA only, per QK^T part: both CTAs' K boxes landed (one arrival per CTA + tx)
  uint64_t k_empty[2];           // both CTAs, per part: K box consumed by the MMAs
  uint64_t v_full[kTcVSlots];    // even CTA only: both CTAs' V box landed (one arrival per CTA + tx)
  uint64_t v_empty[kTcVSlots];   // both CTAs: V box consumed (one commit per PV warp)
  uint64_t fix;                  // per CTA: local load of a ragged V box
  uint64_t s_full[2];            // both: QK^T of a tile done (one commit per part)
  uint64_t s_empty[2];           // even CTA only: every softmax warp of both CTAs has read S
  uint64_t p_full;               // even CTA only: P (and corrected O) of a tile ready in both CTAs
  uint64_t p_empty;              // both: PV of a tile done reading P (one commit per PV warp)
  uint64_t o_ready;              // both: PV of a tile done writing O (one phase per tile, two commits)
  uint64_t o_final;              // both: the last PV of a segment done (one phase per segment, two commits)
  uint64_t o_free;               // both: every softmax warp of both CTAs has read O of a segment
  uint64_t q_full;               // even CTA only: Q of both CTAs landed (one phase per segment)
  uint64_t q_empty;              // both: QK^T of a segment's last tile done (two commits)
};
static_assert(sizeof(TcBars) <= 256, "barrier block");
static_assert(kTcSmemBytes <= 232448, "shared memory budget");

// Row of (seq b, token t) for a TMA coordinate; -kTcTile (a fully out-of-bounds box, which the
// TMA unit fills with zeros) when the mapping is invalid.
__device__ __forceinline__ int tma_row(const CacheView& v, int b, int t) {
  const int64_t r = cache_row(v, b, t);
  return r < 0 ? -kTcTile : static_cast<int>(r);
}

__device__ __forceinline__ uint32_t lbar(const void* p) { return mapa_shared(smem_u32(p), 0); }

// 3-D TMA load (x: element in a 64-wide dim-slab, y: cache row, z: dim-slab) into this CTA's
// shared memory; completion counted on a barrier that may live in the peer CTA.
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* m, uint32_t bar_cluster_addr, int x,
                                                 int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster_addr), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 4-D TMA load (x: element in a 64-wide chunk, y: cache row, z: chunk, w: latent half).
__device__ __forceinline__ void tma_load_4d_pair(void* dst, const CUtensorMap* m, uint32_t bar_cluster_addr, int x,
                                                 int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster_addr), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d_local(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int y, int z,
                                                  int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

// ------------------------------------------------------------------------------ TMA producer
// One warp.  Lane 0 issues the copies, in the order K(0), K(1), V(0), K(2), V(1), ..., V(n-1):
// K one tile ahead, so QK^T of tile i+1 never waits behind V of tile i.  All lanes pull the K
// rows of the tile kTcPrefetchTiles ahead into L2 with plain prefetches, so each K copy reads L2.
//  K(i): CTA r's 64 tokens [tile0 + 64r, +64) x 576 dims as two boxes, one per QK^T part
//        (5 and 4 dim-slabs).  A half-tile past the split end is loaded from a negative row
//        (zeros); its scores are masked anyway.
//  V(i): per 64-token half h of the tile, latent [256n + 128r, +128) for n = 0, 1 in one box,
//        laid out [n][chunk][64 rows][128 B].
__device__ __forceinline__ void zero_v_rows(uint8_t* box, int v) {
  for (int q = 0; q < 4; ++q)
    for (int row = v; row < 64; ++row) {
      uint4* p = reinterpret_cast<uint4*>(box + q * kTcSlab + row * 128);
#pragma unroll
      for (int u = 0; u < 8; ++u) p[u] = make_uint4(0, 0, 0, 0);
    }
}

__device__ __forceinline__ void prefetch_l2(const void* ptr) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
}

__device__ bool tc_producer(const CUtensorMap* tm_ka, const CUtensorMap* tm_kb, const CUtensorMap* tm_v,
                            const CUtensorMap* tm_q, const DecodeTcArgs& a, const TcPlan& plan, uint8_t* smem,
                            TcBars* bars, uint32_t rank, int pair, volatile int* abort_flag) {
  const int lane = threadIdx.x & 31;
  const bool l0 = lane == 0;
  const bool leader = rank == 0;
  // Lane 0 waits; the verdict (and an abort seen meanwhile) is shared with the warp.
  auto wait0 = [&](uint64_t* bar, uint32_t parity, uint32_t site) -> bool {
    int ok = 1;
    if (l0) ok = (mbar_wait(bar, parity, site) && !*abort_flag) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
  };
  SegmentCursor cur{plan.b0, plan.off0, plan.start, plan.end, plan.b_end, pair, true, plan.len0};
  Segment sg;
  int g = 0;    // global tile index of the range (K copies)
  int vn = 0;   // V boxes issued
  int k = 0;    // segment index
  uint32_t fix_phase = 0;
  bool ok = true;
  while (ok && cur.next(a.seq_lens, a.capacity, sg)) {
    const int b = sg.b, t_begin = sg.tok_begin, t_end = sg.tok_end, n_tiles = sg.n_tiles;
    // Q of sequence b.  The buffer is free once both QK^T parts have finished the previous segment.
    // Arrivals on the even CTA's barriers that only count (the data and its visibility come with
    // the TMA's complete_tx) are relaxed.
    if (k > 0 && !wait0(&bars->q_empty, static_cast<uint32_t>(k - 1) & 1u, 0x14)) {
      ok = false;
      break;
    }
    if (l0) {
      tma_load_3d_pair(smem + kTcOffQ, tm_q, lbar(&bars->q_full), 0, b * kHeads + 64 * static_cast<int>(rank), 0);
      if (leader)
        mbar_arrive_expect_tx_relaxed(lbar(&bars->q_full), 2u * kTcQBytes);
      else
        mbar_arrive_relaxed(lbar(&bars->q_full));
    }
    auto prefetch_k = [&](int j) {
      const int my0 = t_begin + j * kTcTile + 64 * static_cast<int>(rank);
      if (j >= n_tiles || my0 >= t_end) return;
      const int64_t row = cache_row(a.v, b, my0);
      if (row < 0) return;
      const int64_t nrows = a.v.num_rows - row < 64 ? a.v.num_rows - row : 64;
      const uint8_t* base = a.cache + row * (kDRow * 2);
      const int lines = static_cast<int>(nrows) * (kDRow * 2 / 128);
      for (int q = lane; q < lines; q += 32) prefetch_l2(base + q * 128);
    };
    auto issue_k = [&](int i) -> bool {
      if (i > 0) prefetch_k(i + kTcPrefetchTiles);
      const int gi = g + i;
      const int my0 = t_begin + i * kTcTile + 64 * static_cast<int>(rank);
      const int y = my0 < t_end ? tma_row(a.v, b, my0) : -kTcTile;
      for (int part = 0; part < 2; ++part) {
        if (gi >= 1 && !wait0(&bars->k_empty[part], static_cast<uint32_t>(gi - 1) & 1u, 0x10 + part)) return false;
        if (l0) {
          tma_load_3d_pair(smem + kTcOffK + tc_part_slab0(part) * kTcSlab, part ? tm_kb : tm_ka,
                           lbar(&bars->k_full[part]), 0, y, tc_part_slab0(part));
          if (leader)
            mbar_arrive_expect_tx_relaxed(lbar(&bars->k_full[part]), 2u * tc_part_slabs(part) * kTcSlab);
          else
            mbar_arrive_relaxed(lbar(&bars->k_full[part]));
        }
      }
      return true;
    };
    auto issue_v = [&](int i) -> bool {
      // The V ring doubles as the epilogue's staging buffer: the first box of a segment waits
      // until the previous segment's epilogue (in both CTAs) is done with it.
      if (i == 0 && k > 0 && !wait0(&bars->o_free, static_cast<uint32_t>(k - 1) & 1u, 0x15)) return false;
      for (int h = 0; h < 2; ++h, ++vn) {
        const int s = vn % kTcVSlots;
        if (vn >= kTcVSlots && !wait0(&bars->v_empty[s], static_cast<uint32_t>((vn / kTcVSlots) - 1) & 1u, 0x12))
          return false;
        uint8_t* box = smem + kTcOffV + s * kTcVBox;
        const int tok0 = t_begin + i * kTcTile + 64 * h;
        const int vcount = min(max(t_end - tok0, 0), 64);
        if (vcount == 64) {
          if (l0) {
            tma_load_4d_pair(box, tm_v, lbar(&bars->v_full[s]), 0, tma_row(a.v, b, tok0), 2 * static_cast<int>(rank), 0);
            if (leader)
              mbar_arrive_expect_tx_relaxed(lbar(&bars->v_full[s]), 2u * kTcVBox);
            else
              mbar_arrive_relaxed(lbar(&bars->v_full[s]));
          }
        } else {
          // Ragged: load through a CTA-local barrier, zero the rows past the end, then publish with
          // release semantics (the zeros are lane 0's own shared-memory writes).
          if (vcount > 0) {
            if (l0) {
              mbar_arrive_expect_tx(&bars->fix, kTcVBox);
              tma_load_4d_local(box, tm_v, &bars->fix, 0, tma_row(a.v, b, tok0), 2 * static_cast<int>(rank), 0);
            }
            if (!wait0(&bars->fix, fix_phase, 0x13)) return false;
            fix_phase ^= 1u;
          }
          if (l0) {
            zero_v_rows(box, vcount);
            fence_proxy_async_smem();
            if (leader)
              mbar_arrive_expect_tx_addr(lbar(&bars->v_full[s]), 0u);
            else
              mbar_arrive_addr(lbar(&bars->v_full[s]));
          }
        }
      }
      return true;
    };
    ok = issue_k(0);
    for (int j = 1; j <= kTcPrefetchTiles; ++j) prefetch_k(j);   // after K(0): it goes out first
    for (int i = 1; ok && i < n_tiles; ++i) ok = issue_k(i) && issue_v(i - 1);
    if (ok) ok = issue_v(n_tiles - 1);
    g += n_tiles;
    ++k;
  }
  return ok;
}

// ------------------------------------------------------------------------------ MMA issuers (even CTA)
// A single issuing thread cannot keep the tensor pipe busy with these shapes (each tcgen05.mma
// holds its thread for about as long as the pair takes to execute an M = 128, N = 128, K = 16
// step), so four warps issue: QK^T part A, QK^T part B (separate S accumulators over disjoint
// dims) and PV (two warps, one per latent half).  QK^T of tile i + 1 then runs on the tensor cores while the softmax warps work on
// tile i and PV of tile i - 1 completes.

// Advance a shared-memory descriptor by `bytes` (a multiple of 16): the start address field
// holds address / 16 in its low 14 bits, and every operand here lies below 256 KB, so the sum
// never carries out of the field.
__device__ __forceinline__ uint64_t sdesc_add(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

// S_part(g) = Q[:, dims of part] . K(g)[:, dims of part]^T into S buffer g & 1 of the part, for
// every global tile g of the range; Q is reloaded for each segment.
__device__ bool tc_mma_qk(uint8_t* smem, TcBars* bars, uint32_t tmem, int part, const DecodeTcArgs& a,
                          const TcPlan& plan, int pair, volatile int* abort_flag) {
  const uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
  const int slab0 = tc_part_slab0(part);
  const int nslabs = tc_part_slabs(part);
  const uint64_t dq = sdesc_sw128(smem_u32(smem + kTcOffQ + slab0 * kTcSlab), 16, 1024);
  const uint64_t dk = sdesc_sw128(smem_u32(smem + kTcOffK + slab0 * kTcSlab), 16, 1024);
  const uint32_t scol = tmem + (part ? kTcColSB : kTcColSA);
  SegmentCursor cur{plan.b0, plan.off0, plan.start, plan.end, plan.b_end, pair, true, plan.len0};
  Segment sg;
  int g = 0, k = 0;
  while (cur.next(a.seq_lens, a.capacity, sg)) {
    if (!mbar_wait_cluster(&bars->q_full, static_cast<uint32_t>(k) & 1u, 0x20)) return false;
    for (int i = 0; i < sg.n_tiles; ++i, ++g) {
      const int j = g & 1;
      // S buffer j last held tile g - 2: every softmax warp of both CTAs must have read it.
      if (g >= 2 && !mbar_wait_cluster(&bars->s_empty[j], static_cast<uint32_t>((g - 2) >> 1) & 1u, 0x24))
        return false;
      if (!mbar_wait_cluster(&bars->k_full[part], static_cast<uint32_t>(g) & 1u, 0x21)) return false;
      tc_fence_after();
      for (int c = 0; c < nslabs; ++c)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16_pair(scol + 64 * j, sdesc_add(dq, c * kTcSlab + 32 * kk), sdesc_add(dk, c * kTcSlab + 32 * kk),
                         idesc_qk, (c | kk) != 0 ? 1u : 0u);
      umma_commit_pair_mc(&bars->k_empty[part], 3);
      umma_commit_pair_mc(&bars->s_full[j], 3);
      if (*abort_flag) return false;
    }
    umma_commit_pair_mc(&bars->q_empty, 3);   // Q of this segment no longer read
    ++k;
  }
  return true;
}

// O[:, latent half nh] += P(g) . V(g)[:, half nh].  Two warps issue, one per half (separate
// accumulators); every release below therefore counts two commits.  The first V box (tokens
// 0..63 of the tile) is consumed first so it is released (and refilled) before the second.  The
// first tile of a segment overwrites O, after the previous segment's epilogue has read it.
__device__ bool tc_mma_pv(uint8_t* smem, TcBars* bars, uint32_t tmem, int nh, const DecodeTcArgs& a,
                          const TcPlan& plan, int pair, volatile int* abort_flag) {
  const uint32_t idesc_pv = idesc_bf16_f32(128, 256, false, true);
  const uint64_t dp = sdesc_sw128(smem_u32(smem + kTcOffP), 16, 1024);
  const uint64_t dv = sdesc_sw128(smem_u32(smem + kTcOffV), kTcSlab, 1024);
  SegmentCursor cur{plan.b0, plan.off0, plan.start, plan.end, plan.b_end, pair, true, plan.len0};
  Segment sg;
  int g = 0, k = 0, vn = 0;
  bool ok = true;
  while (ok && cur.next(a.seq_lens, a.capacity, sg)) {
    if (k > 0 && !mbar_wait_cluster(&bars->o_free, static_cast<uint32_t>(k - 1) & 1u, 0x25)) {
      ok = false;
      break;
    }
    for (int i = 0; i < sg.n_tiles && ok; ++i, ++g) {
      if (!mbar_wait_cluster(&bars->p_full, static_cast<uint32_t>(g) & 1u, 0x22)) {
        ok = false;
        break;
      }
      for (int h = 0; h < 2 && ok; ++h, ++vn) {
        const int vs = vn % kTcVSlots;
        if (!mbar_wait_cluster(&bars->v_full[vs], static_cast<uint32_t>(vn / kTcVSlots) & 1u, 0x23)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4) {
          const int gt = 4 * h + g4;   // 16-token group of the tile
          umma_bf16_pair(tmem + kTcColO + 128 * nh, sdesc_add(dp, h * kTcSlab + 32 * g4),
                         sdesc_add(dv, vs * kTcVBox + nh * 2 * kTcSlab + g4 * 2048), idesc_pv,
                         (i > 0 || gt > 0) ? 1u : 0u);
        }
        umma_commit_pair_mc(&bars->v_empty[vs], 3);
      }
      if (!ok) break;
      umma_commit_pair_mc(&bars->p_empty, 3);
      umma_commit_pair_mc(&bars->o_ready, 3);
      if (*abort_flag) ok = false;
    }
    // A dedicated barrier (one phase per segment) says "all PV of the segment done" to its
    // epilogue; o_ready cannot serve by parity (it may be two phases short when the epilogue starts).
    umma_commit_pair_mc(&bars->o_final, 3);
    ++k;
  }
  return ok;
}

// Each lane holds 128 bytes (w[0..31]) of its own row r = lane of a 32-row block whose rows lie
// row_stride bytes apart from row0.  Written through a 4 KB per-warp staging buffer (16-byte
// chunks XOR-swizzled by row, so both passes are free of bank conflicts beyond the 4 wavefronts
// a 512-byte access needs), each global store instruction covers four whole 128-byte row
// segments instead of 32 scattered 16-byte pieces.
__device__ __forceinline__ void store_rows_128b(uint8_t* stage, const uint32_t (&w)[32], uint8_t* row0,
                                                size_t row_stride, int lane) {
  __syncwarp();
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4*>(stage + lane * 128 + ((c ^ (lane & 7)) << 4)) =
        make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int row = 4 * j + (lane >> 3);
    const int c = lane & 7;
    const uint4 v = *reinterpret_cast<const uint4*>(stage + row * 128 + ((c ^ (row & 7)) << 4));
    *reinterpret_cast<uint4*>(row0 + row * row_stride + c * 16) = v;
  }
}

// ------------------------------------------------------------------------------ softmax warps
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Eight warps: warp w reads TMEM lane quadrant w % 4 and column half ch = w / 4, so thread
// (t = TMEM lane, ch) owns head 64*rank + (t & 63), the 32 tokens 64*(t >> 6) + 32*ch + [0, 32)
// of every tile, and O columns [128*ch, 128*ch + 128) of its lane (latent 256*ch + 128*(t >> 6)
// + [0, 128)).  The four threads (t, ch), (t ^ 64, ch), (t, ch ^ 1), (t ^ 64, ch ^ 1) share a
// head and exchange tile maxima and row sums through shared memory.
// Writes one segment's output for the head of this thread's TMEM lane: when the segment covers its
// sequence, O from TMEM divided by l_tot as bf16 into the head's output row `row` and its lse into
// *m_or_lse (if not null); else the unnormalised fp32 partial into the workspace row `row` with m
// and l into *m_or_lse and *l_out.  Kept out of line (it runs once per segment and its registers
// would otherwise crowd the per-tile loop) and given plain pointers, so that no argument struct
// has to be copied to the stack for it.
__device__ __noinline__ void tc_write_segment(bool direct, void* row, float* m_or_lse, float* l_out, uint8_t* smem,
                                              uint32_t tmem, float m_used, float l_tot) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ch = warp >> 2;
  const int t = 32 * (warp & 3) + lane;
  const int half = t >> 6;
  const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
  const int lat0 = 256 * ch + 128 * half;
  const uint32_t ocol = tmem + lane_base + kTcColO + 128 * ch;
  // Every MMA and copy of the segment is done (o_final) and the producer holds the next
  // segment's V copies until o_free: the V buffers give 4 KB of staging per warp.
  uint8_t* stage = smem + kTcOffV + warp * 4096;
  if (direct) {
    const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(row) + lat0;
    uint8_t* row0 = reinterpret_cast<uint8_t*>(dst) - static_cast<size_t>(lane) * kDLat * 2;
    for (int qb = 0; qb < 2; ++qb) {   // 64 latent columns (128 bytes of bf16) per pass
      uint32_t r[4][16];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld16(ocol + 16 * (4 * qb + q), r[q]);
      tmem_ld_wait();
      uint32_t w[32];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          __nv_bfloat162 h2 =
              __floats2bfloat162_rn(__uint_as_float(r[q][2 * e]) * inv, __uint_as_float(r[q][2 * e + 1]) * inv);
          w[8 * q + e] = *reinterpret_cast<uint32_t*>(&h2);
        }
      store_rows_128b(stage, w, row0 + 128 * qb, static_cast<size_t>(kDLat) * 2, lane);
    }
    if (half == 0 && ch == 0 && m_or_lse != nullptr)
      *m_or_lse = l_tot > 0.f ? (m_used + log2f(l_tot)) * kLn2 : -INFINITY;
  } else {
    float* dst = static_cast<float*>(row) + lat0;
    uint8_t* row0 = reinterpret_cast<uint8_t*>(dst) - static_cast<size_t>(lane) * kDLat * 4;
    for (int qb = 0; qb < 4; ++qb) {   // 32 latent columns (128 bytes of fp32) per pass
      uint32_t w[32];
      tmem_ld16(ocol + 32 * qb, *reinterpret_cast<uint32_t(*)[16]>(&w[0]));
      tmem_ld16(ocol + 32 * qb + 16, *reinterpret_cast<uint32_t(*)[16]>(&w[16]));
      tmem_ld_wait();
      store_rows_128b(stage, w, row0 + 128 * qb, static_cast<size_t>(kDLat) * 4, lane);
    }
    if (half == 0 && ch == 0) {
      *m_or_lse = m_used;
      *l_out = l_tot;
    }
  }
}

__device__ void tc_softmax(const DecodeTcArgs& a, const TcPlan& plan, int pair, uint8_t* smem, TcBars* bars,
                           float* red, uint32_t tmem, uint32_t rank, volatile int* abort_flag) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ch = warp >> 2;
  const int t = 32 * (warp & 3) + lane;   // TMEM lane
  const int hl = t & 63;                  // head within this CTA
  const int half = t >> 6;                // token half of a tile / latent quarter of O
  const int me = ch * 128 + t;            // slot in the exchange arrays
  const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
  SegmentCursor cur{plan.b0, plan.off0, plan.start, plan.end, plan.b_end, pair, true, plan.len0};
  Segment sg;
  int g = 0;   // global tile index of the range
  int k = 0;   // segment index
  bool ok = true;
  while (cur.next(a.seq_lens, a.capacity, sg)) {
  const int t_begin = sg.tok_begin, t_end = sg.tok_end, n_tiles = sg.n_tiles;
  float m_used = -INFINITY;
  float l_run = 0.f;
  for (int i = 0; i < n_tiles && ok; ++i, ++g) {
    const int j = g & 1;
    if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[j], static_cast<uint32_t>(g >> 1) & 1u, 0x30))) {
      ok = false;
      break;
    }
    tc_fence_after();
    // S = S_A + S_B (the two QK^T parts over disjoint dims).
    float sc[32];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t ra[16], rb[16];
      tmem_ld16(tmem + lane_base + kTcColSA + 64 * j + 32 * ch + 16 * q, ra);
      tmem_ld16(tmem + lane_base + kTcColSB + 64 * j + 32 * ch + 16 * q, rb);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 16; ++e) sc[16 * q + e] = __uint_as_float(ra[e]) + __uint_as_float(rb[e]);
    }
    // S is in registers (tcgen05.wait::ld above): its TMEM buffer may take tile i + 2.  The
    // arrival orders nothing else, so it is relaxed.
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_relaxed(lbar(&bars->s_empty[j]));
    // Tokens at or past the split end (only in a ragged last tile) get a score of -inf.
    const int tok0 = t_begin + i * kTcTile + 64 * half + 32 * ch;
    const int nvalid = t_end - tok0;
    if (nvalid < 32) {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (e >= nvalid) sc[e] = -INFINITY;
    }
    float mloc = sc[0];
#pragma unroll
    for (int e = 1; e < 32; ++e) mloc = fmaxf(mloc, sc[e]);
    mloc *= a.scale_log2;   // scale > 0, so the max commutes with the scaling
    float* rm = red + j * 256;
    rm[me] = mloc;
    named_bar_sync(1, 256);
    const float m_tile = fmaxf(fmaxf(mloc, rm[me ^ 64]), fmaxf(rm[me ^ 128], rm[me ^ 192]));
    float alpha = 1.f;
    bool need = false;
    if (m_used == -INFINITY) {
      m_used = m_tile;
      alpha = 0.f;
    } else if (m_tile > m_used + kTcRescaleThreshold) {
      alpha = ex2_approx(m_used - m_tile);
      m_used = m_tile;
      need = true;
    }
    if (__any_sync(0xffffffffu, need)) {
      // O must hold PV(g-1) before it is scaled (g-1 is in this segment: the first tile of a
      // segment never rescales).  Waiting on phase g-1 by parity is unambiguous: PV(g-2) is done
      // (tile g-1 waited for it before writing P) and PV(g) needs this tile's P, so o_ready has
      // completed g-1 or g phases.
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_ready, static_cast<uint32_t>(g - 1) & 1u, 0x31))) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int qb = 0; qb < 4; ++qb) {   // 2 TMEM loads in flight per wait
        const uint32_t addr = tmem + lane_base + kTcColO + 128 * ch + 32 * qb;
        uint32_t r[2][16];
#pragma unroll
        for (int k = 0; k < 2; ++k) tmem_ld16(addr + 16 * k, r[k]);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 2; ++k) {
#pragma unroll
          for (int e = 0; e < 16; ++e) r[k][e] = __float_as_uint(__uint_as_float(r[k][e]) * alpha);
          tmem_st16(addr + 16 * k, r[k]);
        }
      }
      tmem_st_wait();
    }
    // P for this tile, packed to bf16 in registers before the buffer is known to be free.
    const float neg_m = -m_used;
    float psum = 0.f;
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float p0 = ex2_approx(fmaf(sc[2 * e], a.scale_log2, neg_m));
      const float p1 = ex2_approx(fmaf(sc[2 * e + 1], a.scale_log2, neg_m));
      psum += p0 + p1;
      __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
      pk[e] = *reinterpret_cast<uint32_t*>(&h2);
    }
    // The P buffer is free once PV(g-1) has read it.  By parity this is unambiguous for the
    // same reason: p_empty has completed g-1 or g phases.
    if (g >= 1 && !__all_sync(0xffffffffu, mbar_wait(&bars->p_empty, static_cast<uint32_t>(g - 1) & 1u, 0x32))) {
      ok = false;
      break;
    }
    uint8_t* prow = smem + kTcOffP + half * kTcSlab + hl * 128;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int unit = 4 * ch + u;   // 16-byte unit (8 tokens) within the 128-byte row
      *reinterpret_cast<uint4*>(prow + ((unit ^ (hl & 7)) << 4)) =
          make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
    }
    l_run = l_run * alpha + psum;
    // Publish: P (generic-proxy writes) made visible to the tensor core, the O correction's
    // tcgen05.st ordered before the thread sync, then one release of the warp's shared-memory
    // writes (restricted to shared memory: P is all that PV reads from this thread's work)
    // followed by a relaxed arrival on the even CTA's barrier.
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      fence_release_smem_to_cluster();
      mbar_arrive_relaxed(lbar(&bars->p_full));
    }
  }
  // ---- epilogue of the segment (every warp passes the same barriers, also after a failure)
  if (ok && !__all_sync(0xffffffffu, mbar_wait(&bars->o_final, static_cast<uint32_t>(k) & 1u, 0x33))) ok = false;
  tc_fence_after();
  float* rl = red + (g & 1) * 256;   // the maxima buffer the segment's last tile did not use
  rl[me] = l_run;
  named_bar_sync(1, 256);
  const float l_tot = (l_run + rl[me ^ 64]) + (rl[me ^ 128] + rl[me ^ 192]);
  const bool write = ok && !*abort_flag;
  if (write) {
    const int64_t h = 64 * static_cast<int>(rank) + hl;
    if (sg.direct) {
      const int64_t bh = static_cast<int64_t>(sg.b) * kHeads + h;
      tc_write_segment(true, a.out_lat + bh * kDLat, a.lse != nullptr ? a.lse + bh : nullptr, nullptr, smem, tmem,
                       m_used, l_tot);
    } else {
      const int64_t ml = static_cast<int64_t>(sg.slot) * kHeads + h;
      tc_write_segment(false, a.ws.o + ml * kDLat, a.ws.m + ml, a.ws.l + ml, smem, tmem, m_used, l_tot);
    }
  }
  // Leave only on `ok`, which every softmax warp reaches at the same wait (they all wait on the
  // same barriers), never on the abort flag, which warps may read at different moments: a warp
  // leaving alone would strand the others at the next named barrier.  After the range's last
  // segment nobody waits for the release below (may_continue is the same in every warp and false
  // only when no segment follows).
  if (!ok || !cur.may_continue()) break;
  // O has been read (tcgen05.wait::ld) and the staging buffer's reads are done: release both to
  // the next segment in both CTAs.  The barrier also keeps the next segment's first tile from
  // overwriting the sums exchange before every warp has read it.
  tc_fence_before();
  fence_proxy_async_smem();
  named_bar_sync(1, 256);
  if (lane == 0) {
    fence_release_smem_to_cluster();
    mbar_arrive_relaxed(mapa_shared(smem_u32(&bars->o_free), 0));
    mbar_arrive_relaxed(mapa_shared(smem_u32(&bars->o_free), 1));
  }
  ++k;
  }
}

// ------------------------------------------------------------------------------ work plan
// Block-wide exclusive prefix sum of one int per thread (every thread of the CTA calls it);
// scratch holds at least 33 ints and is free again on return.
__device__ void block_scan(int v, int* scratch, int& excl, int& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int incl = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += u;
  }
  if (lane == 31) scratch[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int x = lane < nw ? scratch[lane] : 0;
    int inc = x;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, inc, d);
      if (lane >= d) inc += u;
    }
    if (lane < nw) scratch[lane] = inc - x;
    if (lane == 31) scratch[32] = inc;
  }
  __syncthreads();
  excl = scratch[w] + incl - v;
  total = scratch[32];
  __syncthreads();
}

// Warp-level inclusive prefix sum.
__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, v, d);
    if (lane >= d) v += u;
  }
  return v;
}

// The plan of tc_make_plan computed by one warp with shuffles only (batches of up to
// kWarpPlanMax sequences, the common case), returned to every lane: the warp that computes it
// (the producer) needs no CTA barrier to start its copies.  Same results as the block-wide version.
constexpr int kWarpPlanMax = 1024;
__device__ TcPlan tc_make_plan_warp(const DecodeTcArgs& a, int pair, bool write_table) {
  const int lane = threadIdx.x & 31;
  const int B = a.batch;
  const int P = a.P;
  // pass 1: total tiles T and the smallest non-empty sequence
  int T = 0, mn = INT_MAX;
  for (int c = 0; c < B; c += 32) {
    const int bb = c + lane;
    const int t = bb < B ? tiles_of(seq_len_checked(a.seq_lens, bb, a.capacity)) : 0;
    if (t > 0) mn = min(mn, t);
    T += __reduce_add_sync(0xffffffffu, t);
  }
  mn = __reduce_min_sync(0xffffffffu, mn);
  const bool per_seq = T > 0 && static_cast<int64_t>(mn) * P >= T;
  const int start_g = T > 0 ? range_start(pair, P, T) : 0;   // the balanced plan's range
  const int end_g = T > 0 ? range_start(pair + 1, P, T) : 0;
  TcPlan pl;
  pl.start = pl.end = 0;
  pl.b0 = pl.off0 = pl.b_end = pl.len0 = 0;
  // pass 2: prefix (of tiles, or of ranges per sequence) and this pair's piece
  int run = 0;   // prefix before this chunk
  for (int c = 0; c < B; c += 32) {
    const int bb = c + lane;
    const int L = bb < B ? seq_len_checked(a.seq_lens, bb, a.capacity) : 0;
    const int t = tiles_of(L);
    int v = t;
    if (per_seq && t > 0) {
      v = muldiv(P, t, T);   // r_b >= 1 by the condition
      v = v < t ? v : t;
    }
    const int incl = warp_incl_scan(v);
    const int excl = run + incl - v;
    if (bb < B && write_table) a.ws.off[bb] = excl;
    if (per_seq) {
      if (v > 0 && excl <= pair && pair < excl + v) {
        const int jj = pair - excl;
        pl.b0 = bb;
        pl.len0 = L;
        pl.start = muldiv(jj, t, v);
        pl.end = muldiv(jj + 1, t, v);
        pl.b_end = bb + 1;
      }
    } else if (t > 0 && start_g < end_g && excl <= start_g && start_g < excl + t) {
      pl.b0 = bb;
      pl.len0 = L;
      pl.off0 = excl;
      pl.start = start_g;
      pl.end = end_g;
      pl.b_end = B;
    }
    run = __shfl_sync(0xffffffffu, excl + v, 31);
  }
  if (write_table && lane == 0) {
    a.ws.off[B] = run;
    a.ws.off[B + 1] = per_seq ? kPlanPerSequence : kPlanBalanced;
  }
  // the lane that found the piece (at most one) hands it to the warp; otherwise the pair is idle
  const unsigned found = __ballot_sync(0xffffffffu, pl.end > pl.start);
  const int src = found ? __ffs(found) - 1 : 0;
  TcPlan r;
  r.start = __shfl_sync(0xffffffffu, pl.start, src);
  r.end = __shfl_sync(0xffffffffu, pl.end, src);
  r.b0 = __shfl_sync(0xffffffffu, pl.b0, src);
  r.off0 = __shfl_sync(0xffffffffu, pl.off0, src);
  r.b_end = __shfl_sync(0xffffffffu, pl.b_end, src);
  r.len0 = __shfl_sync(0xffffffffu, pl.len0, src);
  return r;
}

// Every thread of the CTA: tile counts of all sequences (into `tiles`, at least `batch` ints of
// shared memory), the plan kind, this pair's range and the sequence it starts in.  The even CTA
// of range 0 also writes the plan table the combine reads.
__device__ void tc_make_plan(const DecodeTcArgs& a, int pair, bool write_table, int* tiles, int* scratch,
                             TcPlan* plan) {
  const int tid = threadIdx.x;
  const int nthr = blockDim.x;
  const int B = a.batch;
  const int per = (B + nthr - 1) / nthr;
  const int lo = min(B, tid * per), hi = min(B, lo + per);
  int sum = 0, mn = INT_MAX;
  for (int bb = lo; bb < hi; ++bb) {
    const int t = tiles_of(seq_len_checked(a.seq_lens, bb, a.capacity));
    tiles[bb] = t;
    sum += t;
    if (t > 0) mn = min(mn, t);
  }
  int excl, T;
  block_scan(sum, scratch, excl, T);
  // smallest non-empty sequence (in tiles)
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, d));
  if ((tid & 31) == 0) scratch[tid >> 5] = mn;
  if (tid == 0) {
    plan->start = plan->end = 0;   // an idle pair unless a thread below finds its range
    plan->b0 = plan->off0 = 0;
    plan->b_end = 0;
    plan->len0 = 0;
  }
  __syncthreads();
  for (int i = 0; i < (nthr >> 5); ++i) mn = min(mn, scratch[i]);
  __syncthreads();
  const bool per_seq = T > 0 && static_cast<int64_t>(mn) * a.P >= T;
  if (per_seq) {
    // r_b = floor(P tiles_b / T) ranges for sequence b (>= 1 by the condition, <= tiles_b)
    auto ranges_of = [&](int t) -> int {
      if (t == 0) return 0;
      const int r = static_cast<int>((static_cast<int64_t>(a.P) * t) / T);
      return r < t ? r : t;
    };
    int rsum = 0;
    for (int bb = lo; bb < hi; ++bb) rsum += ranges_of(tiles[bb]);
    int rexcl, R;
    block_scan(rsum, scratch, rexcl, R);
    int r0 = rexcl;
    for (int bb = lo; bb < hi; ++bb) {
      const int t = tiles[bb], r = ranges_of(t);
      if (write_table) a.ws.off[bb] = r0;
      if (r0 <= pair && pair < r0 + r) {
        const int j = pair - r0;
        plan->b0 = bb;
        plan->len0 = seq_len_checked(a.seq_lens, bb, a.capacity);
        plan->off0 = 0;
        plan->start = static_cast<int>((static_cast<int64_t>(j) * t) / r);
        plan->end = static_cast<int>((static_cast<int64_t>(j + 1) * t) / r);
        plan->b_end = bb + 1;
      }
      r0 += r;
    }
    if (write_table && tid == 0) {
      a.ws.off[B] = R;
      a.ws.off[B + 1] = kPlanPerSequence;
    }
  } else {
    const int start = T > 0 ? range_start(pair, a.P, T) : 0;
    const int end = T > 0 ? range_start(pair + 1, a.P, T) : 0;
    int off = excl;   // global tile offset of sequence lo
    for (int bb = lo; bb < hi; ++bb) {
      if (write_table) a.ws.off[bb] = off;
      if (start < end && off <= start && start < off + tiles[bb]) {
        plan->b0 = bb;
        plan->len0 = seq_len_checked(a.seq_lens, bb, a.capacity);
        plan->off0 = off;
        plan->start = start;
        plan->end = end;
        plan->b_end = B;
      }
      off += tiles[bb];
    }
    if (write_table && tid == 0) {
      a.ws.off[B] = T;
      a.ws.off[B + 1] = kPlanBalanced;
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------------------------ kernel
// grid = 2 * P CTAs, clusters of 2 along x: blockIdx.x = 2 * pair + rank.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTcThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_ka, const __grid_constant__ CUtensorMap tm_kb,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q,
                     const DecodeTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  TcBars* bars = reinterpret_cast<TcBars*>(smem + kTcOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kTcOffMisc);
  int* abort_flag = reinterpret_cast<int*>(smem + kTcOffMisc + 16);
  TcPlan* plan = reinterpret_cast<TcPlan*>(smem + kTcOffMisc + 32);
  float* red = reinterpret_cast<float*>(smem + kTcOffMisc + 64);   // [2][256] tile maxima, reused for sums

  // The 128-byte swizzle atoms need a 1024-byte aligned base; the layout above has no slack for
  // realigning, so a misaligned base is reported instead of used (every CTA sees the same base).
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) set_dev_error(0x8);
    return;
  }
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int warp = threadIdx.x >> 5;
  // Setup that touches no global memory overlaps the previous kernel in the stream.
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int part = 0; part < 2; ++part) {
      mbar_init(&bars->k_full[part], 2);   // one arrival per CTA of the pair (plus the copies' bytes)
      mbar_init(&bars->k_empty[part], 1);
    }
    for (int s = 0; s < kTcVSlots; ++s) {
      mbar_init(&bars->v_full[s], 2);   // one arrival per CTA of the pair (plus the copies' bytes)
      mbar_init(&bars->v_empty[s], 2);   // one commit per PV warp
    }
    mbar_init(&bars->fix, 1);
    mbar_init(&bars->s_full[0], 2);   // one commit per QK^T part
    mbar_init(&bars->s_full[1], 2);
    mbar_init(&bars->s_empty[0], 2 * kTcSoftmaxWarps);   // every softmax warp of both CTAs
    mbar_init(&bars->s_empty[1], 2 * kTcSoftmaxWarps);
    mbar_init(&bars->p_full, 2 * kTcSoftmaxWarps);   // every softmax warp of both CTAs
    mbar_init(&bars->p_empty, 2);   // one commit per PV warp
    mbar_init(&bars->o_ready, 2);
    mbar_init(&bars->o_final, 2);
    mbar_init(&bars->o_free, 2 * kTcSoftmaxWarps);   // every softmax warp of both CTAs
    mbar_init(&bars->q_full, 2);
    mbar_init(&bars->q_empty, 2);   // one commit per QK^T part
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kTcMmaWarp) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  if (warp == kTcProducerWarp && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tm_ka);
    tma_prefetch_desc(&tm_kb);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_q);
  }
  // The barrier inits and the TMEM allocation reach the peer CTA through the cluster barrier, whose
  // wait comes after the plan.
  tc_fence_before();
  cluster_arrive_release();
  // seq_lens (read by the plan) may come from the previous kernel.
  pdl_wait();
  if (a.batch <= kWarpPlanMax) {
    // The producer warp computes the plan and hands it to the other warps through named barrier 2
    // (it only arrives, so its first copies need not wait for them).
    if (warp == kTcProducerWarp) {
      const TcPlan w = tc_make_plan_warp(a, pair, pair == 0 && rank == 0);
      if ((threadIdx.x & 31) == 0) *plan = w;
      __syncwarp();
      named_bar_arrive(2, kTcThreads);
    } else {
      named_bar_sync(2, kTcThreads);
    }
  } else {
    // The block-wide plan uses the V ring (idle until the first V copy) for the tile counts and
    // the exchange buffer for its scans; it ends with a CTA barrier.
    tc_make_plan(a, pair, pair == 0 && rank == 0, reinterpret_cast<int*>(smem + kTcOffV), reinterpret_cast<int*>(red),
                 plan);
  }
  cluster_wait_acquire();
  tc_fence_after();
  const TcPlan pl = *plan;
  const bool busy = pl.start < pl.end;   // the same in both CTAs of the pair
  const uint32_t tmem = *tmem_slot;

  if (!busy) {
    // an idle range: only the teardown below
  } else if (warp < kTcSoftmaxWarps) {
    tc_softmax(a, pl, pair, smem, bars, red, tmem, rank, abort_flag);
  } else if (warp == kTcProducerWarp) {
    if (!tc_producer(&tm_ka, &tm_kb, &tm_v, &tm_q, a, pl, smem, bars, rank, pair, abort_flag) &&
        (threadIdx.x & 31) == 0)
      *abort_flag = 1;
  } else if (rank == 0 && (threadIdx.x & 31) == 0) {
    bool ok = true;
    if (warp == kTcMmaWarp) ok = tc_mma_qk(smem, bars, tmem, 0, a, pl, pair, abort_flag);
    else if (warp == kTcMmaBWarp) ok = tc_mma_qk(smem, bars, tmem, 1, a, pl, pair, abort_flag);
    else if (warp == kTcPvWarp) ok = tc_mma_pv(smem, bars, tmem, 0, a, pl, pair, abort_flag);
    else ok = tc_mma_pv(smem, bars, tmem, 1, a, pl, pair, abort_flag);
    if (!ok) *abort_flag = 1;
  }
  __syncwarp();
  if (*reinterpret_cast<volatile int*>(abort_flag)) __nanosleep(200000);  // let stray copies land
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (warp == kTcMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace mla
