// decode_tc.cuh — split-KV MLA decode on the tcgen05 tensor cores, one CTA pair per work range
// of 128-token tiles (the plan in decode_common.cuh: a range is one piece of one sequence, or a
// run of tiles that crosses sequences; each sequence piece it meets is a segment).
//
// What it computes (《DeepSeek-V2》深度解读报告 §2.3 Absorption, §2.4 Decoupled RoPE): for every
// head h the score of cached token t is  s = scale * q_full[h] . row_t  over the 576-wide row
// [c (512) | RoPE(k^R) (64)] (content plus position channel), an online softmax over the segment's
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
// latent halves (32 KB, 2 copies per tile) into a 2-slot V ring.  Separate K and V buffers let
// the K copy of the next tile proceed while V of the current tile waits for its softmax.
// V rows past the segment end are zeroed in shared memory before PV (rows past a sequence's end
// may hold anything, and 0 * NaN would poison the sum).
//
// Segments.  Every role walks the same segments of its range with a SegmentCursor.  A new
// segment loads its sequence's Q (once both QK^T parts are done with the previous Q), restarts
// the softmax state, overwrites O with its first PV (after the previous segment's epilogue has
// read O and released the V ring it stages through), and ends with an epilogue that writes either
// the final output (a segment covering its whole sequence) or an fp32 partial for the combine.
//
// Warp roles (416 threads): warps 0-7 softmax / O correction / epilogue (two warps per TMEM lane
// quadrant, each owning half of the S columns), warp 8 work plan and TMA producer, and in the
// even CTA only: warps 9 and 11 QK^T, each the 16-deep K steps of its parity into its own S
// accumulator (warp 9 also allocates TMEM in both CTAs), warps 10 and 12 PV for the two latent
// halves.
//
// FP8 cache (kFp8, 544 threads).  Rows are 576 E4M3 codes with a power-of-two scale per token (an
// E8M0 exponent byte, 2^(e - 127)): code * scale is exact in bf16, so the MMAs, the softmax and
// the epilogue are those of the bf16 cache.  The producer copies a box's codes into the upper half
// of the bf16 buffer it will become, and the box's 64 scale bytes to the buffer's start, on a
// CTA-local barrier; four converter warps (13-16) read both into registers, and after a barrier
// among themselves write the exact bf16 values of code * scale over the whole buffer in the
// swizzled layout the MMAs read (zeroing V rows past the segment end), then publish the buffer to
// the pair barrier the MMA waits on.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <climits>

#include "decode_common.cuh"

namespace mla {

constexpr int kTcTile = 128;                 // tokens per tile
constexpr int kTcSlab = 8192;                // 64 rows x 128 bytes
// QK^T of a tile is split along the 576 dims into two parts with their own K slot, issuing warp
// and S accumulator (the softmax adds the two): part A = dim-slabs [0, 5), part B = [5, 9).
constexpr int kTcKSlabsA = 5;
constexpr int kTcKSlabsB = 4;
static_assert(kTcKSlabsB <= kTcKSlabsA, "the QK^T issue loop is unrolled to part A's slab count");
__host__ __device__ constexpr int tc_part_slab0(int part) { return part ? kTcKSlabsA : 0; }
__host__ __device__ constexpr int tc_part_slabs(int part) { return part ? kTcKSlabsB : kTcKSlabsA; }
constexpr int kTcVSlots = 2;                 // one slot per 64-token half of a tile (the PV issuer relies on it)
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

// TMEM columns of each CTA (512 allocated): S of QK^T issuer 0 (2 buffers x 64), of issuer 1
// (2 x 64), O (256).
constexpr uint32_t kTcColSA = 0;
constexpr uint32_t kTcColSB = 128;
constexpr uint32_t kTcColO = 256;

constexpr int kTcSoftmaxWarps = 8;
constexpr int kTcProducerWarp = 8;
constexpr int kTcMmaWarp = 9;     // TMEM allocation (both CTAs); QK^T even K steps (even CTA)
constexpr int kTcPvWarp = 10;     // PV issue, first latent half (even CTA)
constexpr int kTcMmaBWarp = 11;   // QK^T odd K steps (even CTA)
constexpr int kTcPv1Warp = 12;    // PV issue, second latent half (even CTA)
constexpr int kTcThreads = 32 * (kTcSoftmaxWarps + 5);
// FP8 cache: four converter warps after the others.
constexpr int kTcConvWarp0 = kTcSoftmaxWarps + 5;
constexpr int kTcConvThreads = 128;
constexpr int kTcThreadsFp8 = kTcThreads + kTcConvThreads;
__host__ __device__ constexpr int tc_threads(bool fp8) { return fp8 ? kTcThreadsFp8 : kTcThreads; }
// Where the codes of a box wait for conversion: the upper half of the bf16 buffer they become.
constexpr int kTcFp8OffA = kTcKSlabsA * kTcSlab / 2;
constexpr int kTcFp8OffB = kTcKSlabsB * kTcSlab / 2;
constexpr int kTcFp8OffV = kTcVBox / 2;

struct DecodeTcArgs {
  CacheView v;
  const int32_t* seq_lens;
  int batch;
  int capacity;        // tokens a sequence can hold (lengths are clamped to it)
  int P;               // work ranges (CTA pairs)
  float scale_log2;    // softmax_scale * log2(e)
  Workspace ws;
  __nv_bfloat16* out_lat;
  float* lse;
  const uint8_t* cache;   // the cache buffer (L2 prefetch addresses)
  int row_bytes;          // bytes of one cached row: 1152 (bf16) or 576 (FP8 codes)
  const int32_t* seq_map; // query row -> cache sequence (chunked prefill), or null: row b reads sequence b
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
  uint64_t k_empty[2];           // both CTAs, per part: K box consumed by the MMAs (one commit per QK^T issuer)
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
  uint64_t kraw[2];              // FP8, per CTA and part: this CTA's K codes and scales landed (+ tx)
  uint64_t vraw[kTcVSlots];      // FP8, per CTA and slot: this CTA's V codes and scales landed (+ tx)
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

// The cache sequence that query row b reads: b itself, or seq_map[b] in a chunked prefill (where
// several query rows, one per new token, read one sequence).  A map entry outside the cache gives
// -1 (rows read as zeros); the producer also reports it through the device error word.
template <bool kMapped>
__device__ __forceinline__ int tc_cache_seq(const DecodeTcArgs& a, int b, bool report) {
  if (!kMapped) return b;
  const int s = a.seq_map[b];
  if (s >= 0 && s < a.v.num_seqs) return s;
  if (report) set_dev_error(0x2);
  return -1;
}

// Block ids of a paged cache for the producer warp, so that the row of a copy needs no dependent
// load of the block table on the way to the copy (211 instead of 223 us for the batch-128 paged
// workload, A/B on identical inputs): lane l holds the ids of pages wp + l (cur) and wp + 32 + l
// (nxt) of cache sequence b.  A lookup past wp + 48 slides the window by 32 pages and requests the
// next 32 ids then, 16 pages (8 tiles) before they are needed; lookups stay within 16 pages behind
// the furthest one (the V copies of a tile follow the K copy of the next one).
struct PageWindow {
  int b = -1, wp = 0, cur = -1, nxt = -1;
};
__device__ __forceinline__ int pw_entry(const CacheView& v, int b, int p) {
  return (p >= 0 && p < v.max_blocks) ? v.block_table[static_cast<int64_t>(b) * v.max_blocks + p] : -1;
}
// TMA row of token t of cache sequence b (every lane calls it with the same arguments and gets the
// same row), or -kTcTile (a fully out-of-bounds box) with the error word set for a bad block id.
__device__ __forceinline__ int pw_row(PageWindow& w, const CacheView& v, int b, int t, int lane) {
  const int p = t / kPage;
  if (b != w.b || p < w.wp || p >= w.wp + 64) {
    w.b = b;
    w.wp = p & ~31;
    w.cur = pw_entry(v, b, w.wp + lane);
    w.nxt = pw_entry(v, b, w.wp + 32 + lane);
  } else if (p >= w.wp + 48) {
    w.cur = w.nxt;
    w.wp += 32;
    w.nxt = pw_entry(v, b, w.wp + 32 + lane);
  }
  const int d = p - w.wp;
  const int blk = __shfl_sync(0xffffffffu, d < 32 ? w.cur : w.nxt, d & 31);
  const int64_t r = static_cast<int64_t>(blk) * kPage + (t % kPage);
  if (blk < 0 || r >= v.num_rows) {
    if (lane == 0) set_dev_error(0x2);
    return -kTcTile;
  }
  return static_cast<int>(r);
}

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
// K one tile ahead, so QK^T of tile i+1 never waits behind V of tile i.  (Pulling later K tiles
// into L2 ahead of their copies with plain prefetches measured no faster and adds code to the
// per-tile loop, so the K copies read HBM directly.)
//  K(i): CTA r's 64 tokens [tile0 + 64r, +64) x 576 dims as two boxes, one per QK^T part
//        (5 and 4 dim-slabs).  A half-tile past the split end is loaded from a negative row
//        (zeros); its scores are masked anyway.
//  V(i): per 64-token half h of the tile, latent [256n + 128r, +128) for n = 0, 1 in one box,
//        laid out [n][chunk][64 rows][128 B].
__device__ __forceinline__ void zero_v_rows(uint8_t* box, int v, int lane) {
  // each row is 4 slabs x 128 bytes: one 16-byte chunk per lane
  uint4* p = reinterpret_cast<uint4*>(box + (lane >> 3) * kTcSlab) + (lane & 7);
  for (int row = v; row < 64; ++row) p[row * 8] = make_uint4(0, 0, 0, 0);
}

// A V box that reaches past the segment end: loaded through a CTA-local barrier (if any row is
// valid), the rows past the end zeroed by all lanes after the copy has landed, then published:
// each lane's proxy fence, the warp barrier, and lane 0's arrival with release semantics on the
// even CTA's v_full.  Out of line: it runs at most twice per segment.  False if a wait failed.
__device__ __noinline__ bool tc_load_ragged_v(uint8_t* box, const CUtensorMap* tm_v, uint64_t* fix, uint32_t fix_phase,
                                              int row, int rank, int vcount, uint32_t vfull, volatile int* abort_flag) {
  const int lane = threadIdx.x & 31;
  if (vcount > 0) {
    int ok = 1;
    if (lane == 0) {
      mbar_arrive_expect_tx(fix, kTcVBox);
      tma_load_4d_local(box, tm_v, fix, 0, row, 2 * rank, 0);
      ok = (mbar_wait(fix, fix_phase, 0x13) && !*abort_flag) ? 1 : 0;
    }
    if (__shfl_sync(0xffffffffu, ok, 0) == 0) return false;
  }
  __syncwarp();
  zero_v_rows(box, vcount, lane);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    if (rank == 0)
      mbar_arrive_expect_tx_addr(vfull, 0u);
    else
      mbar_arrive_addr(vfull);
  }
  return true;
}

template <bool kMapped, bool kFp8>
__device__ bool tc_producer(const CUtensorMap* tm_ka, const CUtensorMap* tm_kb, const CUtensorMap* tm_v,
                            const CUtensorMap* tm_q, const CUtensorMap* tm_sc, const DecodeTcArgs& a,
                            const TcPlan& plan, uint8_t* smem, TcBars* bars, uint32_t rank, int pair,
                            volatile int* abort_flag) {
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
  PageWindow pw;
  const bool paged = a.v.page_size != 0;
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
    // TMA row of token t of query row b's sequence (a fully out-of-bounds box for a bad map entry).
    // Every lane calls it (the paged lookup shares the block ids across the warp).
    const int cb = tc_cache_seq<kMapped>(a, b, true);
    auto row_of = [&](int t) -> int {
      if (kMapped && cb < 0) return -kTcTile;
      return paged ? pw_row(pw, a.v, cb, t, lane) : tma_row(a.v, cb, t);
    };
    auto issue_k = [&](int i) -> bool {
      const int gi = g + i;
      const int my0 = t_begin + i * kTcTile + 64 * static_cast<int>(rank);
      const int y = my0 < t_end ? row_of(my0) : -kTcTile;
#pragma unroll 1
      for (int part = 0; part < 2; ++part) {
        if (gi >= 1 && !wait0(&bars->k_empty[part], static_cast<uint32_t>(gi - 1) & 1u, 0x10 + part)) return false;
        uint8_t* slot = smem + kTcOffK + tc_part_slab0(part) * kTcSlab;
        if (l0) {
          if constexpr (kFp8) {
            // codes to the slot's upper half, the 64 rows' scale bytes to its start (this CTA only;
            // the converter warps publish the converted slot to k_full)
            mbar_arrive_expect_tx(&bars->kraw[part], static_cast<uint32_t>(tc_part_slabs(part) * kTcSlab / 2 + 64));
            tma_load_3d(slot + (part ? kTcFp8OffB : kTcFp8OffA), part ? tm_kb : tm_ka, &bars->kraw[part], 0, y,
                        tc_part_slab0(part));
            tma_load_1d(slot, tm_sc, &bars->kraw[part], y);
          } else {
            tma_load_3d_pair(slot, part ? tm_kb : tm_ka, lbar(&bars->k_full[part]), 0, y, tc_part_slab0(part));
            if (leader)
              mbar_arrive_expect_tx_relaxed(lbar(&bars->k_full[part]), 2u * tc_part_slabs(part) * kTcSlab);
            else
              mbar_arrive_relaxed(lbar(&bars->k_full[part]));
          }
        }
      }
      return true;
    };
    auto issue_v = [&](int i) -> bool {
      // The V ring doubles as the epilogue's staging buffer: the first box of a segment waits
      // until the previous segment's epilogue (in both CTAs) is done with it.
      if (i == 0 && k > 0 && !wait0(&bars->o_free, static_cast<uint32_t>(k - 1) & 1u, 0x15)) return false;
#pragma unroll 1
      for (int h = 0; h < 2; ++h, ++vn) {
        const int s = vn % kTcVSlots;
        if (vn >= kTcVSlots && !wait0(&bars->v_empty[s], static_cast<uint32_t>((vn / kTcVSlots) - 1) & 1u, 0x12))
          return false;
        uint8_t* box = smem + kTcOffV + s * kTcVBox;
        const int tok0 = t_begin + i * kTcTile + 64 * h;
        const int vcount = min(max(t_end - tok0, 0), 64);
        const int row = vcount > 0 ? row_of(tok0) : 0;
        if constexpr (kFp8) {
          // The converter warps zero the rows past the segment end; a box with none in the
          // segment is not copied, its barrier completes on the arrival alone.
          if (l0) {
            if (vcount > 0) {
              mbar_arrive_expect_tx(&bars->vraw[s], static_cast<uint32_t>(kTcVBox / 2 + 64));
              tma_load_4d_local(box + kTcFp8OffV, tm_v, &bars->vraw[s], 0, row, 2 * static_cast<int>(rank), 0);
              tma_load_1d(box, tm_sc, &bars->vraw[s], row);
            } else {
              mbar_arrive(&bars->vraw[s]);
            }
          }
          continue;
        }
        if (vcount == 64) {
          if (l0) {
            tma_load_4d_pair(box, tm_v, lbar(&bars->v_full[s]), 0, row, 2 * static_cast<int>(rank), 0);
            if (leader)
              mbar_arrive_expect_tx_relaxed(lbar(&bars->v_full[s]), 2u * kTcVBox);
            else
              mbar_arrive_relaxed(lbar(&bars->v_full[s]));
          }
        } else {
          if (!tc_load_ragged_v(box, tm_v, &bars->fix, fix_phase, row,
                                static_cast<int>(rank), vcount, lbar(&bars->v_full[s]), abort_flag))
            return false;
          if (vcount > 0) fix_phase ^= 1u;
        }
      }
      return true;
    };
    // K(i) then V(i - 1): one call site each (the loop runs one step past the last K).  (Paged rows
    // pulled into L2 two tiles ahead by this warp's lanes measured slower: 211 -> 232 us for the
    // batch-128 paged workload, A/B on identical inputs.)
    for (int i = 0; ok && i <= n_tiles; ++i) {
      if (i < n_tiles) ok = issue_k(i);
      if (i > 0 && ok) ok = issue_v(i - 1);
    }
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

// S_j(g) = the sum over the 16-deep K steps (slab c, step kk) with kk % 2 == j of Q . K(g)^T, into
// S buffer g & 1 of issuer j (the softmax adds S_0 + S_1), for every global tile g of the range; Q
// is reloaded for each segment.  Both issuers walk the part-A slabs (0-4) first and then part B's
// (5-8), so part A's K slot is released halfway through the tile's QK^T (its next copy then
// overlaps the second half and PV) and QK^T of the next tile needs part B's copy only halfway in.
__device__ bool tc_mma_qk(uint8_t* smem, TcBars* bars, uint32_t tmem, int j, const int32_t* seq_lens, int capacity,
                          SegmentCursor cur, volatile int* abort_flag) {
  const uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
  const uint64_t dq = sdesc_sw128(smem_u32(smem + kTcOffQ), 16, 1024);
  const uint64_t dk = sdesc_sw128(smem_u32(smem + kTcOffK), 16, 1024);
  const uint32_t scol = tmem + (j ? kTcColSB : kTcColSA);
  Segment sg;
  int g = 0, k = 0;
  while (cur.next(seq_lens, capacity, sg)) {
    if (!mbar_wait_cluster(&bars->q_full, static_cast<uint32_t>(k) & 1u, 0x20)) return false;
    for (int i = 0; i < sg.n_tiles; ++i, ++g) {
      const uint32_t sb = scol + 64 * (g & 1);
      // S buffer g & 1 last held tile g - 2: every softmax warp of both CTAs must have read it.
      if (g >= 2 && !mbar_wait_cluster(&bars->s_empty[g & 1], static_cast<uint32_t>((g - 2) >> 1) & 1u, 0x24))
        return false;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        if (!mbar_wait_cluster(&bars->k_full[part], static_cast<uint32_t>(g) & 1u, 0x21)) return false;
        tc_fence_after();
        // Fully unrolled (the issue rate of this thread bounds the tensor pipe here): every
        // descriptor is a constant offset from the base.
#pragma unroll
        for (int c = tc_part_slab0(part); c < tc_part_slab0(part) + tc_part_slabs(part); ++c)
#pragma unroll
          for (int kk = 0; kk < 4; kk += 2) {
            const uint32_t off = c * kTcSlab + 32 * (kk + j);
            umma_bf16_pair(sb, sdesc_add(dq, off), sdesc_add(dk, off), idesc_qk, (c | kk) != 0 ? 1u : 0u);
          }
        umma_commit_pair_mc(&bars->k_empty[part], 3);
      }
      umma_commit_pair_mc(&bars->s_full[g & 1], 3);
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
__device__ bool tc_mma_pv(uint8_t* smem, TcBars* bars, uint32_t tmem, int nh, const int32_t* seq_lens,
                          int capacity, SegmentCursor cur, volatile int* abort_flag) {
  const uint32_t idesc_pv = idesc_bf16_f32(128, 256, false, true);
  const uint64_t dp = sdesc_sw128(smem_u32(smem + kTcOffP), 16, 1024);
  const uint64_t dv = sdesc_sw128(smem_u32(smem + kTcOffV + nh * 2 * kTcSlab), kTcSlab, 1024);
  const uint32_t ocol = tmem + kTcColO + 128 * nh;
  Segment sg;
  int g = 0, k = 0;
  bool ok = true;
  while (ok && cur.next(seq_lens, capacity, sg)) {
    if (k > 0 && !mbar_wait_cluster(&bars->o_free, static_cast<uint32_t>(k - 1) & 1u, 0x25)) {
      ok = false;
      break;
    }
    for (int i = 0; i < sg.n_tiles && ok; ++i, ++g) {
      if (!mbar_wait_cluster(&bars->p_full, static_cast<uint32_t>(g) & 1u, 0x22)) {
        ok = false;
        break;
      }
      // V box 2g + h sits in slot h of the 2-slot ring, in its (g + 1)-th fill.
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int vs = h;
        if (!mbar_wait_cluster(&bars->v_full[vs], static_cast<uint32_t>(g) & 1u, 0x23)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t pb = sdesc_add(dp, h * kTcSlab);
        const uint64_t vb = sdesc_add(dv, vs * kTcVBox);
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4)   // 16-token groups; the segment's first MMA overwrites O
          umma_bf16_pair(ocol, sdesc_add(pb, 32 * g4), sdesc_add(vb, g4 * 2048), idesc_pv,
                         (i > 0 || h > 0 || g4 > 0) ? 1u : 0u);
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

// ------------------------------------------------------------------------------ FP8 converter warps
// 2^(e - 127) of an E8M0 scale byte (e = 255, not written by the FP8 append, is read as 2^128 = inf).
__device__ __forceinline__ float e8m0_value(uint32_t e) {
  return e == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(e << 23);
}

// 16 E4M3 codes (one 16-byte chunk) times the row scale, as 16 exact bf16 values in two 16-byte
// chunks (codes 0-7, codes 8-15).
__device__ __forceinline__ void e4m3x16_to_bf16(const uint4& c, float mult, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  uint32_t o[8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const uint32_t f2 = e4m3x2_to_f16x2(static_cast<uint16_t>(w[q] >> (16 * hh)));
      const __half2 h2 = *reinterpret_cast<const __half2*>(&f2);
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(__low2float(h2) * mult, __high2float(h2) * mult);
      o[2 * q + hh] = *reinterpret_cast<const uint32_t*>(&b2);
    }
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// One box: wait for its codes and scale bytes (a CTA-local barrier), read this thread's chunks and
// its two rows' scales, meet the other converter threads (the buffer is then free to overwrite),
// write the bf16 values into the 128-byte-swizzled slab layout of the buffer (rows at or past
// `vcount` as zeros), and publish the buffer on the even CTA's barrier `done`.  The staged codes
// are laid out [slab][row][64 bytes], so converter thread ct takes chunk ct + 128 j: piece ct & 3
// of row (ct >> 2) + 32 (j & 1) of slab j >> 1.  False (the same in every converter thread) if
// the wait failed or the kernel is aborting.
template <int kSlabs>
__device__ __forceinline__ bool tc_convert_box(uint8_t* buf, int codes_off, int vcount, uint64_t* raw, uint32_t parity,
                                               uint32_t done, volatile int* abort_flag, int ct) {
  const bool got = mbar_wait(raw, parity, 0x17) && !*abort_flag;
  if (!named_bar_red_and(3, kTcConvThreads, got)) return false;
  const int pc = ct & 3;
  const int rb = ct >> 2;
  uint4 c[2 * kSlabs];
#pragma unroll
  for (int j = 0; j < 2 * kSlabs; ++j)
    c[j] = *reinterpret_cast<const uint4*>(buf + codes_off + 16 * (ct + kTcConvThreads * j));
  const float m0 = e8m0_value(buf[rb]);
  const float m1 = e8m0_value(buf[rb + 32]);
  named_bar_sync(3, kTcConvThreads);   // every staged byte has been read
#pragma unroll
  for (int j = 0; j < 2 * kSlabs; ++j) {
    const int row = rb + 32 * (j & 1);
    uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
    if (row < vcount) e4m3x16_to_bf16(c[j], (j & 1) ? m1 : m0, lo, hi);
    uint8_t* dst = buf + (j >> 1) * kTcSlab + row * 128;
    *reinterpret_cast<uint4*>(dst + (((2 * pc) ^ (row & 7)) << 4)) = lo;
    *reinterpret_cast<uint4*>(dst + (((2 * pc + 1) ^ (row & 7)) << 4)) = hi;
  }
  fence_proxy_async_smem();
  named_bar_sync(3, kTcConvThreads);
  if (ct == 0) {
    fence_release_smem_to_cluster();
    mbar_arrive_relaxed(done);
  }
  return true;
}

// The converter warps walk the boxes in the producer's order: K(0), K(1), V(0), K(2), V(1), ...
// (both parts of a K tile, then both 64-token V boxes of a tile).
template <bool kMapped>
__device__ bool tc_convert(const DecodeTcArgs& a, const TcPlan& plan, int pair, uint8_t* smem, TcBars* bars,
                           volatile int* abort_flag) {
  const int ct = static_cast<int>(threadIdx.x) - 32 * kTcConvWarp0;
  SegmentCursor cur{plan.b0, plan.off0, plan.start, plan.end, plan.b_end, pair, true, plan.len0};
  Segment sg;
  int g = 0, vn = 0;
  bool ok = true;
  while (ok && cur.next(a.seq_lens, a.capacity, sg)) {
    const int t_begin = sg.tok_begin, t_end = sg.tok_end, n_tiles = sg.n_tiles;
    for (int i = 0; ok && i <= n_tiles; ++i) {
      if (i < n_tiles) {
        const uint32_t par = static_cast<uint32_t>(g + i) & 1u;
        ok = tc_convert_box<kTcKSlabsA>(smem + kTcOffK, kTcFp8OffA, 64, &bars->kraw[0], par, lbar(&bars->k_full[0]),
                                        abort_flag, ct) &&
             tc_convert_box<kTcKSlabsB>(smem + kTcOffK + kTcKSlabsA * kTcSlab, kTcFp8OffB, 64, &bars->kraw[1], par,
                                        lbar(&bars->k_full[1]), abort_flag, ct);
      }
      for (int h = 0; ok && i > 0 && h < 2; ++h, ++vn) {
        const int s = vn % kTcVSlots;
        const int tok0 = t_begin + (i - 1) * kTcTile + 64 * h;
        const int vcount = min(max(t_end - tok0, 0), 64);
        ok = tc_convert_box<4>(smem + kTcOffV + s * kTcVBox, kTcFp8OffV, vcount, &bars->vraw[s],
                               static_cast<uint32_t>(vn / kTcVSlots) & 1u, lbar(&bars->v_full[s]), abort_flag, ct);
      }
    }
    g += n_tiles;
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
// L2 prefetch of the K rows the producer will copy kTcPfDist tiles later.  A K copy is issued only
// once QK^T has released the slot it refills (a single K slot per part), so its HBM latency sits
// on the critical loop; with the rows already in L2 it shrinks to the L2 latency.  The softmax
// warps issue the prefetches (plain prefetch.global.L2, not the TMA unit, which serialises its
// copies): this CTA's 64 rows of the tile are one contiguous 72 KB run, 576 lines over 256
// threads, once per tile.  Contiguous caches only: with pages at permuted addresses the
// prefetches measured slower (b32 x 4096 paged 65.6 -> 66.6 us, 128 mixed lengths paged 219 ->
// 223 us), against 61.8 -> 58.6 and 200 -> 195 us for the same batches contiguous; and slower
// still with the page rows handed over by the producer from its block-id window, so that no
// thread waits for the block table (212 -> 225 us for the batch-128 paged workload).
constexpr int kTcPfDist = 2;
template <bool kMapped>
__device__ __forceinline__ void tc_prefetch_tile(const DecodeTcArgs& a, int b, int tok0, int t_end) {
  if (tok0 >= t_end || a.v.page_size != 0) return;
  const int cb = tc_cache_seq<kMapped>(a, b, false);   // b is the query row
  if (kMapped && cb < 0) return;
  const int64_t r = cache_row(a.v, cb, tok0);
  if (r < 0) return;
  int n = min(64, t_end - tok0);
  if (a.v.num_rows - r < n) n = static_cast<int>(a.v.num_rows - r);   // rows of the buffer only
  const uint8_t* base = a.cache + r * a.row_bytes;
  const int lines = (n * a.row_bytes + 127) / 128;
  for (int L = threadIdx.x; L < lines; L += 32 * kTcSoftmaxWarps)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(base + 128 * L));
}

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

// O row slice *= alpha (128 fp32 columns of this thread's TMEM lane from addr).  Out of line: the
// lazy rescale runs on few tiles, and the per-tile loop stays compact.
__device__ __noinline__ void tc_rescale_o(uint32_t addr, float alpha) {
  for (int qb = 0; qb < 4; ++qb, addr += 32) {   // 2 TMEM loads in flight per wait
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

template <bool kMapped>
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
  for (int d = 1; d < kTcPfDist && d < n_tiles; ++d)
    tc_prefetch_tile<kMapped>(a, sg.b, t_begin + d * kTcTile + 64 * static_cast<int>(rank), t_end);
  for (int i = 0; i < n_tiles && ok; ++i, ++g) {
    const int j = g & 1;
    if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[j], static_cast<uint32_t>(g >> 1) & 1u, 0x30))) {
      ok = false;
      break;
    }
    tc_fence_after();
    // S = S_0 + S_1 (the two QK^T issuers' sums over disjoint K steps).
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
      tc_rescale_o(tmem + lane_base + kTcColO + 128 * ch, alpha);
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
    if (i + kTcPfDist < n_tiles)
      tc_prefetch_tile<kMapped>(a, sg.b, t_begin + (i + kTcPfDist) * kTcTile + 64 * static_cast<int>(rank), t_end);
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
// One warp computes the plan; every CTA computes it for itself (it only reads seq_lens), and the
// even CTA of range 0 also writes the table the combine reads (balanced: the cost prefix of each
// sequence and the total cost; per sequence: the first range of each and the ranges used).  Lane l
// walks the contiguous chunk of sequences [l per, (l + 1) per): three passes over it (tile totals,
// the smallest and largest sequence and the non-empty count; per-chunk sums of the prefix counts
// and, balanced, of the costs; the prefixes themselves, the table and this pair's piece), with warp
// reductions or scans between passes.  Every lane returns the same plan.  For batches of up to 128
// sequences (per <= 4) the lane's lengths are loaded once, all loads in flight together, and kept
// in registers for the three passes.
constexpr int kTcPlanCached = 4;
__device__ __noinline__ TcPlan tc_make_plan(const int32_t* seq_lens, int capacity, int B, int P, int32_t* table,
                                               int pair, bool write_table) {
  const int lane = threadIdx.x & 31;
  const int per = (B + 31) / 32;
  const int lo = min(B, lane * per), hi = min(B, lo + per);
  const bool cached = per <= kTcPlanCached;
  int lens[kTcPlanCached];
#pragma unroll
  for (int u = 0; u < kTcPlanCached; ++u) lens[u] = (cached && lo + u < hi) ? seq_len_checked(seq_lens, lo + u, capacity) : 0;
  // fn(bb, L) for every sequence bb of this lane's chunk, in order, with its checked length L
  auto for_chunk = [&](auto&& fn) {
    if (cached) {
#pragma unroll
      for (int u = 0; u < kTcPlanCached; ++u)
        if (lo + u < hi) fn(lo + u, lens[u]);
    } else {
#pragma unroll 1
      for (int bb = lo; bb < hi; ++bb) fn(bb, seq_len_checked(seq_lens, bb, capacity));
    }
  };
  // pass 1: total tiles T, the smallest non-empty sequence, the largest, the non-empty count
  int sum = 0, mn = INT_MAX, mx = 0, nne = 0;
  for_chunk([&](int, int L) {
    const int t = tiles_of(L);
    sum += t;
    mx = max(mx, t);
    if (t > 0) {
      mn = min(mn, t);
      ++nne;
    }
  });
  const int T = __reduce_add_sync(0xffffffffu, sum);
  mn = __reduce_min_sync(0xffffffffu, mn);
  mx = __reduce_max_sync(0xffffffffu, mx);
  const bool per_seq = T > 0 && static_cast<int64_t>(mn) * P >= T;
  if (per_seq && mx == mn && static_cast<int64_t>(mn) * B == T) {
    // Every sequence has the same tile count t (the usual case): r_b = floor(P t / (B t)) =
    // floor(P / B) for all b, so the prefix is b r and no scan is needed.  Same plan as below.
    const int t = mn;
    const int r = min(P / B, t);
    if (write_table) {
      #pragma unroll 1
      for (int bb = lo; bb < hi; ++bb) table[bb] = bb * r;
      if (lane == 0) {
        table[B] = B * r;
        table[B + 1] = kPlanPerSequence;
      }
    }
    TcPlan pl;
    pl.start = pl.end = 0;
    pl.b0 = pl.off0 = pl.b_end = pl.len0 = 0;
    const int b0 = pair / r, jj = pair - b0 * r;
    if (b0 < B) {
      pl.b0 = b0;
      pl.len0 = seq_len_checked(seq_lens, b0, capacity);
      pl.start = muldiv(jj, t, r);
      pl.end = muldiv(jj + 1, t, r);
      pl.b_end = b0 + 1;
    }
    return pl;
  }
  // what each sequence contributes to the prefix: its tiles, or (per sequence) its ranges
  // r_b = floor(P tiles_b / T), which the condition makes >= 1 and which is at most tiles_b
  auto count_of = [&](int t) -> int {
    if (!per_seq || t == 0) return t;
    const int r = muldiv(P, t, T);
    return r < t ? r : t;
  };
  // pass 2: this lane's share of the prefix, and (balanced) of the cost line
  int csum = sum;
  if (per_seq) {
    csum = 0;
    for_chunk([&](int, int L) { csum += count_of(tiles_of(L)); });
  }
  const int wsum = sum + kSegCost * nne;
  int incl = csum, wincl = wsum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, d);
    const int uw = __shfl_up_sync(0xffffffffu, wincl, d);
    if (lane >= d) {
      incl += u;
      wincl += uw;
    }
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  const int C = __shfl_sync(0xffffffffu, wincl, 31);
  // pass 3: the prefixes, the table, and the piece of this pair.  Balanced: the range's cost
  // interval [x0, x1) of the cost line; the lane whose sequence span holds x0 finds the start
  // (and the first sequence), the one whose span holds x1 the end (none: x1 = C, the end is T).
  const int x0 = (T > 0 && !per_seq) ? muldiv(pair, C, P) : 0;
  const int x1 = (T > 0 && !per_seq) ? muldiv(pair + 1, C, P) : 0;
  TcPlan pl;
  pl.start = pl.end = 0;
  pl.b0 = pl.off0 = pl.b_end = pl.len0 = 0;
  bool found_start = false, found_end = false;
  int run = incl - csum;
  int W = wincl - wsum;
  for_chunk([&](int bb, int L) {
    const int t = tiles_of(L);
    const int v = count_of(t);
    if (write_table) table[bb] = per_seq ? run : W;
    if (per_seq) {
      if (v > 0 && run <= pair && pair < run + v) {
        const int jj = pair - run;
        pl.b0 = bb;
        pl.len0 = L;
        pl.start = muldiv(jj, t, v);
        pl.end = muldiv(jj + 1, t, v);
        pl.b_end = bb + 1;
        found_start = found_end = true;
      }
    } else if (t > 0) {
      if (W <= x0 && x0 < W + kSegCost + t) {
        pl.b0 = bb;
        pl.len0 = L;
        pl.off0 = run;
        pl.start = run + max(0, x0 - W - kSegCost);
        pl.b_end = B;
        found_start = true;
      }
      if (W <= x1 && x1 < W + kSegCost + t) {
        pl.end = run + max(0, x1 - W - kSegCost);
        found_end = true;
      }
      W += kSegCost + t;
    }
    run += v;
  });
  if (write_table && lane == 0) {
    table[B] = per_seq ? total : C;
    table[B + 1] = per_seq ? kPlanPerSequence : kPlanBalanced;
  }
  // the lanes that found the start and the end (at most one each) hand them to the warp;
  // otherwise the pair is idle (or, balanced, its range ends at T)
  const unsigned fs = __ballot_sync(0xffffffffu, found_start);
  const unsigned fe = __ballot_sync(0xffffffffu, found_end);
  const int ss = fs ? __ffs(fs) - 1 : 0;
  const int se = fe ? __ffs(fe) - 1 : 0;
  TcPlan r;
  r.start = __shfl_sync(0xffffffffu, pl.start, ss);
  r.end = __shfl_sync(0xffffffffu, pl.end, se);
  r.b0 = __shfl_sync(0xffffffffu, pl.b0, ss);
  r.off0 = __shfl_sync(0xffffffffu, pl.off0, ss);
  r.b_end = __shfl_sync(0xffffffffu, pl.b_end, ss);
  r.len0 = __shfl_sync(0xffffffffu, pl.len0, ss);
  if (!per_seq) {
    if (!fe) r.end = T;
    if (!fs) r.start = r.end = 0;   // no tiles at all (T = 0)
  } else if (!fs) {
    r.start = r.end = 0;
  }
  return r;
}

// ------------------------------------------------------------------------------ kernel
// grid = 2 * P CTAs, clusters of 2 along x: blockIdx.x = 2 * pair + rank.  kMapped: query rows
// read the cache sequences of a.seq_map (chunked prefill); the decode instance carries none of it.
// kFp8: the cache holds E4M3 codes with E8M0 row scales (tm_ka, tm_kb, tm_v are byte maps of the
// codes, tm_sc the 1-D byte map of the scales; unused otherwise).
template <bool kMapped, bool kFp8 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(tc_threads(kFp8), 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_ka, const __grid_constant__ CUtensorMap tm_kb,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_sc, const DecodeTcArgs a) {
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
      mbar_init(&bars->k_empty[part], 2);   // one commit per QK^T issuer
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
    if (kFp8) {
      for (int part = 0; part < 2; ++part) mbar_init(&bars->kraw[part], 1);   // this CTA's producer (plus bytes)
      for (int s = 0; s < kTcVSlots; ++s) mbar_init(&bars->vraw[s], 1);
    }
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
    if (kFp8) tma_prefetch_desc(&tm_sc);
  }
  // The barrier inits and the TMEM allocation reach the peer CTA through the cluster barrier, whose
  // wait comes after the plan.
  tc_fence_before();
  cluster_arrive_release();
  // seq_lens (read by the plan) may come from the previous kernel.
  pdl_wait();
  // The producer warp computes the plan and hands it to the other warps through named barrier 2
  // (it only arrives, so its first copies need not wait for them).
  if (warp == kTcProducerWarp) {
    const TcPlan w = tc_make_plan(a.seq_lens, a.capacity, a.batch, a.P, a.ws.off, pair, pair == 0 && rank == 0);
    if ((threadIdx.x & 31) == 0) *plan = w;
    __syncwarp();
    named_bar_arrive(2, tc_threads(kFp8));
  } else {
    named_bar_sync(2, tc_threads(kFp8));
  }
  cluster_wait_acquire();
  tc_fence_after();
  const TcPlan pl = *plan;
  const bool busy = pl.start < pl.end;   // the same in both CTAs of the pair
  const uint32_t tmem = *tmem_slot;

  if (!busy) {
    // an idle range: only the teardown below
  } else if (warp < kTcSoftmaxWarps) {
    tc_softmax<kMapped>(a, pl, pair, smem, bars, red, tmem, rank, abort_flag);
  } else if (warp == kTcProducerWarp) {
    if (!tc_producer<kMapped, kFp8>(&tm_ka, &tm_kb, &tm_v, &tm_q, &tm_sc, a, pl, smem, bars, rank, pair,
                                    abort_flag) &&
        (threadIdx.x & 31) == 0)
      *abort_flag = 1;
  } else if (kFp8 && warp >= kTcConvWarp0) {
    if (!tc_convert<kMapped>(a, pl, pair, smem, bars, abort_flag) && threadIdx.x == 32 * kTcConvWarp0)
      *abort_flag = 1;
  } else if (rank == 0 && (threadIdx.x & 31) == 0) {
    bool ok = true;
    // One out-of-line copy of each issuer serves both of its warps (part / latent half as argument).
    const SegmentCursor cur{pl.b0, pl.off0, pl.start, pl.end, pl.b_end, pair, true, pl.len0};
    if (warp == kTcMmaWarp || warp == kTcMmaBWarp)
      ok = tc_mma_qk(smem, bars, tmem, warp == kTcMmaWarp ? 0 : 1, a.seq_lens, a.capacity, cur, abort_flag);
    else
      ok = tc_mma_pv(smem, bars, tmem, warp == kTcPvWarp ? 0 : 1, a.seq_lens, a.capacity, cur, abort_flag);
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
