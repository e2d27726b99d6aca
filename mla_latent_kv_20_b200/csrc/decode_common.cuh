// decode_common.cuh — work plan of the split decode and the cross-range combine.
//
// Split-KV flash decoding (not on the pages; the standard exact identity of the softmax): the
// tokens of a sequence are cut into ranges; each range yields an unnormalised partial
// (O_r = sum_t e^{s_t - m_r} c_t, m_r, l_r = sum_t e^{s_t - m_r}); the partials merge exactly.
// Scores are carried in the log2 domain (scale * log2(e) folded into one factor) so the kernels
// use exp2; lse is converted back to the natural log at the end.
//
// Work plan.  Every sequence is cut into 128-token tiles (the last one ragged); T = total tiles.
// P work ranges (one CTA pair each) share them in one of two ways:
//  * per sequence (when every non-empty sequence has at least T / P tiles): sequence b gets
//    r_b = floor(P tiles_b / T) >= 1 ranges that split its tiles evenly, so every range holds one
//    piece of one sequence (pairs beyond sum r_b stay idle);
//  * balanced (otherwise): the tiles of the batch are laid end to end (sequence b owns global
//    tiles [off_b, off_b + tiles_b)) and the ranges cut that line into P pieces of equal cost,
//    where a non-empty sequence costs kSegCost + tiles_b: a range spends a few tiles' worth of
//    time at each segment it starts (the new Q, the pipeline refill, the epilogue of the previous
//    segment), so a range that meets more sequences takes fewer tiles.  On the cost line sequence
//    b spans [W_b, W_b + kSegCost + tiles_b) (W_b the sum over earlier non-empty sequences); the
//    boundary x_p = floor(p C / P) (C the total cost) falls in one such span and becomes global
//    tile off_b + max(0, x_p - W_b - kSegCost) (off_b itself when it falls in the sequence's
//    segment charge), or T when p = P.  Range p takes tiles [bound_p, bound_{p+1}) (possibly none);
//    the part of each sequence a range touches is a segment.  Tile j of sequence b sits at cost
//    y = W_b + kSegCost + j, and bound_p <= its global index exactly when x_p <= y, so the ranges
//    holding a sequence's tiles follow from W_b, tiles_b and C in closed form (the combine).
// A segment that covers its whole sequence is finished by the decode kernel; otherwise (in the
// balanced plan at most the first and the last segment of a range) its partial goes to
// workspace slot 2p (the range's first segment) or 2p + 1 (its last) and the combine merges the
// partials of the sequence in ascending range order.  The plan depends only on the sequence
// lengths and P, so paged and contiguous caches with equal lengths use the same ranges.
#pragma once

#include <cuda_bf16.h>

#include "append.cuh"

namespace mla {

constexpr int kTile = 128;               // tokens per tile of the work plan and of the decode kernel
// What a segment start costs a range in the balanced plan, in tiles: the decode kernel's range
// time fits 5.1 us per segment against 2.7 us per steady-state tile (per-tile timestamps, batch
// 128 with lengths uniform in [1024, 8192]).
constexpr int kSegCost = 2;
constexpr int kMaxDecodeBatch = 16384;   // sequences per decode call (the plan's prefix fits in smem)

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Workspace layout for P work ranges and `batch` sequences:
//   O      [2P][128][512] fp32   (unnormalised partial sums of c)
//   m      [2P][128]      fp32   (running max, log2 domain)
//   l      [2P][128]      fp32   (running sum of exp2(s - m))
//   plan   [batch + 2]    int32  (balanced: cost prefix W_b of each sequence, [batch] = C;
//                                 per sequence: first range of each sequence, [batch] = ranges used;
//                                 [batch + 1] = the plan kind)
struct Workspace {
  float* o;
  float* m;
  float* l;
  int32_t* off;
};
__host__ __device__ __forceinline__ Workspace ws_carve(void* base, int P) {
  Workspace w;
  w.o = reinterpret_cast<float*>(base);
  w.m = w.o + static_cast<int64_t>(2 * P) * kHeads * kDLat;
  w.l = w.m + static_cast<int64_t>(2 * P) * kHeads;
  w.off = reinterpret_cast<int32_t*>(w.l + static_cast<int64_t>(2 * P) * kHeads);
  return w;
}
__host__ __device__ __forceinline__ size_t ws_bytes(int batch, int P) {
  const size_t partials = static_cast<size_t>(2 * P) * kHeads * (kDLat + 2) * sizeof(float);
  return partials + ((static_cast<size_t>(batch) + 2) * sizeof(int32_t) + 15) / 16 * 16;
}

// Effective length of sequence b: seq_lens[b] clamped to [0, capacity] (error word set if it
// had to be clamped).
__device__ __forceinline__ int seq_len_checked(const int32_t* seq_lens, int b, int capacity) {
  int L = seq_lens[b];
  if (L < 0 || L > capacity) {
    set_dev_error(0x4);
    L = L < 0 ? 0 : capacity;
  }
  return L;
}
__host__ __device__ __forceinline__ int tiles_of(int L) { return (L + kTile - 1) / kTile; }

// floor(x y / z) for x, y >= 0 and z > 0, exact; 32-bit arithmetic when x y fits (the wide
// division is out of line: it is rarely taken and its code is long).
__host__ __device__ __noinline__ int muldiv_wide(uint64_t p, uint32_t z) { return static_cast<int>(p / z); }
__host__ __device__ __forceinline__ int muldiv(int x, int y, int z) {
  const uint64_t p = static_cast<uint64_t>(x) * static_cast<uint32_t>(y);
  if (p <= 0xffffffffull) return static_cast<int>(static_cast<uint32_t>(p) / static_cast<uint32_t>(z));
  return muldiv_wide(p, static_cast<uint32_t>(z));
}

// The (non-empty) range of the balanced plan that holds the tile at cost y (0 <= y < C): the last
// p with x_p = floor(p C / P) <= y, i.e. ceil((y + 1) P / C) - 1.
__host__ __device__ __forceinline__ int range_of_cost(int y, int P, int C) {
  const uint64_t x = static_cast<uint64_t>(y + 1) * static_cast<uint32_t>(P) + static_cast<uint32_t>(C - 1);
  if (x <= 0xffffffffull) return static_cast<int>(static_cast<uint32_t>(x) / static_cast<uint32_t>(C)) - 1;
  return muldiv_wide(x, static_cast<uint32_t>(C)) - 1;
}

constexpr int kPlanBalanced = 0;
constexpr int kPlanPerSequence = 1;

// One segment of a work range: tokens [tok_begin, tok_end) of sequence b.
struct Segment {
  int b;
  int tok_begin;
  int tok_end;
  int n_tiles;
  bool direct;   // covers the whole sequence: the decode kernel writes the final output
  int slot;      // workspace slot of the partial otherwise
};

// Walks the segments of one work range in order.  Every role of a CTA walks the same sequence.
struct SegmentCursor {
  int b;       // next sequence to look at
  int off;     // its tile offset (global in the balanced plan, 0 in the per-sequence plan)
  int start;   // the range's tiles [start, end) in the same frame
  int end;
  int b_end;   // sequences [b, b_end) may hold segments
  int pair;
  bool first;
  int len0;    // length of the first sequence b (known from the plan: no memory read on the way in)

  // False only if next() will return false (true may still be followed by no segment).
  __device__ bool may_continue() const { return b < b_end && off < end; }

  __device__ bool next(const int32_t* seq_lens, int capacity, Segment& s) {
    while (b < b_end && off < end) {
      const int L = first ? len0 : seq_len_checked(seq_lens, b, capacity);
      const int tiles = tiles_of(L);
      const int t0 = (start > off ? start : off) - off;
      const int t1 = (end < off + tiles ? end : off + tiles) - off;
      const int cur = b;
      off += tiles;
      ++b;
      if (t1 > t0) {
        s.b = cur;
        s.tok_begin = t0 * kTile;
        s.tok_end = min(t1 * kTile, L);
        s.n_tiles = t1 - t0;
        s.direct = t0 == 0 && t1 == tiles;
        s.slot = first ? 2 * pair : 2 * pair + 1;
        first = false;
        return true;
      }
    }
    return false;
  }
};

// Combine: one warp per (b, h) at a time; lanes own 16 of the 512 latent columns.  grid = (batch,
// 128 / (4 hpw)), block = 128: warp w of block (b, y) takes heads 4 hpw y + w hpw + [0, hpw), so the
// row's plan entries are read once for hpw heads (hpw = 1 for decode batches; 8 for many rows, as in
// a prefill, where most rows are finished by the decode kernel and the blocks only read the plan).
// At most 64 registers a thread for hpw = 1 (8 blocks per SM: a 32-sequence batch is one wave),
// 128 otherwise.  Empty rows get out_lat = 0 and lse = -inf; rows finished by the decode kernel
// (one segment) are skipped; the others merge their partials in ascending range order.
template <int hpw>
__global__ void __launch_bounds__(128, hpw == 1 ? 8 : 4) combine_kernel(Workspace ws, int P, __nv_bfloat16* __restrict__ out_lat,
                                                      float* __restrict__ lse) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x;
  const int h0 = (blockIdx.y * 4 + (threadIdx.x >> 5)) * hpw;
  const int lane = threadIdx.x & 31;
  const int B = gridDim.x;
  const bool per_seq = ws.off[B + 1] == kPlanPerSequence;
  const int off = ws.off[b];
  const int span = ws.off[b + 1] - off;   // kSegCost + tiles (balanced) or ranges (per sequence) of b
  if (span == 0) {
    for (int h = h0; h < h0 + hpw; ++h) {
      __nv_bfloat16* dst = out_lat + (static_cast<int64_t>(b) * kHeads + h) * kDLat;
      for (int i = lane; i < kDLat / 8; i += 32) reinterpret_cast<uint4*>(dst)[i] = make_uint4(0, 0, 0, 0);
      if (lse != nullptr && lane == 0) lse[static_cast<int64_t>(b) * kHeads + h] = -INFINITY;
    }
    return;
  }
  // Ranges [p0, p1] that hold pieces of b; in the per-sequence plan each holds one (slot 2p).
  // Ranges [p0, p1] that hold pieces of b; in the per-sequence plan each holds one (slot 2p); in
  // the balanced plan those holding its first and last tiles, at costs off + kSegCost and off + span - 1.
  const int C = ws.off[B];
  const int p0 = per_seq ? off : range_of_cost(off + kSegCost, P, C);
  const int p1 = per_seq ? off + span - 1 : range_of_cost(off + span - 1, P, C);
  if (p0 == p1) return;
  // The merge over the ranges, with the slot and emptiness of range p given by the plan kind (two
  // copies of the loop, so that each keeps only what its kind needs live).
  auto merge_rows = [&](auto slot_of, auto nonempty) {
#pragma unroll 1
    for (int h = h0; h < h0 + hpw; ++h) {
      __nv_bfloat16* dst = out_lat + (static_cast<int64_t>(b) * kHeads + h) * kDLat;
      // Online merge in ascending range order: after each range, (M, den, acc) hold the merge of the
      // ranges so far relative to M.  Two ranges are fetched per step so their loads overlap (every
      // partial's m is finite: a non-empty range holds at least one valid token of b).
      float M = -INFINITY, den = 0.f;
      float acc[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = 0.f;
      auto fetch = [&](int p, float& m, float& l, float4 (&o)[4]) -> bool {
        if (p > p1 || !nonempty(p)) return false;
        const int64_t ml = static_cast<int64_t>(slot_of(p)) * kHeads + h;
        m = ws.m[ml];
        l = ws.l[ml];
        const float4* src = reinterpret_cast<const float4*>(ws.o + ml * kDLat);
#pragma unroll
        for (int i = 0; i < 4; ++i) o[i] = src[lane + 32 * i];
        return true;
      };
      auto merge = [&](float m, float l, const float4 (&o)[4]) {
        const float Mn = fmaxf(M, m);
        const float sa = M == -INFINITY ? 0.f : exp2f(M - Mn);
        const float w = exp2f(m - Mn);
        den = den * sa + w * l;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[4 * i + 0] = acc[4 * i + 0] * sa + w * o[i].x;
          acc[4 * i + 1] = acc[4 * i + 1] * sa + w * o[i].y;
          acc[4 * i + 2] = acc[4 * i + 2] * sa + w * o[i].z;
          acc[4 * i + 3] = acc[4 * i + 3] * sa + w * o[i].w;
        }
        M = Mn;
      };
      constexpr int kStep = 2;
      for (int p = p0; p <= p1; p += kStep) {
        float m[kStep], l[kStep];
        float4 o[kStep][4];
        bool has[kStep];
#pragma unroll
        for (int u = 0; u < kStep; ++u) has[u] = fetch(p + u, m[u], l[u], o[u]);
#pragma unroll
        for (int u = 0; u < kStep; ++u)
          if (has[u]) merge(m[u], l[u], o[u]);
      }
      const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc[4 * i + 0] * inv, acc[4 * i + 1] * inv);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc[4 * i + 2] * inv, acc[4 * i + 3] * inv);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        reinterpret_cast<uint2*>(dst)[lane + 32 * i] = pk;
      }
      if (lse != nullptr && lane == 0)
        lse[static_cast<int64_t>(b) * kHeads + h] = den > 0.f ? (M + log2f(den)) * kLn2 : -INFINITY;
    }
  };
  if (per_seq) {
    merge_rows([](int p) { return 2 * p; }, [](int) { return true; });   // one piece per range: slot 2p
  } else {
    // Range p began before b (b is not its first segment: slot 2p + 1) when x_p < W_b = off, and is
    // empty when x_{p+1} = x_p (then the kernel wrote nothing for it).
    merge_rows([&](int p) { return muldiv(p, C, P) < off ? 2 * p + 1 : 2 * p; },
               [&](int p) { return muldiv(p, C, P) < muldiv(p + 1, C, P); });
  }
}

}  // namespace mla
