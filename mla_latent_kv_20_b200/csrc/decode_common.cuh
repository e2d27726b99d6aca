// decode_common.cuh — split-KV plan and the cross-split combine.
//
// Split-KV flash decoding (not on the pages; the standard exact identity of the softmax): the
// tokens of a sequence are cut into S ranges; each range yields an unnormalised partial
// (O_s = sum_t e^{s_t - m_s} c_t, m_s, l_s = sum_t e^{s_t - m_s}); the partials merge exactly.
// Scores are carried in the log2 domain (scale * log2(e) folded into one factor) so the kernels
// use exp2; lse is converted back to the natural log at the end.
#pragma once

#include <cuda_bf16.h>

#include "append.cuh"

namespace mla {

// Tokens per split for a sequence of length L cut into at most S ranges: ceil(L/S) rounded up
// to `align` (the decode kernel's tile).  Depends only on L, S and align, so paged and
// contiguous caches with the same lengths use identical ranges.
__host__ __device__ __forceinline__ int split_chunk(int L, int S, int align) {
  const int per = (L + S - 1) / S;
  return ((per + align - 1) / align) * align;
}
__host__ __device__ __forceinline__ int splits_used(int L, int S, int align) {
  if (L <= 0) return 0;
  const int c = split_chunk(L, S, align);
  return (L + c - 1) / c;
}

constexpr int kSplitAlign = 128;  // split boundaries are multiples of this many tokens

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Workspace layout for `batch` sequences and S splits:
//   O  [batch][S][128][512] fp32   (unnormalised partial sums of c)
//   m  [batch][S][128]      fp32   (running max, log2 domain)
//   l  [batch][S][128]      fp32   (running sum of exp2(s - m))
struct Workspace {
  float* o;
  float* m;
  float* l;
};
__host__ __device__ __forceinline__ Workspace ws_carve(void* base, int batch, int S) {
  Workspace w;
  w.o = reinterpret_cast<float*>(base);
  w.m = w.o + static_cast<int64_t>(batch) * S * kHeads * kDLat;
  w.l = w.m + static_cast<int64_t>(batch) * S * kHeads;
  return w;
}
__host__ __device__ __forceinline__ size_t ws_bytes(int batch, int S) {
  return static_cast<size_t>(batch) * S * kHeads * (kDLat + 2) * sizeof(float);
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

// Combine: one warp per (b, h); lanes own 16 of the 512 latent columns.  Splits are merged in
// ascending order.  grid = (batch, 128 / 4), block = 128.
// Sequences whose tokens fit in one split were finalised by the decode kernel itself
// (`single_done`); the combine only writes empty sequences (out_lat = 0, lse = -inf) and merges
// sequences with two or more used splits.
__global__ void __launch_bounds__(128) combine_kernel(Workspace ws, const int32_t* __restrict__ seq_lens, int S,
                                                      int align, int capacity, int single_done,
                                                      __nv_bfloat16* __restrict__ out_lat,
                                                      float* __restrict__ lse) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x;
  const int h = blockIdx.y * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  int L = seq_lens[b];
  L = L < 0 ? 0 : (L > capacity ? capacity : L);
  const int n = splits_used(L, S, align);
  if (n == 1 && single_done) return;
  const int64_t base = static_cast<int64_t>(b) * S * kHeads;
  float M = -INFINITY;
  for (int s = 0; s < n; ++s) M = fmaxf(M, ws.m[base + static_cast<int64_t>(s) * kHeads + h]);
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  float den = 0.f;
  for (int s = 0; s < n; ++s) {
    const int64_t ml = base + static_cast<int64_t>(s) * kHeads + h;
    const float w = exp2f(ws.m[ml] - M);
    den += w * ws.l[ml];
    const float4* o = reinterpret_cast<const float4*>(ws.o + ml * kDLat);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = o[lane + 32 * i];
      acc[4 * i + 0] += w * v.x;
      acc[4 * i + 1] += w * v.y;
      acc[4 * i + 2] += w * v.z;
      acc[4 * i + 3] += w * v.w;
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  __nv_bfloat16* dst = out_lat + (static_cast<int64_t>(b) * kHeads + h) * kDLat;
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

}  // namespace mla
