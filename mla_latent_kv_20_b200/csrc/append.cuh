// append.cuh — cache append (RoPE on the shared decoupled key, then the latent row write) and
// the rotary step for the decoupled query part.
//
// 《DeepSeek-V2》深度解读报告 §2.4 Decoupled Rotary Position Embedding: RoPE acts only on the
// d_R = 64-wide position branch; the key k^R is shared by all heads and cached next to c^KV,
// so a token's cached row is [c^KV (512) | RoPE(k^R) (64)].
//
// RoPE angles are formed in fp64 (pos * base^(-2i/64) reaches ~1.3e5 rad at 128K context, where
// fp32 would lose ~1e-2 rad) and the rotated pair is rounded once to bf16.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace mla {

constexpr int kHeads = 128;
constexpr int kDHead = 128;
constexpr int kDLat = 512;
constexpr int kDRope = 64;
constexpr int kDRow = 576;
constexpr int kPage = 64;

struct CacheView {
  int32_t page_size;       // 0 contiguous, 64 paged
  int32_t max_seq_len;     // contiguous row stride between sequences / paged capacity
  int32_t max_blocks;      // paged: block-table row length
  int64_t num_rows;        // rows in the cache buffer
  const int32_t* block_table;
  int32_t num_seqs;        // contiguous: num_rows / max_seq_len ; paged: rows of block_table (or INT_MAX)
};

// Row index of (seq, token) in the cache buffer, or -1 (with the device error word set) if the
// mapping leaves the buffer.
__device__ __forceinline__ int64_t cache_row(const CacheView& v, int seq, int t) {
  if (v.page_size == 0) {
    const int64_t r = static_cast<int64_t>(seq) * v.max_seq_len + t;
    return (r >= 0 && r < v.num_rows) ? r : -1;
  }
  const int32_t blk = v.block_table[static_cast<int64_t>(seq) * v.max_blocks + t / kPage];
  const int64_t r = static_cast<int64_t>(blk) * kPage + (t % kPage);
  if (blk < 0 || r >= v.num_rows) {
    set_dev_error(0x2);
    return -1;
  }
  return r;
}

// Rotate 4 interleaved pairs (8 values starting at element 8*chunk of the 64-wide branch).
__device__ __forceinline__ uint4 rope8(uint4 raw, int chunk, int pos, double base) {
  const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(&raw);
  uint4 res;
  __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(&res);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int i = chunk * 4 + p;  // pair index 0..31
    const double theta = pow(base, -2.0 * static_cast<double>(i) / static_cast<double>(kDRope));
    double s, c;
    sincos(static_cast<double>(pos) * theta, &s, &c);
    const double xe = static_cast<double>(__bfloat162float(x[2 * p]));
    const double xo = static_cast<double>(__bfloat162float(x[2 * p + 1]));
    y[2 * p] = __double2bfloat16(xe * c - xo * s);
    y[2 * p + 1] = __double2bfloat16(xe * s + xo * c);
  }
  return res;
}

// One CTA of 72 threads per new token: threads 0..63 copy the latent (16 B each), threads
// 64..71 rotate and write the 64-wide key (4 pairs each).
__global__ void __launch_bounds__(72) cache_append_kernel(const uint4* __restrict__ c_new,
                                                          const uint4* __restrict__ kr_new,
                                                          const int32_t* __restrict__ seq_ids,
                                                          const int32_t* __restrict__ pos, uint4* cache,
                                                          CacheView v, double rope_base) {
  const int i = blockIdx.x;
  const int seq = seq_ids ? seq_ids[i] : i;
  const int p = pos[i];
  const int capacity = v.page_size == 0 ? v.max_seq_len : v.max_blocks * kPage;
  if (p < 0 || p >= capacity || seq < 0 || seq >= v.num_seqs) {
    if (threadIdx.x == 0) set_dev_error(0x1);
    return;
  }
  const int64_t row = cache_row(v, seq, p);
  if (row < 0) return;
  uint4* dst = cache + row * (kDRow / 8);
  const int t = threadIdx.x;
  if (t < 64) {
    dst[t] = c_new[static_cast<int64_t>(i) * (kDLat / 8) + t];
  } else {
    const int ch = t - 64;
    dst[64 + ch] = rope8(kr_new[static_cast<int64_t>(i) * (kDRope / 8) + ch], ch, p, rope_base);
  }
}

// q_full[b, h, 512:576] = q_pe[b, h, :] rotated at q_pos[b] (or copied when q_pos is NULL).
// grid = batch, block = 128 x 8 threads: one 16-byte chunk of one head per thread.
__global__ void __launch_bounds__(1024) qpe_kernel(const uint4* __restrict__ q_pe, const int32_t* __restrict__ q_pos,
                                                   uint4* __restrict__ q_full, double rope_base) {
  const int b = blockIdx.x;
  const int h = threadIdx.x >> 3;
  const int ch = threadIdx.x & 7;
  const uint4 raw = q_pe[(static_cast<int64_t>(b) * kHeads + h) * (kDRope / 8) + ch];
  const uint4 r = q_pos ? rope8(raw, ch, q_pos[b], rope_base) : raw;
  q_full[(static_cast<int64_t>(b) * kHeads + h) * (kDRow / 8) + kDLat / 8 + ch] = r;
}

}  // namespace mla
