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

// Inverse frequencies base^(-2i/64) of the 32 rotation pairs, formed once on the host in fp64.
struct RopeFreq {
  double inv_freq[kDRope / 2];
};

// Rotate one interleaved pair (x_{2i}, x_{2i+1}) by pos * inv_freq[i]: the angle and the rotation
// in fp64, one rounding to bf16 per output.
__device__ __forceinline__ __nv_bfloat162 rope_pair(__nv_bfloat162 x, double c, double s) {
  const double xe = static_cast<double>(__low2float(x));
  const double xo = static_cast<double>(__high2float(x));
  __nv_bfloat162 y;
  y.x = __double2bfloat16(xe * c - xo * s);
  y.y = __double2bfloat16(xe * s + xo * c);
  return y;
}

// One CTA of 96 threads per new token: threads 0..63 copy the latent (16 B each), threads
// 64..95 rotate one pair of the 64-wide key each (one fp64 sincos per thread, all in parallel).
__global__ void __launch_bounds__(96) cache_append_kernel(const uint4* __restrict__ c_new,
                                                          const __nv_bfloat162* __restrict__ kr_new,
                                                          const int32_t* __restrict__ seq_ids,
                                                          const int32_t* __restrict__ pos, uint4* cache,
                                                          CacheView v, RopeFreq f) {
  pdl_trigger();
  pdl_wait();
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
  const int t = threadIdx.x;
  if (t < 64) {
    uint4* dst = cache + row * (kDRow / 8);
    dst[t] = c_new[static_cast<int64_t>(i) * (kDLat / 8) + t];
  } else {
    const int pr = t - 64;   // pair index 0..31
    double sn, cs;
    sincos(static_cast<double>(p) * f.inv_freq[pr], &sn, &cs);
    __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(cache + row * (kDRow / 8) + kDLat / 8);
    dst[pr] = rope_pair(kr_new[static_cast<int64_t>(i) * (kDRope / 2) + pr], cs, sn);
  }
}

}  // namespace mla
