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

// ------------------------------------------------------------------------------------------
// FP8 (E4M3) latent cache rows (《DeepSeek-V2》深度解读报告 §4.2 效率证据: FP8 serving with the KV cache
// at about 6 bits per element; the format is this library's reading).  A token's row is the 576
// values [c^KV | RoPE(k^R, pos)], taken in fp64 (the latent exactly from its bf16 input, the key
// rotated in fp64 and never rounded to bf16), stored as 576 OCP E4M3 codes plus one fp32 scale per
// token: the power of two 2^k, k the smallest integer with amax <= 448 * 2^k (amax the row's
// largest magnitude, k = 0 for an all-zero row), kept as its E8M0 byte k + 127.  A value x is
// coded as the E4M3 value nearest to the fp32 rounding of x * 2^-k (ties to even, saturating at
// +-448).  A code times its scale is exact in bf16, so the decode expands FP8 tiles into exact bf16
// MMA operands.
// ------------------------------------------------------------------------------------------
constexpr double kE4m3Max = 448.0;

// Two E4M3 codes (round to nearest even, saturating to +-448) of lo and hi; lo in the low byte.
__device__ __forceinline__ uint16_t e4m3x2_rn_sat(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

// k of the row scale 2^k: the smallest integer with amax <= 448 * 2^k (0 for amax = 0).
__device__ __forceinline__ int fp8_scale_exp(double amax) {
  if (!(amax > 0.0)) return 0;
  int e = 0;
  (void)frexp(amax / kE4m3Max, &e);   // amax / 448 = f 2^e, f in [0.5, 1): 2^e bounds it up to rounding
  int k = e;
  if (amax > kE4m3Max * ldexp(1.0, k)) ++k;          // settle k by exact comparisons
  if (amax <= kE4m3Max * ldexp(1.0, k - 1)) --k;
  return k;
}

// One CTA of 96 threads per new token: threads 0..63 hold 8 latent values each, threads 64..95
// one rotated pair each (fp64); the CTA reduces the row's largest magnitude, then every thread
// codes its values and writes them, and thread 0 writes the token's scale.
__global__ void __launch_bounds__(96) cache_append_fp8_kernel(const uint4* __restrict__ c_new,
                                                              const __nv_bfloat162* __restrict__ kr_new,
                                                              const int32_t* __restrict__ seq_ids,
                                                              const int32_t* __restrict__ pos, uint8_t* cache,
                                                              uint8_t* scales, CacheView v, RopeFreq f) {
  __shared__ double red[3];
  pdl_trigger();
  pdl_wait();
  const int i = blockIdx.x;
  const int seq = seq_ids ? seq_ids[i] : i;
  const int p = pos[i];
  const int capacity = v.page_size == 0 ? v.max_seq_len : v.max_blocks * kPage;
  if (p < 0 || p >= capacity || seq < 0 || seq >= v.num_seqs) {   // the same for every thread of the CTA
    if (threadIdx.x == 0) set_dev_error(0x1);
    return;
  }
  const int64_t row = cache_row(v, seq, p);
  if (row < 0) return;
  const int t = threadIdx.x;
  double x[8];
  int nv = 2;
  if (t < 64) {
    const uint4 u = c_new[static_cast<int64_t>(i) * (kDLat / 8) + t];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      x[2 * j] = static_cast<double>(__low2float(h[j]));
      x[2 * j + 1] = static_cast<double>(__high2float(h[j]));
    }
    nv = 8;
  } else {
    const int pr = t - 64;   // pair index 0..31
    double sn, cs;
    sincos(static_cast<double>(p) * f.inv_freq[pr], &sn, &cs);
    const __nv_bfloat162 k2 = kr_new[static_cast<int64_t>(i) * (kDRope / 2) + pr];
    const double xe = static_cast<double>(__low2float(k2));
    const double xo = static_cast<double>(__high2float(k2));
    x[0] = xe * cs - xo * sn;
    x[1] = xe * sn + xo * cs;
#pragma unroll
    for (int j = 2; j < 8; ++j) x[j] = 0.0;
  }
  double am = 0.0;
#pragma unroll
  for (int j = 0; j < 8; ++j) am = fmax(am, fabs(x[j]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmax(am, __shfl_xor_sync(0xffffffffu, am, o));
  if ((t & 31) == 0) red[t >> 5] = am;
  __syncthreads();
  const double amax = fmax(fmax(red[0], red[1]), red[2]);
  // The E8M0 byte holds k in [-127, 127]; bf16 inputs keep amax within it.
  const int k = min(max(fp8_scale_exp(amax), -127), 127);
  const double inv = ldexp(1.0, -k);   // x * 2^-k is exact in fp64
  uint8_t* dst = cache + row * kDRow;
  if (nv == 8) {
    uint32_t w[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t lo = e4m3x2_rn_sat(static_cast<float>(x[4 * j] * inv), static_cast<float>(x[4 * j + 1] * inv));
      const uint32_t hi = e4m3x2_rn_sat(static_cast<float>(x[4 * j + 2] * inv), static_cast<float>(x[4 * j + 3] * inv));
      w[j] = lo | (hi << 16);
    }
    *reinterpret_cast<uint2*>(dst + 8 * t) = make_uint2(w[0], w[1]);
  } else {
    *reinterpret_cast<uint16_t*>(dst + kDLat + 2 * (t - 64)) =
        e4m3x2_rn_sat(static_cast<float>(x[0] * inv), static_cast<float>(x[1] * inv));
  }
  if (t == 0) scales[row] = static_cast<uint8_t>(k + 127);
}

}  // namespace mla
