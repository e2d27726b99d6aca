// decode_simt.cuh — split-KV decode on CUDA cores (fp32 FMA), used for the first parity pass of
// the decode path before the tensor-core kernel.  One CTA handles 16 heads of one (sequence,
// split) pair and streams the split's cached rows through shared memory in 64-token tiles with
// an online softmax (《DeepSeek-V2》深度解读报告 §2.3/§2.4: score = q_abs.c + q_pe.k^R, the
// content and position channels summed; the latent row is both key and value).
#pragma once

#include "decode_common.cuh"

namespace mla {

constexpr int kSimtHeads = 16;
constexpr int kSimtTile = 64;
constexpr int kSimtRowPad = 584;  // bf16 per padded row in shared memory (1168 B, 16-B multiple)
constexpr int kSplitAlign = 128;  // split boundaries are multiples of this many tokens

constexpr size_t simt_smem_bytes() {
  return sizeof(__nv_bfloat16) * (kSimtHeads * kDRow + kSimtTile * kSimtRowPad) +
         sizeof(float) * (kSimtHeads * kSimtTile + 3 * kSimtHeads);
}

// grid = (128 / 16, S, batch), block = 256.
__global__ void __launch_bounds__(256) decode_simt_kernel(const __nv_bfloat16* __restrict__ q_full,
                                                          const __nv_bfloat16* __restrict__ cache, CacheView v,
                                                          const int32_t* __restrict__ seq_lens, int S,
                                                          float scale_log2, Workspace ws) {
  extern __shared__ uint4 smem_v4[];
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(smem_v4);
  __nv_bfloat16* Ks = Qs + kSimtHeads * kDRow;
  float* Ps = reinterpret_cast<float*>(Ks + kSimtTile * kSimtRowPad);
  float* s_alpha = Ps + kSimtHeads * kSimtTile;
  float* s_m = s_alpha + kSimtHeads;
  float* s_l = s_m + kSimtHeads;

  const int h0 = blockIdx.x * kSimtHeads;
  const int split = blockIdx.y;
  const int b = blockIdx.z;
  const int tid = threadIdx.x;
  const int capacity = v.page_size == 0 ? v.max_seq_len : v.max_blocks * kPage;
  const int L = seq_len_checked(seq_lens, b, capacity);
  const int chunk = split_chunk(L, S, kSplitAlign);
  const int t_begin = split * chunk;
  if (L == 0 || t_begin >= L) return;  // empty range: the combine never reads this split
  const int t_end = min(L, t_begin + chunk);

  // q rows of this head group
  for (int i = tid; i < kSimtHeads * (kDRow / 8); i += 256) {
    const int hh = i / (kDRow / 8), ch = i % (kDRow / 8);
    reinterpret_cast<uint4*>(Qs)[hh * (kDRow / 8) + ch] =
        reinterpret_cast<const uint4*>(q_full)[(static_cast<int64_t>(b) * kHeads + h0 + hh) * (kDRow / 8) + ch];
  }
  if (tid < kSimtHeads) {
    s_m[tid] = -INFINITY;
    s_l[tid] = 0.f;
  }

  const int hh = tid >> 4;  // head within the group for the score and O phases
  const int jj = tid & 15;
  float o[32];
#pragma unroll
  for (int r = 0; r < 32; ++r) o[r] = 0.f;

  for (int t0 = t_begin; t0 < t_end; t0 += kSimtTile) {
    __syncthreads();
    for (int i = tid; i < kSimtTile * (kDRow / 8); i += 256) {
      const int row = i / (kDRow / 8), ch = i % (kDRow / 8);
      const int t = t0 + row;
      uint4 val = make_uint4(0, 0, 0, 0);
      if (t < t_end) {
        const int64_t r = cache_row(v, b, t);
        if (r >= 0) val = reinterpret_cast<const uint4*>(cache)[r * (kDRow / 8) + ch];
      }
      *reinterpret_cast<uint4*>(Ks + row * kSimtRowPad + ch * 8) = val;
    }
    __syncthreads();
    // scores for (hh, t = jj + 16 i)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tt = jj + 16 * i;
      const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(Qs + hh * kDRow);
      const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(Ks + tt * kSimtRowPad);
      float acc = 0.f;
#pragma unroll 8
      for (int k = 0; k < kDRow / 2; ++k) {
        const float2 a = __bfloat1622float2(q2[k]);
        const float2 c = __bfloat1622float2(k2[k]);
        acc = fmaf(a.x, c.x, acc);
        acc = fmaf(a.y, c.y, acc);
      }
      Ps[hh * kSimtTile + tt] = (t0 + tt < t_end) ? acc * scale_log2 : -INFINITY;
    }
    __syncthreads();
    // online softmax: warp w owns heads 2w and 2w+1
    {
      const int w = tid >> 5, lane = tid & 31;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int hq = 2 * w + q;
        const float a0 = Ps[hq * kSimtTile + lane], a1 = Ps[hq * kSimtTile + lane + 32];
        float mx = fmaxf(a0, a1);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_old = s_m[hq];
        const float m_new = fmaxf(m_old, mx);
        const float p0 = exp2f(a0 - m_new), p1 = exp2f(a1 - m_new);
        float sum = p0 + p1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        Ps[hq * kSimtTile + lane] = p0;
        Ps[hq * kSimtTile + lane + 32] = p1;
        __syncwarp();
        if (lane == 0) {
          const float alpha = exp2f(m_old - m_new);
          s_alpha[hq] = alpha;
          s_l[hq] = s_l[hq] * alpha + sum;
          s_m[hq] = m_new;
        }
      }
    }
    __syncthreads();
    {
      const float alpha = s_alpha[hh];
#pragma unroll
      for (int r = 0; r < 32; ++r) o[r] *= alpha;
      const int ntok = min(kSimtTile, t_end - t0);
      for (int tt = 0; tt < ntok; ++tt) {
        const float p = Ps[hh * kSimtTile + tt];
        const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(Ks + tt * kSimtRowPad);
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const float2 c = __bfloat1622float2(v2[jj + 16 * r]);
          o[2 * r] = fmaf(p, c.x, o[2 * r]);
          o[2 * r + 1] = fmaf(p, c.y, o[2 * r + 1]);
        }
      }
    }
  }
  __syncthreads();
  const int64_t ml = (static_cast<int64_t>(b) * S + split) * kHeads + h0 + hh;
  float2* dst = reinterpret_cast<float2*>(ws.o + ml * kDLat);
#pragma unroll
  for (int r = 0; r < 16; ++r) dst[jj + 16 * r] = make_float2(o[2 * r], o[2 * r + 1]);
  if (jj == 0) {
    ws.m[ml] = s_m[hh];
    ws.l[ml] = s_l[hh];
  }
}

}  // namespace mla
