// gemm_tc.cuh — per-head projection GEMMs on the 5th-generation tensor cores (tcgen05).
//
// Query absorption (《DeepSeek-V2》深度解读报告 §2.3 Absorption): q_abs[b,h,:] = q_nope[b,h,:] W_UK[h]
// Value un-absorption (same section; W_UV applied after attention):  out[b,h,:] = out_lat[b,h,:] W_UV[h]
//
// Both are 128 independent GEMMs (one per head) with a small batch dimension, so they are run
// "swap-AB": the weight is the M operand (M = d_c or d_h, read from HBM once) and the batch is
// the N operand (N = batch rounded up to 16, at most 256 per CTA):
//     D[m, n] = sum_k Wt[m, k] * X[n, k]
// A = Wt is MN-major in memory (the weight's output index is contiguous), B = X is K-major.
// One CTA computes a 128 x N tile of one head: TMA streams 64-wide K slabs of A and B into a
// ring of shared-memory stages (128-byte swizzle), one thread issues tcgen05.mma into a TMEM
// accumulator, four warps read TMEM back and store bf16.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace mla {

constexpr int kGemmThreads = 192;    // warps 0-3: epilogue, warp 4: TMA producer, warp 5: MMA issuer
constexpr int kGemmKSlab = 64;       // K per stage (one 128-byte swizzle row of bf16)
constexpr int kGemmASlabBytes = 2 * 64 * 128;  // two 64-wide M chunks x 64 K rows x 128 B

__host__ __device__ constexpr int gemm_stage_bytes(int nt) { return kGemmASlabBytes + nt * 128; }

// KTOT: contraction length (128 for absorption, 512 for un-absorption).
// tmA: 2-D view of the weight, inner = M_total (output index), outer = heads * KTOT; box {64, 64}.
// tmB: 2-D view of the activation, inner = heads * KTOT, outer = batch; box {64, nt}.
// out element (n, h, m) is stored at out[n * out_bstride + h * out_hstride + m].
template <int KTOT, int NSTAGE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     __nv_bfloat16* __restrict__ out, int batch, int nt, int64_t out_bstride,
                     int out_hstride) {
  constexpr int KSLABS = KTOT / kGemmKSlab;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stage_bytes = gemm_stage_bytes(nt);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NSTAGE * stage_bytes);
  uint64_t* empty = full + NSTAGE;
  uint64_t* done = empty + NSTAGE;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128;
  const int h = blockIdx.y;
  const int n0 = blockIdx.z * nt;
  const uint32_t tmem_cols = nt <= 32 ? 32u : (nt <= 64 ? 64u : (nt <= 128 ? 128u : 256u));

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  // Setup above overlaps the previous kernel; nothing global is touched before this point.
  pdl_trigger();
  pdl_wait();

  if (warp == 4 && lane == 0) {
    // ---------------- TMA producer
    int armed[NSTAGE];
#pragma unroll
    for (int s = 0; s < NSTAGE; ++s) armed[s] = 0;
    for (int ks = 0; ks < KSLABS; ++ks) {
      const int s = ks % NSTAGE;
      if (ks >= NSTAGE && !mbar_wait(&empty[s], ((ks / NSTAGE) - 1) & 1)) {
        *abort_flag = 1;
        break;
      }
      if (*reinterpret_cast<volatile int*>(abort_flag)) break;
      uint8_t* sa = smem + s * stage_bytes;
      uint8_t* sb = sa + kGemmASlabBytes;
      mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(stage_bytes));
      const int krow = h * KTOT + ks * kGemmKSlab;
      tma_load_2d(sa, &tmA, &full[s], m0, krow);
      tma_load_2d(sa + 8192, &tmA, &full[s], m0 + 64, krow);
      tma_load_2d(sb, &tmB, &full[s], krow, n0);
      ++armed[s];
    }
    // Drain: never leave the CTA while one of its copies is still landing.
    for (int s = 0; s < NSTAGE; ++s)
      if (armed[s] > 0) mbar_wait(&full[s], (armed[s] - 1) & 1);
  } else if (warp == 5 && lane == 0) {
    // ---------------- MMA issuer
    const uint32_t idesc = idesc_bf16_f32(128, nt, /*a_mn_major=*/true, /*b_mn_major=*/false);
    bool ok = true;
    for (int ks = 0; ks < KSLABS && ok; ++ks) {
      const int s = ks % NSTAGE;
      if (!mbar_wait(&full[s], (ks / NSTAGE) & 1)) {
        *abort_flag = 1;
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + s * stage_bytes);
      const uint32_t sb = sa + kGemmASlabBytes;
#pragma unroll
      for (int kk = 0; kk < kGemmKSlab / 16; ++kk) {
        // A (MN-major): 16 K rows per MMA = 2 swizzle atoms of 1024 B; M chunks 8192 B apart.
        const uint64_t adesc = sdesc_sw128(sa + kk * 2048, 8192, 1024);
        // B (K-major): 16 K elements = 32 B into each 128-byte row; 8-row groups 1024 B apart.
        const uint64_t bdesc = sdesc_sw128(sb + kk * 32, 16, 1024);
        umma_bf16_ss(tmem_d, adesc, bdesc, idesc, (ks | kk) != 0 ? 1u : 0u);
      }
      umma_commit(&empty[s]);
    }
    umma_commit(done);  // also fires when nothing was issued, so the epilogue never waits forever
  } else if (warp < 4) {
    // ---------------- epilogue: TMEM -> registers -> bf16 global
    const bool ok = mbar_wait(done, 0);
    tc_fence_after();
    if (ok && !*reinterpret_cast<volatile int*>(abort_flag)) {
      const int m = m0 + warp * 32 + lane;
      const uint32_t trow = tmem_d + (static_cast<uint32_t>(warp * 32) << 16);
      __nv_bfloat16* o = out + static_cast<int64_t>(h) * out_hstride + m;
      for (int c = 0; c < nt; c += 16) {
        uint32_t r[16];
        tmem_ld16(trow + c, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int n = n0 + c + i;
          if (n < batch) o[static_cast<int64_t>(n) * out_bstride] = __float2bfloat16_rn(__uint_as_float(r[i]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_d, tmem_cols);
  }
}

}  // namespace mla
