// out_proj.cuh — the attention block's output projection on the tcgen05 tensor cores.
//
// What it computes (《DeepSeek-V2》深度解读报告 §2.3 Absorption: W_U^V belongs with the output
// projection W_O; §3.3: model width d = 5120): for each sequence b,
//     y[b] = W_O [out[b, 0, :] | out[b, 1, :] | ... | out[b, 127, :]]      (5120 <- 16384)
// on the un-absorbed heads' outputs.  Products exact in fp32, sums over the 16384 inputs in fp32,
// one rounding of y to bf16.
//
// B200 mapping.  The weight (5120 x 16384 bf16, 168 MB) streams from HBM once per N tile and is the
// M operand ("swap-AB": M = output dims in 40 tiles of 128, N = sequences in tiles of NT = 32, or
// of 128 for batches above 32 so that the weight streams once per 128 sequences, K = 16384); K is
// split over the SPLIT CTAs of a cluster (8: twice as many such clusters are resident at once as
// 16-CTA ones), each streaming its share through a ring of 40 KB (NT = 32, 4 stages) or 64 KB
// (NT = 128, 3 stages) stages while two threads issue the MMAs into two TMEM accumulators; the
// SPLIT partial tiles are reduced through distributed shared memory (CTA r sums rows [R r, R r + R),
// R = 128 / SPLIT) and written as bf16.
// grid = (SPLIT, 40, ceil(B / NT)), clusters of SPLIT along x (set at launch); 224 threads: warps
// 0-3 epilogue and reduction, warp 4 TMA producer, warps 5-6 MMA issuers.
#pragma once

#include <cuda_bf16.h>

#include "down_proj.cuh"
#include "ptx.cuh"

namespace mla {

constexpr int kOpIn = kHeads * kDHead;   // 16384 inputs
constexpr int kOpOut = kDHidden;         // 5120 outputs
constexpr int kOpMTiles = kOpOut / 128;
constexpr int kOpKS = 128;               // contraction columns per stage
constexpr int kOpThreads = 224;
constexpr int kOpWBytes = kOpKS * 128 * 2;
static_assert(kOpOut % 128 == 0, "M tiles");
// Per N tile of NT sequences (32, or 128 for larger batches, so that W_O streams once per 128
// sequences): stages in flight, stage and shared-memory bytes.
template <int NT>
struct OpShape {
  static constexpr int kRing = NT <= 32 ? 4 : 3;
  static constexpr int kXBytes = kOpKS * NT * 2;
  static constexpr int kStageBytes = kOpWBytes + kXBytes;
  static constexpr int kSmemBytes = 1024 + kRing * kStageBytes + 256;
  static_assert(128 * (NT + 1) * 4 <= kRing * kStageBytes, "reduction tile fits in the operand ring");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// tmW: 3-D view of W_O [5120][16384] (64-column chunk, row, chunk index), box {64, 128, 2}.
// tmX: the same view of out [B][16384], box {64, NT, 2} (rows past B arrive as zeros).
template <int SPLIT, int NT>
__global__ void __launch_bounds__(kOpThreads, 1)
    out_proj_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                    __nv_bfloat16* __restrict__ y, int batch) {
  static_assert(SPLIT == 8 || SPLIT == 16, "cluster sizes");
  constexpr int KPER = kOpIn / SPLIT;       // contraction columns of one CTA
  constexpr int NST = KPER / kOpKS;         // its stages
  constexpr int R = 128 / SPLIT;            // tile rows each CTA reduces
  constexpr int JN = NT * R / 128;          // outputs per thread in the reduction
  using Sh = OpShape<NT>;
  constexpr int kOpRing = Sh::kRing;
  constexpr int kOpStageBytes = Sh::kStageBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOpRing * kOpStageBytes);
  uint64_t* empty = full + kOpRing;
  uint64_t* done = empty + kOpRing;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(smem);   // reuses the ring once the MMAs are done

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const int mt = blockIdx.y;
  const int n0 = blockIdx.z * NT;
  const int kc0 = rank * KPER / 64;   // first 64-column chunk of this CTA
  constexpr uint32_t kAccCols = NT;
  constexpr uint32_t kTmemCols = 2 * NT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kOpRing; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 2);   // one commit per issuing warp
    }
    mbar_init(done, 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    // The weight does not depend on earlier kernels: pull this CTA's share into L2 meanwhile.
    for (int q = 0; q < NST; ++q) tma_prefetch_l2_3d(&tmW, 0, 128 * mt, kc0 + q * (kOpKS / 64));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  pdl_trigger();
  pdl_wait();

  if (warp == 4 && lane == 0) {
    // ---------------- TMA producer
    int q = 0;
    for (; q < NST; ++q) {
      const int s = q % kOpRing;
      if (q >= kOpRing && !mbar_wait(&empty[s], static_cast<uint32_t>((q / kOpRing) - 1) & 1u)) {
        *abort_flag = 1;
        break;
      }
      uint8_t* sa = smem + s * kOpStageBytes;
      mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(kOpStageBytes));
      tma_load_3d(sa, &tmW, &full[s], 0, 128 * mt, kc0 + q * (kOpKS / 64));
      tma_load_3d(sa + kOpWBytes, &tmX, &full[s], 0, n0, kc0 + q * (kOpKS / 64));
    }
    // never leave (or let the ring be reused) while a copy is still landing
    for (int t = q > kOpRing ? q - kOpRing : 0; t < q; ++t)
      if (!mbar_wait(&full[t % kOpRing], static_cast<uint32_t>(t / kOpRing) & 1u)) *abort_flag = 1;
  } else if (warp >= 5 && lane == 0) {
    // ---------------- MMA issuers: warp 5 + j takes the 16-deep K steps with index % 2 == j
    const int j = warp - 5;
    const uint32_t acc = tmem_d + j * kAccCols;
    const uint32_t idesc = idesc_bf16_f32(128, NT, /*a_mn_major=*/false, /*b_mn_major=*/false);
    bool first = true;
    for (int q = 0; q < NST; ++q) {
      const int s = q % kOpRing;
      if (!mbar_wait(&full[s], static_cast<uint32_t>(q / kOpRing) & 1u)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + s * kOpStageBytes);
      const uint32_t sb = sa + kOpWBytes;
#pragma unroll
      for (int kk = j; kk < kOpKS / 16; kk += 2) {
        // A (K-major): chunk kk / 4 of 128 rows x 128 B; B (K-major): chunk kk / 4 of 32 rows x 128 B.
        const uint64_t adesc = sdesc_sw128(sa + (kk >> 2) * (128 * 128) + (kk & 3) * 32, 16, 1024);
        const uint64_t bdesc = sdesc_sw128(sb + (kk >> 2) * (NT * 128) + (kk & 3) * 32, 16, 1024);
        umma_bf16_ss(acc, adesc, bdesc, idesc, first ? 0u : 1u);
        first = false;
      }
      umma_commit(&empty[s]);
    }
    umma_commit(done);   // also fires when nothing was issued, so the epilogue never waits forever
  } else if (warp < 4) {
    // ---------------- epilogue part 1: this CTA's partial tile into its reduction tile red[m][n]
    const bool ok = mbar_wait(done, 0);
    tc_fence_after();
    const int m = warp * 32 + lane;
    const uint32_t trow = tmem_d + (static_cast<uint32_t>(warp * 32) << 16);
    uint32_t r0[16], r1[16];
#pragma unroll
    for (int c = 0; c < NT; c += 16) {
      tmem_ld16(trow + c, r0);
      tmem_ld16(trow + kAccCols + c, r1);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i)
        red[m * (NT + 1) + c + i] = ok ? __uint_as_float(r0[i]) + __uint_as_float(r1[i]) : 0.f;
    }
    if (!ok) *abort_flag = 1;
    // Cluster barrier 1 (each thread arrives once; warps 4-6 arrive below, after their roles).
    tc_fence_before();
    __syncwarp();
    cluster_arrive_release();
    cluster_wait_acquire();

    // ---------------- epilogue part 2: rows [R rank, R rank + R) of the cluster's sum
    const int t = threadIdx.x;
    const int mr = R * rank + (t % R);
    const uint32_t red_addr = smem_u32(red);
    int flags = 0;
    {
      float f[SPLIT];
#pragma unroll
      for (int q = 0; q < SPLIT; ++q) f[q] = ld_shared_cluster_f32(mapa_shared(smem_u32(abort_flag), q));
#pragma unroll
      for (int q = 0; q < SPLIT; ++q) flags |= __float_as_int(f[q]);
    }
    constexpr int kJC = JN < 4 ? JN : 4;   // outputs per batch of loads
#pragma unroll 1
    for (int j0 = 0; j0 < JN; j0 += kJC) {
      float part[kJC][SPLIT];   // a batch's loads all in flight at once, then the sums in rank order
#pragma unroll
      for (int jj = 0; jj < kJC; ++jj) {
        const int nl = t / R + (128 / R) * (j0 + jj);
        const uint32_t off = red_addr + 4u * static_cast<uint32_t>(mr * (NT + 1) + nl);
#pragma unroll
        for (int q = 0; q < SPLIT; ++q) part[jj][q] = ld_shared_cluster_f32(mapa_shared(off, q));
      }
#pragma unroll
      for (int jj = 0; jj < kJC; ++jj) {
        float sum = 0.f;
#pragma unroll
        for (int q = 0; q < SPLIT; ++q) sum += part[jj][q];
        const int n = n0 + t / R + (128 / R) * (j0 + jj);
        if (n < batch && flags == 0)
          y[static_cast<int64_t>(n) * kOpOut + 128 * mt + mr] = __float2bfloat16_rn(sum);
      }
    }
  }
  if (warp >= 4) {
    // producer and issuer warps (all lanes, reconverged): cluster barrier 1
    __syncwarp();
    tc_fence_before();
    cluster_arrive_release();
    cluster_wait_acquire();
  }
  cluster_sync();   // no CTA leaves while a peer may still read its reduction tile
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_d, kTmemCols);
  }
}

}  // namespace mla
