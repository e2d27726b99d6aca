// out_proj.cuh — the attention block's output projection on the tcgen05 tensor cores.
//
// What it computes (《DeepSeek-V2》深度解读报告 §2.3 Absorption: W_U^V belongs with the output
// projection W_O; §3.3: model width d = 5120): for each sequence b,
//     y[b] = W_O [out[b, 0, :] | out[b, 1, :] | ... | out[b, 127, :]]      (5120 <- 16384)
// on the un-absorbed heads' outputs.  Products exact in fp32, sums over the 16384 inputs in fp32,
// one rounding of y to bf16.
//
// B200 mapping.  The weight (5120 x 16384 bf16, 168 MB) is the M operand ("swap-AB": M = output
// dims, N = sequences in tiles of NT = 32, or of 128 for batches above 32, K = 16384) and streams
// from HBM once per N tile.  Streaming it is the whole cost, so every SM streams an equal share in
// one wave: the work is 2560 units of R rows x 65536 / R columns (R = 256: 20 M tiles x 128 units;
// R = 128: 40 x 64), laid out M tile by M tile, and CTA c of G (one per SM) takes units
// [c U / G, (c + 1) U / G) (17 or 18 on 148 SMs), which cross at most one M-tile boundary, so a CTA
// accumulates at most two segments (two accumulators each, one per MMA-issuing warp, in TMEM).  Each segment's fp32 partial goes to a
// library-owned scratch buffer (so calls on different streams must not overlap), and a second
// kernel sums the partials of each M tile in CTA order (fp32, the same order every call) and
// rounds y to bf16.  (Clusters that reduce through distributed shared memory cannot give every SM
// an equal share: 8-CTA clusters ran 16 at a time, so 40 of them took three waves, the last on a
// fifth of the SMs.)
#pragma once

#include <cuda_bf16.h>

#include "down_proj.cuh"
#include "ptx.cuh"

namespace mla {

constexpr int kOpIn = kHeads * kDHead;   // 16384 inputs
constexpr int kOpOut = kDHidden;         // 5120 outputs
constexpr int kOpUnitElems = 256 * 128;  // W elements of a unit: R rows x (65536 / R) columns
constexpr int kOpUnits = kOpOut * kOpIn / kOpUnitElems;   // 2560
constexpr int kOpThreads = 224;          // warps 0-3 epilogue, warp 4 TMA producer, warps 5-6 MMA issuers
constexpr int kOpMaxCtas = 160;          // CTAs of the split kernel (one per SM)
constexpr int kOpMaxNt = 128;
constexpr int kOpMaxRows = 256;
constexpr int kOpMaxMTiles = kOpOut / 128;
// Scratch slots of [NT][256] fp32 partials: slot c for CTA c's first segment, kOpMaxCtas + k - 1
// for the segment of M tile k that a CTA starts after crossing the boundary into it.
constexpr int kOpSlots = kOpMaxCtas + kOpMaxMTiles - 1;
__device__ float g_op_partial[static_cast<size_t>(kOpSlots) * kOpMaxRows * kOpMaxNt];

// A unit is R rows (256: one 128-row half per MMA-issuing warp; 128: the warps split its K steps)
// by Z 64-column chunks (Z = 512 / R: every row of a unit's weight box is 128 Z contiguous bytes).
template <int NT, int R>
struct OpShape {
  static constexpr int Z = 512 / R;
  static constexpr int kMTiles = kOpOut / R;
  static constexpr int kUnitsPerTile = kOpIn / (64 * Z);
  static constexpr int kWBytes = R * Z * 128;
  static constexpr int kXBytes = NT * Z * 128;
  static constexpr int kStageBytes = kWBytes + kXBytes;
  static constexpr int kRing = (227 * 1024 - 2048) / kStageBytes < 4 ? (227 * 1024 - 2048) / kStageBytes : 4;
  static constexpr int kSmemBytes = 1024 + kRing * kStageBytes + 256;
  static_assert(R == 128 || R == 256, "unit rows");
  static_assert(kRing >= 2 && kSmemBytes <= 232448, "shared memory budget");
  static_assert(NT <= kOpMaxNt && 4 * NT <= 512, "TMEM: two segments x two accumulators of NT columns");
  static_assert(kMTiles * kUnitsPerTile == kOpUnits, "units");
};

// Units [u0, u1) of CTA c of G, and the scratch slot of segment `seg` (0 or 1) of M tile m.
__host__ __device__ __forceinline__ int op_unit0(int c, int G) { return c * kOpUnits / G; }
__device__ __forceinline__ int op_slot(int c, int seg, int m) { return seg == 0 ? c : kOpMaxCtas + m - 1; }
// The CTA whose units hold unit u: the last c with op_unit0(c) <= u, i.e. ceil((u + 1) G / U) - 1.
__device__ __forceinline__ int op_cta_of(int u, int G) { return ((u + 1) * G + kOpUnits - 1) / kOpUnits - 1; }

// tmW: 3-D view of W_O [5120][16384] (64-column chunk, row, chunk index), box {64, R, Z}.
// tmX: the same view of out [B][16384], box {64, NT, Z} (rows past B arrive as zeros).
// grid = G (kOpUnits / G <= units per M tile, G <= kOpMaxCtas), one CTA per SM; N tile of
// sequences [n0, n0 + NT).
template <int NT, int R>
__global__ void __launch_bounds__(kOpThreads, 1)
    out_proj_split_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, int n0) {
  using Sh = OpShape<NT, R>;
  constexpr int kRing = Sh::kRing;
  constexpr int kStage = Sh::kStageBytes;
  constexpr int Z = Sh::Z;
  constexpr int kStages = Sh::kUnitsPerTile;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRing * kStage);
  uint64_t* empty = full + kRing;
  uint64_t* seg_done = empty + kRing;   // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(seg_done + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int c = blockIdx.x;
  const int u0 = op_unit0(c, G), u1 = op_unit0(c + 1, G);
  const int m_first = u0 / kStages;
  const int n_seg = (u1 > u0) ? (u1 - 1) / kStages - m_first + 1 : 0;
  constexpr uint32_t kTmemCols = 4 * NT < 32 ? 32 : 4 * NT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 2);   // one commit per issuing warp
    }
    mbar_init(&seg_done[0], 2);
    mbar_init(&seg_done[1], 2);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    // The weight does not depend on earlier kernels: pull this CTA's first units into L2 meanwhile.
    for (int u = u0; u < u1 && u < u0 + 8; ++u) tma_prefetch_l2_3d(&tmW, 0, R * (u / kStages), (u % kStages) * Z);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  pdl_trigger();
  pdl_wait();   // the activation, and the scratch (read by the previous call's sum kernel)

  if (warp == 4 && lane == 0) {
    // ---------------- TMA producer
    int q = 0;
    for (; q < u1 - u0; ++q) {
      const int s = q % kRing;
      if (q >= kRing && !mbar_wait(&empty[s], static_cast<uint32_t>((q / kRing) - 1) & 1u)) break;
      const int u = u0 + q;
      uint8_t* sa = smem + s * kStage;
      mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(kStage));
      tma_load_3d(sa, &tmW, &full[s], 0, R * (u / kStages), (u % kStages) * Z);
      tma_load_3d(sa + Sh::kWBytes, &tmX, &full[s], 0, n0, (u % kStages) * Z);
    }
    // never leave while a copy is still landing
    for (int t = q > kRing ? q - kRing : 0; t < q; ++t) mbar_wait(&full[t % kRing], static_cast<uint32_t>(t / kRing) & 1u);
  } else if (warp >= 5 && lane == 0) {
    // ---------------- MMA issuers, warp 5 + j: R = 256, rows [128 j, 128 j + 128) of each unit over
    // all its K steps; R = 128, the K steps of parity j.  Each into its own accumulator of the segment.
    const int j = warp - 5;
    const uint32_t idesc = idesc_bf16_f32(128, NT, /*a_mn_major=*/false, /*b_mn_major=*/false);
    constexpr int kSteps = 4 * Z;                    // 16-deep K steps of a unit
    constexpr int kStep = R == 256 ? 1 : 2;
    for (int q = 0; q < u1 - u0; ++q) {
      const int s = q % kRing;
      const int u = u0 + q;
      const int seg = u / kStages - m_first;
      const bool seg_start = q == 0 || u % kStages == 0;
      if (!mbar_wait(&full[s], static_cast<uint32_t>(q / kRing) & 1u)) break;
      tc_fence_after();
      const uint32_t acc = tmem_d + static_cast<uint32_t>((2 * seg + j) * NT);
      const uint32_t sa = smem_u32(smem + s * kStage) + (R == 256 ? j * (128 * 128) : 0);
      const uint32_t sb = smem_u32(smem + s * kStage) + Sh::kWBytes;
#pragma unroll
      for (int kk = (R == 256 ? 0 : j); kk < kSteps; kk += kStep) {
        // A (K-major): chunk kk / 4 of R rows x 128 B; B (K-major): chunk kk / 4 of NT rows x
        // 128 B.  16 K elements = 32 B into each row.
        const uint64_t adesc = sdesc_sw128(sa + (kk >> 2) * (R * 128) + (kk & 3) * 32, 16, 1024);
        const uint64_t bdesc = sdesc_sw128(sb + (kk >> 2) * (NT * 128) + (kk & 3) * 32, 16, 1024);
        umma_bf16_ss(acc, adesc, bdesc, idesc, (seg_start && kk == (R == 256 ? 0 : j)) ? 0u : 1u);
      }
      umma_commit(&empty[s]);
      if (u % kStages == kStages - 1 || q == u1 - u0 - 1) umma_commit(&seg_done[seg]);
    }
  } else if (warp < 4) {
    // ---------------- epilogue: each segment's partial [NT][256] fp32 to its scratch slot (for a
    // given n the 32 lanes' rows are contiguous: one 128-byte store per warp and n)
    for (int seg = 0; seg < n_seg; ++seg) {
      const bool ok = mbar_wait(&seg_done[seg], 0);
      tc_fence_after();
      const int m = m_first + seg;
      float* dst = g_op_partial + static_cast<size_t>(op_slot(c, seg, m)) * kOpMaxRows * kOpMaxNt;
      const uint32_t trow = tmem_d + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(2 * seg * NT);
      if constexpr (R == 256) {
#pragma unroll 1
        for (int j = 0; j < 2; ++j) {
          const int r = 128 * j + 32 * warp + lane;
#pragma unroll 1
          for (int cc = 0; cc < NT; cc += 16) {
            uint32_t v[16];
            tmem_ld16(trow + static_cast<uint32_t>(j * NT + cc), v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) dst[(cc + i) * R + r] = ok ? __uint_as_float(v[i]) : 0.f;
          }
        }
      } else {
        const int r = 32 * warp + lane;   // the two accumulators hold the same rows: their sum
#pragma unroll 1
        for (int cc = 0; cc < NT; cc += 16) {
          uint32_t v0[16], v1[16];
          tmem_ld16(trow + static_cast<uint32_t>(cc), v0);
          tmem_ld16(trow + static_cast<uint32_t>(NT + cc), v1);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            dst[(cc + i) * R + r] = ok ? __uint_as_float(v0[i]) + __uint_as_float(v1[i]) : 0.f;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_d, kTmemCols);
  }
}

// Sum of the partials of M tile blockIdx.x for sequence n0 + blockIdx.y: thread r takes row r (R
// threads); the CTAs whose runs hold units of the tile (at most kOpSumMaxCtas) are summed in CTA
// order, their loads all in flight at once.
constexpr int kOpSumMaxCtas = 16;
template <int NT, int R>
__global__ void __launch_bounds__(R) out_proj_sum_kernel(__nv_bfloat16* __restrict__ y, int batch, int n0, int G) {
  pdl_trigger();
  pdl_wait();
  constexpr int kStages = OpShape<NT, R>::kUnitsPerTile;
  const int m = blockIdx.x;
  const int n = blockIdx.y;
  const int r = threadIdx.x;
  if (n0 + n >= batch) return;
  const int c_lo = op_cta_of(m * kStages, G), c_hi = op_cta_of(m * kStages + kStages - 1, G);
  float v[kOpSumMaxCtas];
#pragma unroll
  for (int i = 0; i < kOpSumMaxCtas; ++i) {
    const int c = c_lo + i;
    v[i] = 0.f;
    if (c <= c_hi) {
      const int seg = m - op_unit0(c, G) / kStages;
      v[i] = g_op_partial[static_cast<size_t>(op_slot(c, seg, m)) * kOpMaxRows * kOpMaxNt + n * R + r];
    }
  }
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < kOpSumMaxCtas; ++i) sum += v[i];   // ascending CTA order; the zeros past c_hi add nothing
  y[static_cast<int64_t>(n0 + n) * kOpOut + R * m + r] = __float2bfloat16_rn(sum);
}

}  // namespace mla
