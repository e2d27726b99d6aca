// down_proj.cuh — fused down-projection + cache append on the tcgen05 tensor cores.
//
// What it computes (《DeepSeek-V2》深度解读报告 §2.2 Low-Rank Key-Value Joint Compression: the
// latent c^KV = W_D^KV h_t; §3.1: k^R is the shared 64-wide projection of h_t on the RoPE branch;
// §2.4: RoPE applies to that branch only; §3.3: model width d = 5120): for each new token i,
//     row_i = [ W_D^KV h_i (512) | RoPE(W^KR h_i, pos_i) (64) ]
// written to the cache slot of (seq_i, pos_i), exactly the row the cache append writes from a
// precomputed (c, k^R).  Products are exact in fp32, sums over the 5120 inputs in fp32; the latent
// is rounded once to bf16, the key rotated in fp64 from the fp32 sum and rounded once to bf16.
//
// B200 mapping.  The weights (576 x 5120 bf16, 5.9 MB) are the M operand ("swap-AB": M = output
// dims, N = tokens, K = d), so a small token count still fills M = 128 tiles:
//   * M tiles 0-3 are W_D^KV rows [128 t, 128 t + 128); M tile 4 is W^KR's 64 rows (a 64-row box
//     per stage; the MMA still computes 128 rows, and rows 64..127 of that tile, which read
//     whatever follows in shared memory, are never used);
//   * N tile = 32 tokens; K = 5120 is split over the SPLIT CTAs of a cluster (16 where the device
//     can place 16-CTA clusters, else 8): 5 stages of 5120 / (5 SPLIT) columns per CTA, all
//     streamed into shared memory at once, while two threads issue the MMAs into two TMEM
//     accumulators (even / odd 16-deep K steps);
//   * the SPLIT partial tiles are reduced through distributed shared memory: every CTA writes its
//     fp32 tile to its own shared memory, and after a cluster barrier CTA r sums rows
//     [R r, R r + R) (R = 128 / SPLIT) of all SPLIT tiles, applies RoPE (M tile 4) and writes its
//     part of each token's cache row.
// grid = (SPLIT, 5, ceil(n / 32)), clusters of SPLIT along x (set at launch); 224 threads: warps
// 0-3 epilogue and reduction, warp 4 TMA producer, warps 5-6 MMA issuers.
#pragma once

#include <cuda_bf16.h>

#include "append.cuh"
#include "ptx.cuh"

namespace mla {

constexpr int kDHidden = 5120;
constexpr int kDpStages = 5;                         // stages per CTA (each its own buffer)
constexpr int kDpNt = 32;                            // tokens per N tile
constexpr int kDpMTiles = 5;                         // 4 latent tiles + 1 RoPE-key tile
constexpr int kDpThreads = 224;
constexpr int kDpRedStride = kDpNt + 1;              // fp32 reduction tile [128][33] (padded)
template <int SPLIT>
struct DpShape {
  static constexpr int KS = kDHidden / SPLIT / kDpStages;   // contraction columns per stage
  static constexpr int kChunks = KS / 64;                   // 64-column (128-byte) chunks per stage
  static constexpr int kWBytes = KS * 128 * 2;              // weight stage: 128 rows x KS columns
  static constexpr int kHBytes = KS * kDpNt * 2;            // hidden stage: 32 tokens x KS columns
  static constexpr int kStageBytes = kWBytes + kHBytes;
  static constexpr int kSmemBytes = 1024 + kDpStages * kStageBytes + 256;
  static constexpr int kRows = 128 / SPLIT;                 // tile rows each CTA reduces
  static_assert(kDHidden % (SPLIT * kDpStages * 64) == 0, "K split");
  static_assert(128 * kDpRedStride * 4 <= kDpStages * kStageBytes, "reduction tile fits in the operand ring");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// Load from a cluster peer's shared memory.  volatile keeps it after the cluster barrier (another
// volatile asm); callers issue their loads into an array before using any, so they overlap.
__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t cluster_addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr));
  return v;
}

// tmW: 3-D view of W_D^KV [512][5120] (64-column chunk, row, chunk index), box {64, 128, chunks}.
// tmK: the same view of W^KR [64][5120], box {64, 64, chunks}.
// tmH: 3-D view of h [n][5120], box {64, 32, chunks} (rows past n arrive as zeros).
template <int SPLIT>
__global__ void __launch_bounds__(kDpThreads, 1)
    down_proj_append_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmH, const int32_t* __restrict__ seq_ids,
                            const int32_t* __restrict__ pos, __nv_bfloat16* cache, CacheView v, int n_tokens,
                            const RopeFreq rope) {
  using Sh = DpShape<SPLIT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kDpStages * Sh::kStageBytes);
  static_assert(SPLIT == 8 || SPLIT == 16, "cluster sizes");
  uint64_t* done = full + kDpStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(smem);   // reuses the operand ring once the MMAs are done

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const int mt = blockIdx.y;
  const int n0 = blockIdx.z * kDpNt;
  const int k0 = rank * (kDHidden / SPLIT);
  constexpr uint32_t kAccCols = kDpNt;   // 32 fp32 columns per accumulator
  constexpr uint32_t kTmemCols = 64;     // two accumulators

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDpStages; ++s) mbar_init(&full[s], 1);
    mbar_init(done, 2);   // one commit per issuing warp
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  const CUtensorMap* tmA = mt < 4 ? &tmW : &tmK;
  const int arow = mt < 4 ? 128 * mt : 0;
  const int arows = mt < 4 ? 128 : kDRope;           // weight rows a stage's box holds
  const uint32_t achunk = static_cast<uint32_t>(arows) * 128;   // bytes per 64-column chunk
  constexpr uint32_t kHChunk = kDpNt * 128;
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(tmA);
    tma_prefetch_desc(&tmH);
    // The weights do not depend on earlier kernels: pull this CTA's share into L2 meanwhile.
    for (int s = 0; s < kDpStages; ++s) tma_prefetch_l2_3d(tmA, 0, arow, (k0 + s * Sh::KS) / 64);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  pdl_trigger();
  pdl_wait();

  if (warp == 4 && lane == 0) {
    // ---------------- TMA producer: all stages at once (each has its own buffer)
    for (int s = 0; s < kDpStages; ++s) {
      uint8_t* sa = smem + s * Sh::kStageBytes;
      uint8_t* sb = sa + Sh::kWBytes;
      mbar_arrive_expect_tx(&full[s], Sh::kChunks * achunk + static_cast<uint32_t>(Sh::kHBytes));
      tma_load_3d(sa, tmA, &full[s], 0, arow, (k0 + s * Sh::KS) / 64);
      tma_load_3d(sb, &tmH, &full[s], 0, n0, (k0 + s * Sh::KS) / 64);
    }
    // never leave (or let the ring be reused) while a copy is still landing
    for (int s = 0; s < kDpStages; ++s)
      if (!mbar_wait(&full[s], 0)) *abort_flag = 1;
  } else if (warp >= 5 && lane == 0) {
    // ---------------- MMA issuers: warp 5 + j takes the 16-deep K steps with index % 2 == j
    const int j = warp - 5;
    const uint32_t acc = tmem_d + j * kAccCols;
    const uint32_t idesc = idesc_bf16_f32(128, kDpNt, /*a_mn_major=*/false, /*b_mn_major=*/false);
    bool first = true;
    for (int s = 0; s < kDpStages; ++s) {
      if (!mbar_wait(&full[s], 0)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + s * Sh::kStageBytes);
      const uint32_t sb = sa + Sh::kWBytes;
#pragma unroll
      for (int kk = j; kk < Sh::KS / 16; kk += 2) {
        // A (K-major): chunk kk / 4 of 128 rows x 128 B; B (K-major): chunk kk / 4 of 32 rows x 128 B;
        // 16 K elements = 32 B into each row.
        const uint64_t adesc = sdesc_sw128(sa + (kk >> 2) * achunk + (kk & 3) * 32, 16, 1024);
        const uint64_t bdesc = sdesc_sw128(sb + (kk >> 2) * kHChunk + (kk & 3) * 32, 16, 1024);
        umma_bf16_ss(acc, adesc, bdesc, idesc, first ? 0u : 1u);
        first = false;
      }
    }
    umma_commit(done);   // also fires when nothing was issued, so the epilogue never waits forever
  } else if (warp < 4) {
    // ---------------- epilogue part 1: the destination of every output this thread will write
    // (part 2 below), looked up while the copies and MMAs run; then this CTA's partial tile (both
    // accumulators summed) into its reduction tile red[m][n] (lane = m = output row of the tile).
    constexpr int R = Sh::kRows;
    constexpr int JN = kDpNt * R / 128;       // outputs per thread in part 2
    const int t = threadIdx.x;
    const int mr = R * rank + (t % R);        // the tile row this thread reduces in part 2
    const bool key = mt == 4;                 // the RoPE-key tile: rows 0..63 are k^R
    const bool valid_row = !key || mr < kDRope;
    int64_t dst[JN];                          // element index in the cache, or -1: nothing to write
    double cs[JN], sn[JN];
#pragma unroll
    for (int jn = 0; jn < JN; ++jn) {
      dst[jn] = -1;
      cs[jn] = 1.0;
      sn[jn] = 0.0;
      const int n = n0 + t / R + (128 / R) * jn;
      if (n >= n_tokens || !valid_row) continue;
      const int seq = seq_ids ? seq_ids[n] : n;
      const int p = pos[n];
      const int capacity = v.page_size == 0 ? v.max_seq_len : v.max_blocks * kPage;
      if (p < 0 || p >= capacity || seq < 0 || seq >= v.num_seqs) {
        if (t % R == 0) set_dev_error(0x1);
        continue;
      }
      const int64_t row = cache_row(v, seq, p);
      if (row < 0) continue;
      dst[jn] = row * kDRow + (key ? kDLat : 128 * mt) + mr;
      if (key) sincos(static_cast<double>(p) * rope.inv_freq[mr >> 1], &sn[jn], &cs[jn]);
    }
    const bool ok = mbar_wait(done, 0);
    tc_fence_after();
    const int m = warp * 32 + lane;
    const uint32_t trow = tmem_d + (static_cast<uint32_t>(warp * 32) << 16);
    uint32_t r0[16], r1[16];
#pragma unroll
    for (int c = 0; c < kDpNt; c += 16) {
      tmem_ld16(trow + c, r0);
      tmem_ld16(trow + kAccCols + c, r1);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i)
        red[m * kDpRedStride + c + i] = ok ? __uint_as_float(r0[i]) + __uint_as_float(r1[i]) : 0.f;
    }
    if (!ok) *abort_flag = 1;
    // Cluster barrier 1 (each thread arrives once; the producer and issuer warps arrive below,
    // after their roles): every CTA's partial tile is in its shared memory.
    tc_fence_before();
    __syncwarp();
    cluster_arrive_release();
    cluster_wait_acquire();

    // ---------------- epilogue part 2: rows [R rank, R rank + R) of the cluster's sum
    const uint32_t red_addr = smem_u32(red);
    // a failed wait in any CTA of the cluster leaves its partial tile incomplete: write nothing
    int flags = 0;
    {
      float f[SPLIT];
#pragma unroll
      for (int q = 0; q < SPLIT; ++q) f[q] = ld_shared_cluster_f32(mapa_shared(smem_u32(abort_flag), q));
#pragma unroll
      for (int q = 0; q < SPLIT; ++q) flags |= __float_as_int(f[q]);
    }
    const bool cluster_ok = flags == 0;
    float part[JN][SPLIT];   // all loads in flight at once, then the sums in rank order
#pragma unroll
    for (int jn = 0; jn < JN; ++jn) {
      const int nl = t / R + (128 / R) * jn;
      const uint32_t off = red_addr + 4u * static_cast<uint32_t>(mr * kDpRedStride + nl);
#pragma unroll
      for (int q = 0; q < SPLIT; ++q) part[jn][q] = ld_shared_cluster_f32(mapa_shared(off, q));
    }
#pragma unroll
    for (int jn = 0; jn < JN; ++jn) {
      float sum = 0.f;
#pragma unroll
      for (int q = 0; q < SPLIT; ++q) sum += part[jn][q];
      // partner row of the RoPE pair (rows 2i and 2i + 1 are lanes t and t ^ 1)
      const float partner = __shfl_xor_sync(0xffffffffu, sum, 1);
      if (dst[jn] < 0 || !cluster_ok) continue;
      __nv_bfloat16 outv;
      if (key) {
        // (x, y) = (row 2i, row 2i + 1) rotated by pos * theta_i in fp64, one rounding each
        const double x = (mr & 1) ? static_cast<double>(partner) : static_cast<double>(sum);
        const double y = (mr & 1) ? static_cast<double>(sum) : static_cast<double>(partner);
        outv = __double2bfloat16((mr & 1) ? x * sn[jn] + y * cs[jn] : x * cs[jn] - y * sn[jn]);
      } else {
        outv = __float2bfloat16_rn(sum);
      }
      cache[dst[jn]] = outv;
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
