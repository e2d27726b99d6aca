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
// dims, N = tokens in tiles of NT = 32, or 128 above 32 tokens, K = d), so a small token count still
// fills M = 128 tiles: M tiles 0-3 are W_D^KV rows [128 t, 128 t + 128); M tile 4 is W^KR's 64 rows
// (a 64-row box per unit; the MMA still computes 128 rows, and rows 64..127 of that tile, which read
// whatever lies past the box in shared memory, are never used).  The work is 5 M tiles x 40 units
// of 128 contraction columns, laid out M tile by M tile, and CTA c of G takes units
// [c U / G, (c + 1) U / G) (two each on 100 CTAs), through a 2-stage TMA ring, with two threads
// issuing the MMAs into two TMEM accumulators (even / odd 16-deep K steps) per segment (the part of
// one M tile a CTA holds; at most two).  Each segment's fp32 partial goes to a library-owned scratch
// buffer (so calls on different streams must not overlap), and a second kernel sums each row's
// partials in CTA order, rotates the key rows (fp64, one rounding) and writes the cache rows.  (The
// previous layout, K split over 16-CTA clusters reduced through distributed shared memory, ran its
// clusters in waves; at 0.05 of HBM the call is latency, not bandwidth.)
#pragma once

#include <cuda_bf16.h>

#include "append.cuh"
#include "ptx.cuh"

namespace mla {

constexpr int kDHidden = 5120;
constexpr int kDpMTiles = 5;                         // 4 latent tiles + 1 RoPE-key tile
constexpr int kDpThreads = 224;                      // warps 0-3 epilogue, warp 4 TMA producer, warps 5-6 MMA issuers
constexpr int kDpKS = 128;                           // contraction columns per unit
constexpr int kDpKUnits = kDHidden / kDpKS;          // 40 units per M tile
constexpr int kDpUnits = kDpMTiles * kDpKUnits;      // 200
constexpr int kDpMaxCtas = 100;                      // CTAs of the split kernel
constexpr int kDpMaxNt = 128;
constexpr int kDpSlots = kDpMaxCtas + kDpMTiles - 1;
constexpr int kDpSumMaxCtas = kDpKUnits * kDpMaxCtas / kDpUnits + 2;   // CTAs holding units of one M tile
static_assert(kDpUnits / kDpMaxCtas <= kDpKUnits, "a CTA's run crosses at most one M-tile boundary");
// Scratch slots of [NT][128] fp32 partials: slot c for CTA c's first segment, kDpMaxCtas + k - 1 for
// the segment of M tile k that a CTA starts after crossing into it.
__device__ float g_dp_partial[static_cast<size_t>(kDpSlots) * 128 * kDpMaxNt];

template <int NT>
struct DpShape {
  static constexpr int kWBytes = 128 * kDpKS * 2;     // weight box: 128 rows (64 for W^KR) x 128 columns
  static constexpr int kHBytes = NT * kDpKS * 2;      // hidden box: NT tokens x 128 columns
  static constexpr int kStageBytes = kWBytes + kHBytes;
  static constexpr int kRing = 2;
  static constexpr int kSmemBytes = 1024 + kRing * kStageBytes + 256;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(NT <= kDpMaxNt && 4 * NT <= 512, "TMEM: two segments x two accumulators");
};

__host__ __device__ __forceinline__ int dp_unit0(int c, int G) { return c * kDpUnits / G; }
__device__ __forceinline__ int dp_slot(int c, int seg, int m) { return seg == 0 ? c : kDpMaxCtas + m - 1; }
__device__ __forceinline__ int dp_cta_of(int u, int G) { return ((u + 1) * G + kDpUnits - 1) / kDpUnits - 1; }

// tmW: 3-D view of W_D^KV [512][5120] (64-column chunk, row, chunk index), box {64, 128, 2}.
// tmK: the same view of W^KR [64][5120], box {64, 64, 2}.
// tmH: 3-D view of h [n][5120], box {64, NT, 2} (rows past n arrive as zeros).
// grid = G (<= kDpMaxCtas), tokens [n0, n0 + NT).
template <int NT>
__global__ void __launch_bounds__(kDpThreads, 1)
    dp_split_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmH, int n0) {
  using Sh = DpShape<NT>;
  constexpr int kRing = Sh::kRing;
  constexpr int kStage = Sh::kStageBytes;
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
  const int u0 = dp_unit0(c, G), u1 = dp_unit0(c + 1, G);
  const int m_first = u0 / kDpKUnits;
  const int n_seg = (u1 > u0) ? (u1 - 1) / kDpKUnits - m_first + 1 : 0;
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
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmH);
    // The weights do not depend on earlier kernels: pull this CTA's share into L2 meanwhile.
    for (int u = u0; u < u1 && u < u0 + 4; ++u) {
      const int m = u / kDpKUnits;
      tma_prefetch_l2_3d(m < 4 ? &tmW : &tmK, 0, m < 4 ? 128 * m : 0, (u % kDpKUnits) * (kDpKS / 64));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  pdl_trigger();
  pdl_wait();   // h, and the scratch (read by the previous call's sum kernel)

  if (warp == 4 && lane == 0) {
    // ---------------- TMA producer
    int q = 0;
    for (; q < u1 - u0; ++q) {
      const int s = q % kRing;
      if (q >= kRing && !mbar_wait(&empty[s], static_cast<uint32_t>((q / kRing) - 1) & 1u)) break;
      const int u = u0 + q;
      const int m = u / kDpKUnits;
      const int kc = (u % kDpKUnits) * (kDpKS / 64);
      uint8_t* sa = smem + s * kStage;
      const uint32_t wbytes = m < 4 ? Sh::kWBytes : Sh::kWBytes / 2;
      mbar_arrive_expect_tx(&full[s], wbytes + static_cast<uint32_t>(Sh::kHBytes));
      tma_load_3d(sa, m < 4 ? &tmW : &tmK, &full[s], 0, m < 4 ? 128 * m : 0, kc);
      tma_load_3d(sa + Sh::kWBytes, &tmH, &full[s], 0, n0, kc);
    }
    for (int t = q > kRing ? q - kRing : 0; t < q; ++t) mbar_wait(&full[t % kRing], static_cast<uint32_t>(t / kRing) & 1u);
  } else if (warp >= 5 && lane == 0) {
    // ---------------- MMA issuers: warp 5 + j takes the 16-deep K steps of parity j of each unit
    const int j = warp - 5;
    const uint32_t idesc = idesc_bf16_f32(128, NT, /*a_mn_major=*/false, /*b_mn_major=*/false);
    for (int q = 0; q < u1 - u0; ++q) {
      const int s = q % kRing;
      const int u = u0 + q;
      const int m = u / kDpKUnits;
      const int seg = m - m_first;
      const bool seg_start = q == 0 || u % kDpKUnits == 0;
      if (!mbar_wait(&full[s], static_cast<uint32_t>(q / kRing) & 1u)) break;
      tc_fence_after();
      const uint32_t acc = tmem_d + static_cast<uint32_t>((2 * seg + j) * NT);
      const uint32_t sa = smem_u32(smem + s * kStage);
      const uint32_t sb = sa + Sh::kWBytes;
      const uint32_t achunk = (m < 4 ? 128u : 64u) * 128u;   // bytes per 64-column chunk of the weight box
#pragma unroll
      for (int kk = j; kk < kDpKS / 16; kk += 2) {
        const uint64_t adesc = sdesc_sw128(sa + (kk >> 2) * achunk + (kk & 3) * 32, 16, 1024);
        const uint64_t bdesc = sdesc_sw128(sb + (kk >> 2) * (NT * 128) + (kk & 3) * 32, 16, 1024);
        umma_bf16_ss(acc, adesc, bdesc, idesc, (seg_start && kk == j) ? 0u : 1u);
      }
      umma_commit(&empty[s]);
      if (u % kDpKUnits == kDpKUnits - 1 || q == u1 - u0 - 1) umma_commit(&seg_done[seg]);
    }
  } else if (warp < 4) {
    // ---------------- epilogue: each segment's partial (both accumulators summed), [NT][128] fp32
    for (int seg = 0; seg < n_seg; ++seg) {
      const bool ok = mbar_wait(&seg_done[seg], 0);
      tc_fence_after();
      const int m = m_first + seg;
      float* dst = g_dp_partial + static_cast<size_t>(dp_slot(c, seg, m)) * 128 * kDpMaxNt;
      const uint32_t trow = tmem_d + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(2 * seg * NT);
      const int r = 32 * warp + lane;
#pragma unroll 1
      for (int cc = 0; cc < NT; cc += 16) {
        uint32_t v0[16], v1[16];
        tmem_ld16(trow + static_cast<uint32_t>(cc), v0);
        tmem_ld16(trow + static_cast<uint32_t>(NT + cc), v1);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[(cc + i) * 128 + r] = ok ? __uint_as_float(v0[i]) + __uint_as_float(v1[i]) : 0.f;
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

// Token n0 + blockIdx.y, M tile blockIdx.x: thread r sums row r's partials in CTA order (loads all
// in flight at once), then writes the latent (M tiles 0-3) or the rotated key (tile 4, rows 0-63:
// pair (2i, 2i + 1) in lanes r and r ^ 1, rotated by pos * theta_i in fp64, one rounding each) into
// the token's cache row.
template <int NT>
__global__ void __launch_bounds__(128)
    dp_sum_kernel(const int32_t* __restrict__ seq_ids, const int32_t* __restrict__ pos, __nv_bfloat16* cache,
                  CacheView v, int n_tokens, const RopeFreq rope, int n0, int G) {
  pdl_trigger();
  pdl_wait();
  const int m = blockIdx.x;
  const int nl = blockIdx.y;
  const int n = n0 + nl;
  const int r = threadIdx.x;
  if (n >= n_tokens) return;
  const int c_lo = dp_cta_of(m * kDpKUnits, G), c_hi = dp_cta_of(m * kDpKUnits + kDpKUnits - 1, G);
  float part[kDpSumMaxCtas];
#pragma unroll
  for (int i = 0; i < kDpSumMaxCtas; ++i) {
    const int c = c_lo + i;
    part[i] = 0.f;
    if (c <= c_hi) {
      const int seg = m - dp_unit0(c, G) / kDpKUnits;
      part[i] = g_dp_partial[static_cast<size_t>(dp_slot(c, seg, m)) * 128 * kDpMaxNt + nl * 128 + r];
    }
  }
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < kDpSumMaxCtas; ++i) sum += part[i];   // ascending CTA order; the zeros add nothing
  const float partner = __shfl_xor_sync(0xffffffffu, sum, 1);
  const int seq = seq_ids ? seq_ids[n] : n;
  const int p = pos[n];
  const int capacity = v.page_size == 0 ? v.max_seq_len : v.max_blocks * kPage;
  if (p < 0 || p >= capacity || seq < 0 || seq >= v.num_seqs) {
    if (m == 0 && r == 0) set_dev_error(0x1);
    return;
  }
  const int64_t row = cache_row(v, seq, p);
  if (row < 0) return;
  if (m < 4) {
    cache[row * kDRow + 128 * m + r] = __float2bfloat16_rn(sum);
  } else if (r < kDRope) {
    double sn, cs;
    sincos(static_cast<double>(p) * rope.inv_freq[r >> 1], &sn, &cs);
    const double x = (r & 1) ? static_cast<double>(partner) : static_cast<double>(sum);
    const double y = (r & 1) ? static_cast<double>(sum) : static_cast<double>(partner);
    cache[row * kDRow + kDLat + r] = __double2bfloat16((r & 1) ? x * sn + y * cs : x * cs - y * sn);
  }
}

}  // namespace mla
