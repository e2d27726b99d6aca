// decode_tc.cuh — split-KV MLA decode on the tcgen05 tensor cores, one CTA pair per
// (sequence, split).
//
// What it computes (《DeepSeek-V2》深度解读报告 §2.3 Absorption, §2.4 Decoupled RoPE): for every
// head h the score of cached token t is  s = scale * q_full[h] . row_t  over the 576-wide row
// [c (512) | RoPE(k^R) (64)] (content plus position channel), an online softmax over the split's
// tokens, and  O[h] = sum_t e^{s - m} c_t  over the 512-wide latent.  Every latent row is read from
// HBM once and shared by all 128 heads, which is what makes QK^T and PV dense contractions.
//
// B200 mapping.  The two CTAs of a cluster run "pair" MMAs (tcgen05 cta_group::2, M = 128): CTA r
// owns heads [64r, 64r+64) (its half of the A operand: Q for QK^T, P for PV) and each CTA's TMEM
// receives a 64-head slice of the accumulator folded over all 128 lanes, so
//   S tile (64 heads x 128 tokens, fp32)  = 64 TMEM columns per CTA (two buffers),
//   O      (64 heads x 512 latent, fp32)  = 256 TMEM columns per CTA.
// Per 128-token tile the B operand of QK^T is split by tokens (CTA r loads tokens [64r, 64r+64),
// all 576 dims, 9 slabs of 64 dims) and the B operand of PV is split by latent columns (CTA r
// loads latent [256n + 128r, +128) of all 128 tokens, 8 slabs of 32 tokens).  All slabs are 8 KB
// per CTA and stream through one ring of shared-memory stages filled by TMA (128-byte swizzle)
// in exactly the order the MMA issuer consumes them:  K(0) K(1) V(0) K(2) V(1) ... V(n-1).
//
// Warp roles (192 threads): warps 0-3 softmax / O correction / epilogue (thread = TMEM lane),
// warp 4 TMA producer, warp 5 TMEM allocation and (even CTA only) MMA issue.
//
// Masking.  Tokens >= the split end are excluded by setting their scores to -inf.  V rows of
// such tokens are zeroed in shared memory before PV (cache rows past a sequence's end may hold
// anything, and 0 * NaN would poison the sum); K rows need no fix because their scores are
// replaced, not scaled.
#pragma once

#include <cuda_bf16.h>

#include "decode_common.cuh"

namespace mla {

constexpr int kTcTile = 128;         // tokens per tile
constexpr int kTcStages = 14;        // 8 KB slabs in the ring
constexpr int kTcSlab = 8192;
constexpr int kTcQBytes = 9 * kTcSlab;
constexpr int kTcPBytes = 2 * kTcSlab;   // 64 heads x 128 tokens bf16, two 64-token K chunks
constexpr float kTcRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows > 2^8

constexpr int kTcOffQ = 0;
constexpr int kTcOffP = kTcOffQ + kTcQBytes;
constexpr int kTcOffRing = kTcOffP + 2 * kTcPBytes;
constexpr int kTcOffBar = kTcOffRing + kTcStages * kTcSlab;
constexpr int kTcOffMisc = kTcOffBar + 512;
constexpr int kTcSmemBytes = kTcOffMisc + 2048 + 1024;   // + slack for 1024-byte alignment

struct DecodeTcArgs {
  CacheView v;
  const int32_t* seq_lens;
  int S;               // splits per sequence
  float scale_log2;    // softmax_scale * log2(e)
  Workspace ws;
  __nv_bfloat16* out_lat;
  float* lse;
};

struct TcBars {
  uint64_t kv_full[kTcStages];   // even CTA only: both CTAs' slab halves landed
  uint64_t kv_empty[kTcStages];  // both CTAs: slab consumed by the MMAs
  uint64_t s_full[2];            // both: QK^T of a tile done
  uint64_t p_full[2];            // even CTA only: P (and corrected O) of a tile ready in both CTAs
  uint64_t p_empty[2];           // both: PV of a tile done reading P
  uint64_t o_ready;              // both: PV of a tile done writing O (one phase per tile)
  uint64_t o_final;              // both: the last PV done (single phase, read by the epilogue)
  uint64_t q_full;               // even CTA only: Q of both CTAs landed
  uint64_t fix;                  // per CTA: local loads of ragged V slabs
};
static_assert(sizeof(TcBars) <= 512, "barrier block");

// Row of (seq b, token t) for a TMA coordinate; -kTcTile (a fully out-of-bounds box, which the
// TMA unit fills with zeros) when the mapping is invalid.
__device__ __forceinline__ int tma_row(const CacheView& v, int b, int t) {
  const int64_t r = cache_row(v, b, t);
  return r < 0 ? -kTcTile : static_cast<int>(r);
}

__device__ __forceinline__ uint32_t lbar(const void* p) { return mapa_shared(smem_u32(p), 0); }

// ------------------------------------------------------------------------------ TMA producer
struct TcRing {
  int n = 0;  // slabs issued / consumed so far
  __device__ __forceinline__ int slot() const { return n % kTcStages; }
  __device__ __forceinline__ uint32_t round_parity() const { return static_cast<uint32_t>(n / kTcStages) & 1u; }
};

// Zero token rows [v, 32) of both 4 KB latent chunks of a V slab (rows are 128 bytes).
__device__ __forceinline__ void zero_v_rows(uint8_t* slab, int v) {
  for (int c = 0; c < 2; ++c)
    for (int row = v; row < 32; ++row) {
      uint4* p = reinterpret_cast<uint4*>(slab + c * 4096 + row * 128);
#pragma unroll
      for (int u = 0; u < 8; ++u) p[u] = make_uint4(0, 0, 0, 0);
    }
}

__device__ bool tc_producer(const CUtensorMap* tm_kc, const CUtensorMap* tm_vc, const CUtensorMap* tm_q,
                            const DecodeTcArgs& a, uint8_t* smem, TcBars* bars, uint32_t rank, int b,
                            int t_begin, int t_end, int n_tiles, volatile int* abort_flag) {
  const bool leader = rank == 0;
  // Q: 9 boxes of 64 dims x 64 heads.
  if (leader)
    mbar_arrive_expect_tx_addr(lbar(&bars->q_full), 2u * kTcQBytes);
  else
    mbar_arrive_addr(lbar(&bars->q_full));
  for (int c = 0; c < 9; ++c)
    tma_load_2d_pair(smem + kTcOffQ + c * kTcSlab, tm_q, lbar(&bars->q_full), 64 * c, b * kHeads + 64 * rank);

  TcRing ring;
  uint32_t fix_phase = 0;
  auto acquire = [&](int& s) -> bool {
    s = ring.slot();
    if (ring.n >= kTcStages && !mbar_wait(&bars->kv_empty[s], ring.round_parity() ^ 1u, 0x10)) return false;
    return !*abort_flag;
  };
  auto issue_k = [&](int i) -> bool {
    const int tile0 = t_begin + i * kTcTile;
    const int my0 = tile0 + 64 * static_cast<int>(rank);
    const int y = my0 < t_end ? tma_row(a.v, b, my0) : -kTcTile;
    for (int c = 0; c < 9; ++c) {
      int s;
      if (!acquire(s)) return false;
      if (leader) mbar_arrive_expect_tx_addr(lbar(&bars->kv_full[s]), 2u * kTcSlab);
      tma_load_2d_pair(smem + kTcOffRing + s * kTcSlab, tm_kc, lbar(&bars->kv_full[s]), 64 * c, y);
      mbar_arrive_addr(lbar(&bars->kv_full[s]));
      ++ring.n;
    }
    return true;
  };
  auto issue_v = [&](int i) -> bool {
    const int tile0 = t_begin + i * kTcTile;
    for (int nh = 0; nh < 2; ++nh)
      for (int kt = 0; kt < 4; ++kt) {
        int s;
        if (!acquire(s)) return false;
        uint8_t* slab = smem + kTcOffRing + s * kTcSlab;
        const int tok0 = tile0 + 32 * kt;
        const int vcount = min(max(t_end - tok0, 0), 32);
        const int x0 = 256 * nh + 128 * static_cast<int>(rank);
        if (vcount == 32) {
          const int y = tma_row(a.v, b, tok0);
          if (leader) mbar_arrive_expect_tx_addr(lbar(&bars->kv_full[s]), 2u * kTcSlab);
          tma_load_2d_pair(slab, tm_vc, lbar(&bars->kv_full[s]), x0, y);
          tma_load_2d_pair(slab + 4096, tm_vc, lbar(&bars->kv_full[s]), x0 + 64, y);
        } else {
          // Ragged: load locally, zero the rows past the end, then publish.
          if (leader) mbar_arrive_expect_tx_addr(lbar(&bars->kv_full[s]), 0u);
          if (vcount > 0) {
            const int y = tma_row(a.v, b, tok0);
            mbar_arrive_expect_tx(&bars->fix, 2u * 4096u);
            tma_load_2d(slab, tm_vc, &bars->fix, x0, y);
            tma_load_2d(slab + 4096, tm_vc, &bars->fix, x0 + 64, y);
            if (!mbar_wait(&bars->fix, fix_phase, 0x11)) return false;
            fix_phase ^= 1u;
          }
          zero_v_rows(slab, vcount);
          fence_proxy_async_smem();
        }
        mbar_arrive_addr(lbar(&bars->kv_full[s]));
        ++ring.n;
      }
    return true;
  };
  bool ok = issue_k(0);
  for (int i = 1; ok && i < n_tiles; ++i) ok = issue_k(i) && issue_v(i - 1);
  if (ok) ok = issue_v(n_tiles - 1);
  return ok;
}

// ------------------------------------------------------------------------------ MMA issuer (even CTA)
__device__ bool tc_mma(uint8_t* smem, TcBars* bars, uint32_t tmem, int n_tiles, volatile int* abort_flag) {
  const uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
  const uint32_t idesc_pv = idesc_bf16_f32(128, 256, false, true);
  const uint32_t sq = smem_u32(smem + kTcOffQ);
  const uint32_t sp = smem_u32(smem + kTcOffP);
  const uint32_t sr = smem_u32(smem + kTcOffRing);
  if (!mbar_wait_cluster(&bars->q_full, 0, 0x20)) return false;
  tc_fence_after();
  TcRing ring;
  auto qk = [&](int i) -> bool {
    const int j = i & 1;
    for (int c = 0; c < 9; ++c) {
      const int s = ring.slot();
      if (!mbar_wait_cluster(&bars->kv_full[s], ring.round_parity(), 0x21)) return false;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t ad = sdesc_sw128(sq + c * kTcSlab + 32 * k, 16, 1024);
        const uint64_t bd = sdesc_sw128(sr + s * kTcSlab + 32 * k, 16, 1024);
        umma_bf16_pair(tmem + 64 * j, ad, bd, idesc_qk, (c | k) != 0 ? 1u : 0u);
      }
      umma_commit_pair_mc(&bars->kv_empty[s], 3);
      ++ring.n;
    }
    umma_commit_pair_mc(&bars->s_full[j], 3);
    return true;
  };
  auto pv = [&](int i) -> bool {
    const int j = i & 1;
    if (!mbar_wait_cluster(&bars->p_full[j], static_cast<uint32_t>(i >> 1) & 1u, 0x22)) return false;
    tc_fence_after();
    for (int nh = 0; nh < 2; ++nh)
      for (int kt = 0; kt < 4; ++kt) {
        const int s = ring.slot();
        if (!mbar_wait_cluster(&bars->kv_full[s], ring.round_parity(), 0x23)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const int g = 2 * kt + kk;  // 16-token group within the tile
          const uint64_t ad = sdesc_sw128(sp + j * kTcPBytes + (g >> 2) * kTcSlab + 32 * (g & 3), 16, 1024);
          const uint64_t bd = sdesc_sw128(sr + s * kTcSlab + kk * 2048, 4096, 1024);
          umma_bf16_pair(tmem + 128 + 128 * nh, ad, bd, idesc_pv, (i > 0 || kt > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit_pair_mc(&bars->kv_empty[s], 3);
        ++ring.n;
      }
    umma_commit_pair_mc(&bars->p_empty[j], 3);
    umma_commit_pair_mc(&bars->o_ready, 3);
    return true;
  };
  bool ok = qk(0);
  for (int i = 1; ok && i < n_tiles; ++i) ok = qk(i) && pv(i - 1);
  if (ok) ok = pv(n_tiles - 1);
  // The epilogue cannot wait on o_ready by parity: when it starts, o_ready may still be two
  // phases short of the last one.  A dedicated single-phase barrier says "all PV done".
  umma_commit_pair_mc(&bars->o_final, 3);
  if (!ok) *abort_flag = 1;
  return ok;
}

// ------------------------------------------------------------------------------ softmax warps
// Thread t (0..127) owns TMEM lane t: head 64*rank + (t & 63); lanes 0-63 hold tokens [0,64) of a
// tile and latent columns 256n + [0,128) of O, lanes 64-127 tokens [64,128) and 256n + [128,256).
__device__ void tc_softmax(const DecodeTcArgs& a, uint8_t* smem, TcBars* bars, float* red, uint32_t tmem,
                           uint32_t rank, int b, int split, int t_begin, int t_end, int n_tiles, bool direct,
                           volatile int* abort_flag) {
  const int t = threadIdx.x;
  const int lane = t & 31;
  const int hl = t & 63;          // head within this CTA
  const int half = t >> 6;        // token half / latent quarter
  const uint32_t lane_base = static_cast<uint32_t>(32 * (t >> 5)) << 16;
  float m_used = -INFINITY;
  float l_run = 0.f;
  bool ok = true;
  for (int i = 0; i < n_tiles && ok; ++i) {
    const int j = i & 1;
    if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[j], static_cast<uint32_t>(i >> 1) & 1u, 0x30))) {
      ok = false;
      break;
    }
    tc_fence_after();
    float sc[64];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t r[16];
      tmem_ld16(tmem + lane_base + 64 * j + 16 * q, r);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 16; ++e) sc[16 * q + e] = __uint_as_float(r[e]);
    }
    const int tok0 = t_begin + i * kTcTile + 64 * half;
    const int nvalid = min(max(t_end - tok0, 0), 64);
    float mloc = -INFINITY;
#pragma unroll
    for (int e = 0; e < 64; ++e) {
      sc[e] = e < nvalid ? sc[e] * a.scale_log2 : -INFINITY;
      mloc = fmaxf(mloc, sc[e]);
    }
    red[j * 128 + t] = mloc;
    named_bar_sync(1, 128);
    const float m_tile = fmaxf(mloc, red[j * 128 + (t ^ 64)]);
    float alpha = 1.f;
    bool need = false;
    if (m_used == -INFINITY) {
      m_used = m_tile;
      alpha = 0.f;
    } else if (m_tile > m_used + kTcRescaleThreshold) {
      alpha = exp2f(m_used - m_tile);
      m_used = m_tile;
      need = true;
    }
    if (__any_sync(0xffffffffu, need)) {
      // O must hold PV(i-1) before it is scaled.  Waiting on phase i-1 by parity is unambiguous
      // here: s_full(i) was committed after PV(i-2), so o_ready is in phase i-1 or i.
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_ready, static_cast<uint32_t>(i - 1) & 1u, 0x31))) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int q = 0; q < 16; ++q) {
        uint32_t r[16];
        const uint32_t addr = tmem + lane_base + 128 + 16 * q;
        tmem_ld16(addr, r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
        tmem_st16(addr, r);
      }
      tmem_st_wait();
    }
    // P buffer j is free once PV(i-2) has read it.
    if (i >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bars->p_empty[j], static_cast<uint32_t>((i - 2) >> 1) & 1u, 0x32))) {
      ok = false;
      break;
    }
    float psum = 0.f;
    uint8_t* prow = smem + kTcOffP + j * kTcPBytes + half * kTcSlab + hl * 128;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      uint32_t pk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p0 = exp2f(sc[8 * u + 2 * e] - m_used);
        const float p1 = exp2f(sc[8 * u + 2 * e + 1] - m_used);
        psum += p0 + p1;
        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        pk[e] = *reinterpret_cast<uint32_t*>(&h2);
      }
      *reinterpret_cast<uint4*>(prow + ((u ^ (hl & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    l_run = l_run * alpha + psum;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_addr(lbar(&bars->p_full[j]));
  }
  // ---- epilogue
  if (ok && !__all_sync(0xffffffffu, mbar_wait(&bars->o_final, 0u, 0x33))) ok = false;
  tc_fence_after();
  red[256 + t] = l_run;
  named_bar_sync(1, 128);
  const float l_tot = l_run + red[256 + (t ^ 64)];
  if (!ok || *abort_flag) return;
  const int h = 64 * static_cast<int>(rank) + hl;
  const int64_t bh = static_cast<int64_t>(b) * kHeads + h;
  if (direct) {
    const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
    for (int nh = 0; nh < 2; ++nh) {
      __nv_bfloat16* dst = a.out_lat + bh * kDLat + 256 * nh + 128 * half;
      for (int q = 0; q < 8; ++q) {
        uint32_t r[16];
        tmem_ld16(tmem + lane_base + 128 + 128 * nh + 16 * q, r);
        tmem_ld_wait();
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[2 * e]) * inv, __uint_as_float(r[2 * e + 1]) * inv);
          pk[e] = *reinterpret_cast<uint32_t*>(&h2);
        }
        uint4* d4 = reinterpret_cast<uint4*>(dst + 16 * q);
        d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
    }
    if (half == 0 && a.lse != nullptr) a.lse[bh] = l_tot > 0.f ? (m_used + log2f(l_tot)) * kLn2 : -INFINITY;
  } else {
    const int64_t ml = (static_cast<int64_t>(b) * a.S + split) * kHeads + h;
    for (int nh = 0; nh < 2; ++nh) {
      float* dst = a.ws.o + ml * kDLat + 256 * nh + 128 * half;
      for (int q = 0; q < 8; ++q) {
        uint32_t r[16];
        tmem_ld16(tmem + lane_base + 128 + 128 * nh + 16 * q, r);
        tmem_ld_wait();
        float4* d4 = reinterpret_cast<float4*>(dst + 16 * q);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          d4[e] = make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]), __uint_as_float(r[4 * e + 2]),
                              __uint_as_float(r[4 * e + 3]));
      }
    }
    if (half == 0) {
      a.ws.m[ml] = m_used;
      a.ws.l[ml] = l_tot;
    }
  }
}

// ------------------------------------------------------------------------------ kernel
// grid = (2 * S, batch), clusters of 2 along x: blockIdx.x = 2 * split + rank.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc,
                     const __grid_constant__ CUtensorMap tm_q, const DecodeTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  TcBars* bars = reinterpret_cast<TcBars*>(smem + kTcOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kTcOffMisc);
  int* abort_flag = reinterpret_cast<int*>(smem + kTcOffMisc + 16);
  float* red = reinterpret_cast<float*>(smem + kTcOffMisc + 64);   // [2][128] maxima + [128] sums

  const uint32_t rank = cluster_ctarank();
  const int split = blockIdx.x >> 1;
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5;
  const int capacity = a.v.page_size == 0 ? a.v.max_seq_len : a.v.max_blocks * kPage;
  const int L = seq_len_checked(a.seq_lens, b, capacity);
  const int chunk = split_chunk(L, a.S, kSplitAlign);
  const int t_begin = split * chunk;
  if (L == 0 || t_begin >= L) return;  // both CTAs of the pair take this exit together
  const int t_end = min(L, t_begin + chunk);
  const int n_tiles = (t_end - t_begin + kTcTile - 1) / kTcTile;
  const bool direct = splits_used(L, a.S, kSplitAlign) == 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&bars->kv_full[s], 3);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(&bars->s_full[j], 1);
      mbar_init(&bars->p_full[j], 8);
      mbar_init(&bars->p_empty[j], 1);
    }
    mbar_init(&bars->o_ready, 1);
    mbar_init(&bars->o_final, 1);
    mbar_init(&bars->q_full, 2);
    mbar_init(&bars->fix, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  if (warp == 4 && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tm_kc);
    tma_prefetch_desc(&tm_vc);
    tma_prefetch_desc(&tm_q);
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    tc_softmax(a, smem, bars, red, tmem, rank, b, split, t_begin, t_end, n_tiles, direct, abort_flag);
  } else if (warp == 4) {
    if ((threadIdx.x & 31) == 0 &&
        !tc_producer(&tm_kc, &tm_vc, &tm_q, a, smem, bars, rank, b, t_begin, t_end, n_tiles, abort_flag))
      *abort_flag = 1;
  } else if (rank == 0 && (threadIdx.x & 31) == 0) {
    tc_mma(smem, bars, tmem, n_tiles, abort_flag);
  }
  __syncwarp();
  if (*reinterpret_cast<volatile int*>(abort_flag)) __nanosleep(200000);  // let stray copies land
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace mla
