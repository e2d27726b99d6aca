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
// One CTA computes a 128 x N tile of one head.  Its operands arrive in few, large TMA copies (each
// copy costs the CTA's TMA unit a roughly fixed time whatever its size): per stage of KS
// contraction rows, one 3-D box of the weight (KS rows x both 64-wide M chunks) and one 3-D box of
// the activation (N rows x KS/64 K slabs), 128-byte swizzled, into a ring of NSTAGE stages.  One
// thread issues tcgen05.mma into a TMEM accumulator; four warps read TMEM back and store bf16.
// The weight tile does not depend on earlier kernels, so it is prefetched into L2 before the
// kernel waits for its predecessor in the stream.
#pragma once

#include <cuda_bf16.h>

#include "append.cuh"
#include "ptx.cuh"

namespace mla {

constexpr int kGemmThreads = 224;    // warps 0-3: epilogue, warp 4: TMA producer, warps 5-6: MMA issuers
constexpr int kGemmIssuers = 2;      // MMA-issuing warps, each with its own accumulator (summed at the end)
constexpr int kGemmKS = 128;         // contraction rows per stage

// Stage bytes: weight KS x 128 MT (2 MT 64-wide M chunks) + activation nt x KS, bf16.
__host__ __device__ constexpr int gemm_stage_bytes(int nt, int mt = 1) { return kGemmKS * 256 * mt + nt * kGemmKS * 2; }

// New tokens' cache rows written by the query-side launch (cache == nullptr: none): the rows of
// mla_cache_append, row = [c_new[i] | RoPE(kr_new[i], pos[i])] at (seq_ids ? seq_ids[i] : i, pos[i]).
struct AppendJob {
  const uint4* c_new;              // [n_tokens, 512] bf16
  const __nv_bfloat162* kr_new;    // [n_tokens, 64] bf16, before RoPE
  const int32_t* seq_ids;          // [n_tokens] or null
  const int32_t* pos;              // [n_tokens]
  uint4* cache;
  CacheView v;
  int n_tokens;
};

// KTOT: contraction length (128 for absorption, 512 for un-absorption).
// tmA: 3-D view of the weight (64-element M chunk, contraction row = h * KTOT + k, M chunk index);
//      box {64, KS, 2}: smem [chunk][KS rows][128 B].
// tmB: 3-D view of the activation (64-element K slab, batch row, slab index = (h * KTOT + k) / 64);
//      box {64, nt, KS / 64}: smem [slab][nt rows][128 B].
// out element (n, h, m) is stored at out[n * out_bstride + h * out_hstride + m].
// Query side only (qpe != nullptr, KTOT = d_h): the epilogue warps also fill the RoPE part of the
// query rows, out[n, h, 512:576] = q_pe[n, h, :] rotated at q_pos[n] (or copied when q_pos is
// null), and write the new tokens' cache rows of `app` (if any), while the MMAs run: CTA c (linear
// index) takes work units c, c + #CTAs, ... (a unit is one new token's cache row and one group of
// heads of one query row).
// MT: 128-row M tiles per CTA.  MT = 1: the two issuing warps split the K steps into two
// accumulators (summed in the epilogue).  MT = 2: issuing warp j computes M tile j over all K
// steps; one CTA then loads the activation once for 256 output rows, and half as many CTAs with
// the same TMEM per CTA (2 nt columns) fit one wave where MT = 1 needs two.
// At most 72 registers a thread, so that four CTAs fit an SM.
template <int KTOT, int NSTAGE, int MT = 1>
__global__ void __launch_bounds__(kGemmThreads, 4)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     __nv_bfloat16* __restrict__ out, int batch, int nt, int64_t out_bstride,
                     int out_hstride, const uint4* __restrict__ qpe, const int32_t* __restrict__ q_pos,
                     const RopeFreq rope, const AppendJob app) {
  constexpr int KSTAGES = KTOT / kGemmKS;
  static_assert(KTOT % kGemmKS == 0, "contraction length");
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  static_assert(MT == 1 || MT == 2, "M tiles per CTA");
  const int stage_bytes = gemm_stage_bytes(nt, MT);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NSTAGE * stage_bytes);
  uint64_t* empty = full + NSTAGE;
  uint64_t* done = empty + NSTAGE;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128 * MT;
  const int h = blockIdx.y;
  const int n0 = blockIdx.z * nt;
  const uint32_t acc_cols = nt <= 32 ? 32u : (nt <= 64 ? 64u : (nt <= 128 ? 128u : 256u));
  const uint32_t tmem_cols = kGemmIssuers * acc_cols;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGemmIssuers);   // one commit per issuing warp
    }
    mbar_init(done, kGemmIssuers);
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
    for (int ks = 0; ks < KSTAGES; ++ks) tma_prefetch_l2_3d(&tmA, 0, h * KTOT + ks * kGemmKS, m0 / 64);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  // Setup above (and the weight prefetch) overlaps the previous kernel; nothing else global is
  // touched before this point.
  pdl_trigger();
  pdl_wait();

  if (warp == 4 && lane == 0) {
    // ---------------- TMA producer
    int armed[NSTAGE];
#pragma unroll
    for (int s = 0; s < NSTAGE; ++s) armed[s] = 0;
    for (int ks = 0; ks < KSTAGES; ++ks) {
      const int s = ks % NSTAGE;
      if (ks >= NSTAGE && !mbar_wait(&empty[s], ((ks / NSTAGE) - 1) & 1)) {
        *abort_flag = 1;
        break;
      }
      if (*reinterpret_cast<volatile int*>(abort_flag)) break;
      uint8_t* sa = smem + s * stage_bytes;
      uint8_t* sb = sa + kGemmKS * 256 * MT;
      mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(stage_bytes));
      const int krow = h * KTOT + ks * kGemmKS;
      tma_load_3d(sa, &tmA, &full[s], 0, krow, m0 / 64);
      tma_load_3d(sb, &tmB, &full[s], 0, n0, krow / 64);
      ++armed[s];
    }
    // Drain: never leave the CTA while one of its copies is still landing.
    for (int s = 0; s < NSTAGE; ++s)
      if (armed[s] > 0) mbar_wait(&full[s], (armed[s] - 1) & 1);
  } else if (warp >= 5 && lane == 0) {
    // ---------------- MMA issuers: warp 5 + j takes the 16-deep K steps g with g % 2 == j into
    // accumulator j (a single thread issues one MMA per ~125 cycles, so two halve the issue time)
    const int j = warp - 5;
    const uint32_t acc = tmem_d + j * acc_cols;
    const uint32_t idesc = idesc_bf16_f32(128, nt, /*a_mn_major=*/true, /*b_mn_major=*/false);
    bool ok = true, first = true;
    for (int ks = 0; ks < KSTAGES && ok; ++ks) {
      const int s = ks % NSTAGE;
      if (!mbar_wait(&full[s], (ks / NSTAGE) & 1)) {
        *abort_flag = 1;
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + s * stage_bytes);
      const uint32_t sb = sa + kGemmKS * 256 * MT;
      // MT = 1: this warp's K steps (kk = j, j + 2, ...); MT = 2: every K step of M tile j, whose
      // two 64-wide M chunks start 2 j chunks into the stage.
      const uint32_t sa_t = MT == 1 ? sa : sa + j * 2 * kGemmKS * 128;
      constexpr int kStep = MT == 1 ? kGemmIssuers : 1;
#pragma unroll
      for (int kk = (MT == 1 ? j : 0); kk < kGemmKS / 16; kk += kStep) {
        // A (MN-major): 16 K rows per MMA = 2 swizzle atoms of 1024 B; M chunks KS * 128 B apart.
        const uint64_t adesc = sdesc_sw128(sa_t + kk * 2048, kGemmKS * 128, 1024);
        // B (K-major): slab kk / 4 of nt rows x 128 B; 16 K elements = 32 B into each row.
        const uint64_t bdesc = sdesc_sw128(sb + (kk >> 2) * nt * 128 + (kk & 3) * 32, 16, 1024);
        umma_bf16_ss(acc, adesc, bdesc, idesc, first ? 0u : 1u);
        first = false;
      }
      umma_commit(&empty[s]);
    }
    umma_commit(done);  // also fires when nothing was issued, so the epilogue never waits forever
  } else if (warp < 4) {
    // ---------------- epilogue: TMEM -> registers -> bf16, staged through shared memory
    // Warp w owns outputs m0 + 32w + [0, 32) for every n of the tile.  Lane = m in TMEM, so the
    // warp's [n][32 m] block goes through a stage in the (now idle) operand ring: each lane writes
    // its column, then every global store instruction covers eight whole 64-byte rows.
    // Work units of the side jobs: unit u is new token u of the append job (u < app.n_tokens) and,
    // for the query rows, head group u % G of row u / G (G groups of 128 / G heads per row, G the
    // largest power of two <= min(16, #CTAs / batch), so a small batch still spreads its rows'
    // rotations over many CTAs).
    const int ncta = gridDim.x * gridDim.y * gridDim.z;
    int G = 1;
    if (qpe != nullptr && batch > 0)
      while (G < 16 && 2 * G * batch <= ncta) G *= 2;
    const int nunits = max(qpe != nullptr ? batch * G : 0, app.cache != nullptr ? app.n_tokens : 0);
    {
      // Angle and rotation in fp64, one rounding per output (the same arithmetic as the cache
      // append's RoPE).  cs_sn: a query row's 32 (cos, sin) pairs, formed by threads 0..31.
      double* cs_sn = reinterpret_cast<double*>(tmem_slot + 4);
      const int c = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
      for (int u = c; u < nunits; u += ncta) {
        if (app.cache != nullptr && u < app.n_tokens) {
          // new token u: threads 0..63 copy the latent (16 B each), 64..95 rotate one key pair each
          const int n = u;
          const int seq = app.seq_ids ? app.seq_ids[n] : n;
          const int p = app.pos[n];
          const int capacity = app.v.page_size == 0 ? app.v.max_seq_len : app.v.max_blocks * kPage;
          if (p < 0 || p >= capacity || seq < 0 || seq >= app.v.num_seqs) {
            if (threadIdx.x == 0) set_dev_error(0x1);
          } else if (threadIdx.x < 96) {
            const int64_t crow = cache_row(app.v, seq, p);
            if (crow >= 0) {
              const int t = threadIdx.x;
              if (t < 64) {
                app.cache[crow * (kDRow / 8) + t] = app.c_new[static_cast<int64_t>(n) * (kDLat / 8) + t];
              } else {
                const int pr = t - 64;
                double sn, cs;
                sincos(static_cast<double>(p) * rope.inv_freq[pr], &sn, &cs);
                reinterpret_cast<__nv_bfloat162*>(app.cache + crow * (kDRow / 8) + kDLat / 8)[pr] =
                    rope_pair(app.kr_new[static_cast<int64_t>(n) * (kDRope / 2) + pr], cs, sn);
              }
            }
          }
        }
        if (qpe == nullptr || u >= batch * G) continue;   // uniform across the 128 threads
        const int n = u / G;
        const int items = (kHeads / G) * (kDRope / 8);      // (head, 16-byte chunk) pairs of the group
        const int item0 = (u % G) * items;
        // The group's q_pe chunks are loaded (kChunk per thread at a time) before the angles are
        // formed, so the two latencies overlap.
        constexpr int kChunk = 4;
        for (int k0 = 0; k0 < items; k0 += 128 * kChunk) {
          uint4 r[kChunk];
#pragma unroll
          for (int k = 0; k < kChunk; ++k) {
            const int idx = k0 + threadIdx.x + 128 * k;
            if (idx < items) r[k] = qpe[static_cast<int64_t>(n) * kHeads * (kDRope / 8) + item0 + idx];
          }
          if (k0 == 0) {
            if (q_pos != nullptr && threadIdx.x < kDRope / 2) {
              double sn, cs;
              sincos(static_cast<double>(q_pos[n]) * rope.inv_freq[threadIdx.x], &sn, &cs);
              cs_sn[2 * threadIdx.x] = cs;
              cs_sn[2 * threadIdx.x + 1] = sn;
            }
            named_bar_sync(1, 128);
          }
#pragma unroll
          for (int k = 0; k < kChunk; ++k) {
            const int idx = k0 + threadIdx.x + 128 * k;
            if (idx >= items) continue;
            const int hh = (item0 + idx) >> 3;
            const int ch = (item0 + idx) & 7;
            if (q_pos != nullptr) {
              __nv_bfloat162* x = reinterpret_cast<__nv_bfloat162*>(&r[k]);
#pragma unroll
              for (int e = 0; e < 4; ++e) x[e] = rope_pair(x[e], cs_sn[2 * (4 * ch + e)], cs_sn[2 * (4 * ch + e) + 1]);
            }
            reinterpret_cast<uint4*>(out + static_cast<int64_t>(n) * out_bstride +
                                     static_cast<int64_t>(hh) * out_hstride)[kDLat / 8 + ch] = r[k];
          }
        }
        named_bar_sync(1, 128);   // the table is read before the next unit overwrites it
      }
    }
    const bool ok = mbar_wait(done, 0);
    tc_fence_after();
    if (ok && !*reinterpret_cast<volatile int*>(abort_flag)) {
      const uint32_t trow = tmem_d + (static_cast<uint32_t>(warp * 32) << 16);
      __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(smem + warp * nt * 64);
#pragma unroll 1
      for (int mtile = 0; mtile < MT; ++mtile) {
        if (mtile > 0) __syncwarp();   // the previous tile's stores have read the stage
        for (int c = 0; c < nt; c += 16) {
          uint32_t r0[16], r1[16];
          tmem_ld16(trow + (MT == 1 ? 0u : mtile * acc_cols) + c, r0);
          if (MT == 1) tmem_ld16(trow + acc_cols + c, r1);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            stage[(c + i) * 32 + lane] =
                __float2bfloat16_rn(MT == 1 ? __uint_as_float(r0[i]) + __uint_as_float(r1[i]) : __uint_as_float(r0[i]));
        }
        __syncwarp();
        const int q = lane & 3;   // 16-byte piece (8 outputs) of a 64-byte row
        for (int n8 = 0; n8 < nt; n8 += 8) {
          const int nl = n8 + (lane >> 2);
          const int n = n0 + nl;
          if (n < batch) {
            const uint4 v = *reinterpret_cast<const uint4*>(stage + nl * 32 + 8 * q);
            *reinterpret_cast<uint4*>(out + static_cast<int64_t>(n) * out_bstride +
                                      static_cast<int64_t>(h) * out_hstride + m0 + 128 * mtile + warp * 32 + 8 * q) = v;
          }
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
