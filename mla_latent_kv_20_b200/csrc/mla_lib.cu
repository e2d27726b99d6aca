// mla_lib.cu — the C ABI declared in include/mla.h: host-side validation, TMA descriptor
// construction and kernel launches.  Single translation unit (the kernels are header-only), so
// the device error word needs no relocatable device code.
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "../../include/mla.h"
#include "append.cuh"
#include "decode_common.cuh"
#include "decode_tc.cuh"
#include "down_proj.cuh"
#include "out_proj.cuh"
#include "gemm_tc.cuh"
#include "ptx.cuh"

namespace {

using mla::CacheView;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Launch with programmatic stream serialisation: the kernel may be scheduled while the previous
// kernel on the stream still runs; it waits for that kernel (griddepcontrol.wait) before it
// touches global memory, so ordering against earlier work on the stream is unchanged.
template <typename... KArgs, typename... Args>
mla_status launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Generic 3-D bf16 view (dims[0] must be 64 elements = one 128-byte swizzle row), 128-byte swizzle.
bool make_map_3d(CUtensorMap* map, const void* base, const cuuint64_t (&dims)[3], const cuuint64_t (&strides)[2],
                 const cuuint32_t (&box)[3]) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Validates a cache descriptor; on success fills the kernel-side view.
mla_status check_cache(const mla_cache_desc& d, const void* cache, const int32_t* block_table, CacheView* v) {
  if (cache == nullptr || !aligned16(cache)) return MLA_ERR_INVALID_ARG;
  if (d.num_seqs <= 0 || d.num_rows <= 0) return MLA_ERR_INVALID_ARG;
  if (d.page_size == 0) {
    if (block_table != nullptr || d.max_seq_len <= 0) return MLA_ERR_INVALID_ARG;
    if (static_cast<int64_t>(d.num_seqs) * d.max_seq_len > d.num_rows) return MLA_ERR_INVALID_ARG;
  } else if (d.page_size == MLA_PAGE_SIZE) {
    if (block_table == nullptr || d.max_blocks_per_seq <= 0 || (d.num_rows % MLA_PAGE_SIZE) != 0)
      return MLA_ERR_INVALID_ARG;
    if (d.max_blocks_per_seq > INT_MAX / MLA_PAGE_SIZE) return MLA_ERR_UNSUPPORTED;
  } else {
    return MLA_ERR_UNSUPPORTED;
  }
  if (d.num_rows > (int64_t(1) << 40)) return MLA_ERR_UNSUPPORTED;
  v->page_size = d.page_size;
  v->max_seq_len = d.max_seq_len;
  v->max_blocks = d.max_blocks_per_seq;
  v->num_rows = d.num_rows;
  v->block_table = block_table;
  v->num_seqs = d.num_seqs;
  return MLA_OK;
}

inline int cache_capacity(const mla_cache_desc& d) {
  return d.page_size == 0 ? d.max_seq_len : d.max_blocks_per_seq * MLA_PAGE_SIZE;
}

constexpr int kMaxBatch = 65536;

}  // namespace

#include "decode_launch.cuh"

namespace mla {
// Self-test of the bounded wait: one thread waits on a barrier nothing arrives on, which must give
// up after limit_ns (setting the wait-timeout error with site 0x7F) and return normally.
__global__ void selftest_wait_kernel(uint64_t limit_ns, int32_t* result) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer_ns();
    const bool completed = mbar_wait_for(&bar, 0, 0x7F, limit_ns);
    result[0] = completed ? 1 : 0;
    result[1] = static_cast<int32_t>((globaltimer_ns() - t0) / 1000);
  }
}
}  // namespace mla

extern "C" {

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_DEVICE: return "MLA_ERR_DEVICE";
  }
  return "MLA_ERR_UNKNOWN";
}

int32_t mla_version(void) { return 100; }

mla_status mla_get_device_error(int32_t* code) {
  if (code == nullptr) return MLA_ERR_INVALID_ARG;
  *code = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return MLA_ERR_CUDA;
  int v = 0, site = 0;
  if (cudaMemcpyFromSymbol(&v, mla::g_mla_dev_error, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&site, mla::g_mla_dev_error_site, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(mla::g_mla_dev_error, &zero, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaMemcpyToSymbol(mla::g_mla_dev_error_site, &zero, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  *code = v | ((site & 0xFF) << 8);
  return MLA_OK;
}

}  // extern "C"

namespace {

// base^(-2i/d_R) for the 32 rotation pairs, in fp64 (the angle pos * inv_freq is formed in fp64 on
// the device).
mla::RopeFreq rope_freq(float rope_base) {
  mla::RopeFreq f;
  for (int i = 0; i < mla::kDRope / 2; ++i)
    f.inv_freq[i] = std::pow(static_cast<double>(rope_base), -2.0 * i / static_cast<double>(mla::kDRope));
  return f;
}

// The output projection for one tile size NT: per N tile of NT sequences, the split kernel (one
// CTA per SM, each an equal share of W_O) and the kernel that sums its partials.
template <int NT, int R>
mla_status launch_output_proj(const mla_bf16* out, const mla_bf16* w_o, mla_bf16* y, int32_t batch, void* stream) {
  using Sh = mla::OpShape<NT, R>;
  CUtensorMap tw, tx;
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(mla::kOpIn) * 2, 128};
  const cuuint64_t dw[3] = {64, static_cast<cuuint64_t>(mla::kOpOut), mla::kOpIn / 64};
  const cuuint64_t dx[3] = {64, static_cast<cuuint64_t>(batch), mla::kOpIn / 64};
  const cuuint32_t bw[3] = {64, static_cast<cuuint32_t>(R), static_cast<cuuint32_t>(Sh::Z)};
  const cuuint32_t bx[3] = {64, static_cast<cuuint32_t>(NT), static_cast<cuuint32_t>(Sh::Z)};
  if (!make_map_3d(&tw, w_o, dw, strides, bw) || !make_map_3d(&tx, out, dx, strides, bx)) return MLA_ERR_CUDA;
  auto split = mla::out_proj_split_kernel<NT, R>;
  if (cudaFuncSetAttribute(split, cudaFuncAttributeMaxDynamicSharedMemorySize, Sh::kSmemBytes) != cudaSuccess)
    return MLA_ERR_CUDA;
  // one CTA per SM; a CTA's run of units must fit in one M tile's units (at most one boundary)
  const int G = std::max(mla::kOpUnits / Sh::kUnitsPerTile, std::min(mla::kOpMaxCtas, device_sm_count()));
  cudaStream_t s = as_stream(stream);
  for (int n0 = 0; n0 < batch; n0 += NT) {
    mla_status st = launch_chained(split, dim3(G), dim3(mla::kOpThreads), static_cast<size_t>(Sh::kSmemBytes), s, tw,
                                   tx, n0);
    if (st != MLA_OK) return st;
    static_assert(Sh::kUnitsPerTile * mla::kOpMaxCtas / mla::kOpUnits + 2 <= mla::kOpSumMaxCtas, "CTAs per M tile");
    st = launch_chained(mla::out_proj_sum_kernel<NT, R>, dim3(Sh::kMTiles, NT), dim3(R), 0, s,
                        reinterpret_cast<__nv_bfloat16*>(y), batch, n0, G);
    if (st != MLA_OK) return st;
  }
  return MLA_OK;
}

// The down-projection + append for one tile size NT: per N tile of NT tokens, the split kernel
// (each CTA an equal share of the weights' 200 units) and the kernel that sums the partials,
// rotates the keys and writes the cache rows.
template <int NT>
mla_status launch_project_append(const mla_bf16* h, const mla_bf16* w_dkv, const mla_bf16* w_kr,
                                 const int32_t* seq_ids, const int32_t* pos, mla_bf16* cache, const CacheView& v,
                                 int32_t n_tokens, float rope_base, void* stream) {
  using Sh = mla::DpShape<NT>;
  // 3-D views (64-column chunk, row, chunk index) of the row-major [rows][5120] matrices.
  CUtensorMap tw, tk, th;
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(mla::kDHidden) * 2, 128};
  const cuuint64_t dw[3] = {64, static_cast<cuuint64_t>(mla::kDLat), mla::kDHidden / 64};
  const cuuint64_t dk[3] = {64, static_cast<cuuint64_t>(mla::kDRope), mla::kDHidden / 64};
  const cuuint64_t dh[3] = {64, static_cast<cuuint64_t>(n_tokens), mla::kDHidden / 64};
  const cuuint32_t bw[3] = {64, 128, static_cast<cuuint32_t>(mla::kDpKS / 64)};
  const cuuint32_t bk[3] = {64, static_cast<cuuint32_t>(mla::kDRope), static_cast<cuuint32_t>(mla::kDpKS / 64)};
  const cuuint32_t bh[3] = {64, static_cast<cuuint32_t>(NT), static_cast<cuuint32_t>(mla::kDpKS / 64)};
  if (!make_map_3d(&tw, w_dkv, dw, strides, bw) || !make_map_3d(&tk, w_kr, dk, strides, bk) ||
      !make_map_3d(&th, h, dh, strides, bh))
    return MLA_ERR_CUDA;
  auto split = mla::dp_split_kernel<NT>;
  if (cudaFuncSetAttribute(split, cudaFuncAttributeMaxDynamicSharedMemorySize, Sh::kSmemBytes) != cudaSuccess)
    return MLA_ERR_CUDA;
  const int G = std::max(mla::kDpMTiles, std::min(mla::kDpMaxCtas, device_sm_count()));
  cudaStream_t s = as_stream(stream);
  const mla::RopeFreq rope = rope_freq(rope_base);
  for (int n0 = 0; n0 < n_tokens; n0 += NT) {
    mla_status st = launch_chained(split, dim3(G), dim3(mla::kDpThreads), static_cast<size_t>(Sh::kSmemBytes), s, tw,
                                   tk, th, n0);
    if (st != MLA_OK) return st;
    st = launch_chained(mla::dp_sum_kernel<NT>, dim3(mla::kDpMTiles, NT), dim3(128), 0, s, seq_ids, pos,
                        reinterpret_cast<__nv_bfloat16*>(cache), v, n_tokens, rope, n0, G);
    if (st != MLA_OK) return st;
  }
  return MLA_OK;
}

}  // namespace

extern "C" {

mla_status mla_cache_append(const mla_bf16* c_new, const mla_bf16* kr_new, const int32_t* seq_ids,
                            const int32_t* pos, mla_bf16* cache, const int32_t* block_table,
                            mla_cache_desc desc, int32_t n_tokens, float rope_base, void* stream) {
  if (n_tokens < 0 || !(rope_base > 0.f) || !std::isfinite(rope_base)) return MLA_ERR_INVALID_ARG;
  CacheView v;
  const mla_status st = check_cache(desc, cache, block_table, &v);
  if (st != MLA_OK) return st;
  if (n_tokens == 0) return MLA_OK;
  if (c_new == nullptr || kr_new == nullptr || pos == nullptr || !aligned16(c_new) || !aligned16(kr_new))
    return MLA_ERR_INVALID_ARG;
  if (seq_ids == nullptr && n_tokens > desc.num_seqs) return MLA_ERR_INVALID_ARG;
  if (n_tokens > INT_MAX / 2) return MLA_ERR_UNSUPPORTED;
  return launch_chained(mla::cache_append_kernel, dim3(n_tokens), dim3(96), 0, as_stream(stream),
                        reinterpret_cast<const uint4*>(c_new), reinterpret_cast<const __nv_bfloat162*>(kr_new),
                        seq_ids, pos, reinterpret_cast<uint4*>(cache), v, rope_freq(rope_base));
}

mla_status mla_cache_append_fp8(const mla_bf16* c_new, const mla_bf16* kr_new, const int32_t* seq_ids,
                                const int32_t* pos, uint8_t* cache, uint8_t* scales, const int32_t* block_table,
                                mla_cache_desc desc, int32_t n_tokens, float rope_base, void* stream) {
  if (n_tokens < 0 || !(rope_base > 0.f) || !std::isfinite(rope_base)) return MLA_ERR_INVALID_ARG;
  CacheView v;
  const mla_status st = check_cache(desc, cache, block_table, &v);
  if (st != MLA_OK) return st;
  if (n_tokens == 0) return MLA_OK;
  if (scales == nullptr) return MLA_ERR_INVALID_ARG;
  if (c_new == nullptr || kr_new == nullptr || pos == nullptr || !aligned16(c_new) || !aligned16(kr_new))
    return MLA_ERR_INVALID_ARG;
  if (seq_ids == nullptr && n_tokens > desc.num_seqs) return MLA_ERR_INVALID_ARG;
  if (n_tokens > INT_MAX / 2) return MLA_ERR_UNSUPPORTED;
  return launch_chained(mla::cache_append_fp8_kernel, dim3(n_tokens), dim3(96), 0, as_stream(stream),
                        reinterpret_cast<const uint4*>(c_new), reinterpret_cast<const __nv_bfloat162*>(kr_new),
                        seq_ids, pos, cache, scales, v, rope_freq(rope_base));
}

mla_status mla_project_append(const mla_bf16* h, const mla_bf16* w_dkv, const mla_bf16* w_kr,
                              const int32_t* seq_ids, const int32_t* pos, mla_bf16* cache,
                              const int32_t* block_table, mla_cache_desc desc, int32_t n_tokens, float rope_base,
                              void* stream) {
  if (n_tokens < 0 || !(rope_base > 0.f) || !std::isfinite(rope_base)) return MLA_ERR_INVALID_ARG;
  CacheView v;
  const mla_status st = check_cache(desc, cache, block_table, &v);
  if (st != MLA_OK) return st;
  if (n_tokens == 0) return MLA_OK;
  if (h == nullptr || w_dkv == nullptr || w_kr == nullptr || pos == nullptr) return MLA_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(w_dkv) || !aligned16(w_kr)) return MLA_ERR_INVALID_ARG;
  if (seq_ids == nullptr && n_tokens > desc.num_seqs) return MLA_ERR_INVALID_ARG;
  if (n_tokens > kMaxBatch) return MLA_ERR_UNSUPPORTED;
  // Tiles of 32 tokens up to 32, else of 128 (the weights then stream once per 128 tokens).
  if (n_tokens <= 32) return launch_project_append<32>(h, w_dkv, w_kr, seq_ids, pos, cache, v, n_tokens, rope_base, stream);
  return launch_project_append<128>(h, w_dkv, w_kr, seq_ids, pos, cache, v, n_tokens, rope_base, stream);
}

mla_status mla_selftest_wait_timeout(uint32_t limit_us, int32_t* result, void* stream) {
  if (result == nullptr || limit_us == 0 || limit_us > 2000000u) return MLA_ERR_INVALID_ARG;
  mla::selftest_wait_kernel<<<1, 32, 0, as_stream(stream)>>>(static_cast<uint64_t>(limit_us) * 1000ull, result);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status mla_output_proj(const mla_bf16* out, const mla_bf16* w_o, mla_bf16* y, int32_t batch, void* stream) {
  if (batch < 0 || batch > kMaxBatch) return batch < 0 ? MLA_ERR_INVALID_ARG : MLA_ERR_UNSUPPORTED;
  if (batch == 0) return MLA_OK;
  if (out == nullptr || w_o == nullptr || y == nullptr) return MLA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(w_o) || !aligned16(y)) return MLA_ERR_INVALID_ARG;
  // Tiles of 32 sequences up to 32, else of 128 (W_O then streams once per 128 sequences).  Units
  // of 128 rows x 512 columns for the small tile (512 contiguous bytes per weight row and box:
  // 46 vs 48 us at one sequence, 63 vs 69 us at 32), of 256 x 256 for the large one, whose
  // activation box then stays half the weight box.
  if (batch <= 32) return launch_output_proj<32, 128>(out, w_o, y, batch, stream);
  return launch_output_proj<128, 256>(out, w_o, y, batch, stream);
}

}  // extern "C"

namespace {

template <int KTOT, int NSTAGE, int MT = 1>
mla_status launch_proj_gemm(const void* weight, int m_total, const void* act, int batch, __nv_bfloat16* out,
                            int64_t out_bstride, int out_hstride, cudaStream_t stream, const void* qpe = nullptr,
                            const int32_t* q_pos = nullptr, float rope_base = 10000.f,
                            const mla::AppendJob* app = nullptr, int nt_cap = 256) {
  // Weight viewed as [heads * KTOT rows][m_total cols]: 3-D (64-element M chunk, row, M chunk index),
  // box {64, KS, 2}.  Activation as [batch rows][heads * KTOT cols]: 3-D (64-element K slab, batch
  // row, slab index), box {64, nt, KS / 64}.
  const int nt = std::min(batch >= 256 ? 256 : ((batch + 15) / 16) * 16, nt_cap);
  const uint64_t krows = static_cast<uint64_t>(mla::kHeads) * KTOT;
  CUtensorMap ta, tb;
  {
    const cuuint64_t dims[3] = {64, krows, static_cast<cuuint64_t>(m_total / 64)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(m_total) * 2, 128};
    const cuuint32_t box[3] = {64, mla::kGemmKS, 2 * MT};
    if (!make_map_3d(&ta, weight, dims, strides, box)) return MLA_ERR_CUDA;
  }
  {
    const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(batch), krows / 64};
    const cuuint64_t strides[2] = {krows * 2, 128};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(nt), mla::kGemmKS / 64};
    if (!make_map_3d(&tb, act, dims, strides, box)) return MLA_ERR_CUDA;
  }
  // ring, barriers, TMEM slot and flag, then the 32 (cos, sin) pairs of the q_pe rotation
  const size_t smem = 1024 + NSTAGE * mla::gemm_stage_bytes(nt, MT) + (2 * NSTAGE + 1) * 8 + 16 + 32 * 16;
  auto kern = mla::proj_gemm_kernel<KTOT, NSTAGE, MT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return MLA_ERR_CUDA;
  dim3 grid(m_total / (128 * MT), mla::kHeads, (batch + nt - 1) / nt);
  return launch_chained(kern, grid, dim3(mla::kGemmThreads), smem, stream, ta, tb, out, batch, nt, out_bstride,
                        out_hstride, reinterpret_cast<const uint4*>(qpe), q_pos, rope_freq(rope_base),
                        app != nullptr ? *app : mla::AppendJob{nullptr, nullptr, nullptr, nullptr, nullptr, {}, 0});
}

// The W_UK GEMM of the query absorption (optionally with the cache append of `app`): two 128-row M
// tiles per CTA for batches of 65..128 rows (256 CTAs in one wave where 512 of one tile took two:
// 16.2 -> 14.8 us at 128 rows, weights cold), one otherwise (at 64 rows and below two tiles per
// CTA measured no faster).
mla_status launch_absorb(const mla_bf16* w_uk, const mla_bf16* q_nope, int batch, mla_bf16* q_full, cudaStream_t s,
                         const mla_bf16* q_pe, const int32_t* q_pos, float rope_base, const mla::AppendJob* app) {
  auto* qf = reinterpret_cast<__nv_bfloat16*>(q_full);
  const int64_t bstride = static_cast<int64_t>(mla::kHeads) * mla::kDRow;
  if (batch > 64 && batch <= 128)
    return launch_proj_gemm<mla::kDHead, 1, 2>(w_uk, mla::kDLat, q_nope, batch, qf, bstride, mla::kDRow, s, q_pe, q_pos,
                                               rope_base, app);
  return launch_proj_gemm<mla::kDHead, 1, 1>(w_uk, mla::kDLat, q_nope, batch, qf, bstride, mla::kDRow, s, q_pe, q_pos,
                                             rope_base, app);
}

}  // namespace

extern "C" {

mla_status mla_absorb_q(const mla_bf16* q_nope, const mla_bf16* q_pe, const int32_t* q_pos,
                        const mla_bf16* w_uk, mla_bf16* q_full, int32_t batch, float rope_base,
                        void* stream) {
  if (batch < 0 || batch > kMaxBatch) return batch < 0 ? MLA_ERR_INVALID_ARG : MLA_ERR_UNSUPPORTED;
  if (batch == 0) return MLA_OK;
  if (q_nope == nullptr || q_pe == nullptr || w_uk == nullptr || q_full == nullptr) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_nope) || !aligned16(q_pe) || !aligned16(w_uk) || !aligned16(q_full)) return MLA_ERR_INVALID_ARG;
  if (q_pos != nullptr && (!(rope_base > 0.f) || !std::isfinite(rope_base))) return MLA_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  // One launch: the W_UK GEMM fills q_full[:, :, 0:512] and its CTAs rotate q_pe into
  // q_full[:, :, 512:576] meanwhile.
  return launch_absorb(w_uk, q_nope, batch, q_full, s, q_pe, q_pos, rope_base, nullptr);
}

mla_status mla_append_absorb(const mla_bf16* c_new, const mla_bf16* kr_new, const int32_t* seq_ids,
                             const int32_t* pos, mla_bf16* cache, const int32_t* block_table, mla_cache_desc desc,
                             int32_t n_tokens, const mla_bf16* q_nope, const mla_bf16* q_pe, const int32_t* q_pos,
                             const mla_bf16* w_uk, mla_bf16* q_full, int32_t batch, float rope_base, void* stream) {
  // the checks of mla_cache_append ...
  if (n_tokens < 0 || !(rope_base > 0.f) || !std::isfinite(rope_base)) return MLA_ERR_INVALID_ARG;
  CacheView v;
  const mla_status st = check_cache(desc, cache, block_table, &v);
  if (st != MLA_OK) return st;
  if (n_tokens > 0) {
    if (c_new == nullptr || kr_new == nullptr || pos == nullptr || !aligned16(c_new) || !aligned16(kr_new))
      return MLA_ERR_INVALID_ARG;
    if (seq_ids == nullptr && n_tokens > desc.num_seqs) return MLA_ERR_INVALID_ARG;
    if (n_tokens > kMaxBatch) return MLA_ERR_UNSUPPORTED;
  }
  // ... and of mla_absorb_q
  if (batch < 0 || batch > kMaxBatch) return batch < 0 ? MLA_ERR_INVALID_ARG : MLA_ERR_UNSUPPORTED;
  if (batch == 0) return n_tokens == 0 ? MLA_OK : mla_cache_append(c_new, kr_new, seq_ids, pos, cache, block_table,
                                                                    desc, n_tokens, rope_base, stream);
  if (q_nope == nullptr || q_pe == nullptr || w_uk == nullptr || q_full == nullptr) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_nope) || !aligned16(q_pe) || !aligned16(w_uk) || !aligned16(q_full)) return MLA_ERR_INVALID_ARG;
  const mla::AppendJob app{reinterpret_cast<const uint4*>(c_new), reinterpret_cast<const __nv_bfloat162*>(kr_new),
                           seq_ids, pos, reinterpret_cast<uint4*>(cache), v, n_tokens};
  return launch_absorb(w_uk, q_nope, batch, q_full, as_stream(stream), q_pe, q_pos, rope_base, &app);
}

mla_status mla_unabsorb_v(const mla_bf16* out_lat, const mla_bf16* w_uv, mla_bf16* out, int32_t batch,
                          void* stream) {
  if (batch < 0 || batch > kMaxBatch) return batch < 0 ? MLA_ERR_INVALID_ARG : MLA_ERR_UNSUPPORTED;
  if (batch == 0) return MLA_OK;
  if (out_lat == nullptr || w_uv == nullptr || out == nullptr) return MLA_ERR_INVALID_ARG;
  if (!aligned16(out_lat) || !aligned16(w_uv) || !aligned16(out)) return MLA_ERR_INVALID_ARG;
  // One CTA per head streams that head's 128 KB of W_UV in four 128-row stages: with a batch of up
  // to 64 rows all four stages fit in shared memory and are requested at once (one HBM round trip);
  // larger batches (larger stages) go through a two-stage ring.  (Two 64-row N tiles per head for
  // batches of 65..128 rows, 256 CTAs, measured no faster.)
  if (batch <= 64)
    return launch_proj_gemm<mla::kDLat, 4>(w_uv, mla::kDHead, out_lat, batch, reinterpret_cast<__nv_bfloat16*>(out),
                                           static_cast<int64_t>(mla::kHeads) * mla::kDHead, mla::kDHead,
                                           as_stream(stream));
  return launch_proj_gemm<mla::kDLat, 2>(w_uv, mla::kDHead, out_lat, batch, reinterpret_cast<__nv_bfloat16*>(out),
                                         static_cast<int64_t>(mla::kHeads) * mla::kDHead, mla::kDHead,
                                         as_stream(stream));
}


}  // extern "C"


extern "C" {

mla_status mla_decode_attn(const mla_bf16* q_full, const mla_bf16* cache, const int32_t* block_table,
                           const int32_t* seq_lens, mla_cache_desc desc, int32_t batch, float softmax_scale,
                           int32_t num_splits, void* workspace, size_t workspace_bytes, mla_bf16* out_lat,
                           float* lse, void* stream) {
  return launch_attn(q_full, cache, block_table, seq_lens, nullptr, desc, batch, softmax_scale, num_splits, workspace,
                     workspace_bytes, out_lat, lse, stream);
}

mla_status mla_decode_attn_fp8(const mla_bf16* q_full, const uint8_t* cache, const uint8_t* scales,
                               const int32_t* block_table, const int32_t* seq_lens, mla_cache_desc desc,
                               int32_t batch, float softmax_scale, int32_t num_splits, void* workspace,
                               size_t workspace_bytes, mla_bf16* out_lat, float* lse, void* stream) {
  if (scales == nullptr) return MLA_ERR_INVALID_ARG;
  return launch_attn(q_full, cache, block_table, seq_lens, nullptr, desc, batch, softmax_scale, num_splits, workspace,
                     workspace_bytes, out_lat, lse, stream, scales);
}

mla_status mla_prefill_attn(const mla_bf16* q_full, const mla_bf16* cache, const int32_t* block_table,
                            const int32_t* q_seq, const int32_t* q_len, mla_cache_desc desc, int32_t n_queries,
                            float softmax_scale, int32_t num_splits, void* workspace, size_t workspace_bytes,
                            mla_bf16* out_lat, float* lse, void* stream) {
  if (n_queries > 0 && q_seq == nullptr) return MLA_ERR_INVALID_ARG;
  return launch_attn(q_full, cache, block_table, q_len, q_seq, desc, n_queries, softmax_scale, num_splits, workspace,
                     workspace_bytes, out_lat, lse, stream);
}

}  // extern "C"

// ------------------------------------------------------------------------------------------
// Decode without caller memory: split partials in a library-owned static device buffer.
// ------------------------------------------------------------------------------------------
namespace {

// One buffer per context: a __device__ array exists once in every CUDA context that loads the
// library (the primary context of each device, and any context a host engine creates and makes
// current).  Host code must not pass the array's host-side symbol to a kernel: its device address
// is looked up with cudaGetSymbolAddress, with the calling thread's context current, on every call.
// The lookup allocates nothing and costs about a microsecond of host time; caching it per device
// would hand a stale address to a call made under another context of the same device, or after
// the device was reset and its context re-created.
__device__ __align__(256) unsigned char g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

mla_status noalloc_scratch(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MLA_ERR_CUDA;
  *out = p;
  return MLA_OK;
}

}  // namespace

extern "C" mla_status mla_decode_attn_noalloc(const mla_bf16* q_full, const mla_bf16* cache,
                                              const int32_t* block_table, const int32_t* seq_lens,
                                              mla_cache_desc desc, int32_t batch, float softmax_scale,
                                              int32_t num_splits, mla_bf16* out_lat, float* lse, void* stream) {
  if (batch < 0 || num_splits < 0) return MLA_ERR_INVALID_ARG;
  if (batch == 0) return MLA_OK;
  const int capacity = desc.page_size == 0 ? desc.max_seq_len : desc.max_blocks_per_seq * MLA_PAGE_SIZE;
  if (capacity <= 0) return MLA_ERR_INVALID_ARG;
  if (mla_decode_workspace_size(batch, capacity, num_splits) > MLA_NOALLOC_SCRATCH_BYTES) return MLA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const mla_status st = noalloc_scratch(&scratch);
  if (st != MLA_OK) return st;
  return mla_decode_attn(q_full, cache, block_table, seq_lens, desc, batch, softmax_scale, num_splits, scratch,
                         MLA_NOALLOC_SCRATCH_BYTES, out_lat, lse, stream);
}

extern "C" size_t mla_noalloc_scratch_bytes(void) { return MLA_NOALLOC_SCRATCH_BYTES; }
