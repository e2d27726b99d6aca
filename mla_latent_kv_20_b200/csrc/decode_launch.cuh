// decode_launch.cuh — host side of the decode call (included by mla_lib.cu, after its helpers):
// the tensor maps of the cache and query boxes, the number of work ranges, and the launch of the
// decode kernel and its combine.  The bench keys its recorded DRAM traffic of the decode call to the
// sources of this file and of the decode kernel.
#pragma once

namespace {

// 3-D bf16 view of [rows][576] as (64-element dim-slab, row, slab index) for boxes of
// 64 elements x 64 rows x box_slabs slabs, 128-byte swizzle: one box fills box_slabs consecutive
// 8 KB slabs of 64 rows x 128 bytes.
bool make_map_slabs(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_slabs) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {64, rows, 9};
  const cuuint64_t strides[2] = {mla::kDRow * 2, 128};
  const cuuint32_t box[3] = {64, 64, box_slabs};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 4-D bf16 view of [rows][576] as (64-element chunk, row, chunk index, latent half) for boxes of
// 64 elements x 64 rows x 2 chunks x 2 halves (32 KB), 128-byte swizzle: the PV operand of one CTA
// for 64 tokens, laid out [half][chunk][row][128 B].
bool make_map_vbox(CUtensorMap* map, const void* base, uint64_t rows) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[4] = {64, rows, 4, 2};
  const cuuint64_t strides[3] = {mla::kDRow * 2, 128, 512};
  const cuuint32_t box[4] = {64, 64, 2, 2};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Byte views of an FP8 cache (E4M3 codes, rows of 576 bytes) with the same box shapes as the bf16
// maps above, no swizzle (the converter warps write the swizzled bf16 layout): boxes of 64 bytes x
// 64 rows x box_slabs slabs, laid out [slab][row][64 B]; the V box [half][chunk][row][64 B]; and
// the scale bytes as a 1-D map with boxes of 64 rows.
bool make_map_u8(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                 const cuuint32_t* box) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
bool make_map_u8_slabs(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_slabs) {
  const cuuint64_t dims[3] = {64, rows, 9};
  const cuuint64_t strides[2] = {mla::kDRow, 64};
  const cuuint32_t box[3] = {64, 64, box_slabs};
  return make_map_u8(map, base, 3, dims, strides, box);
}
bool make_map_u8_vbox(CUtensorMap* map, const void* base, uint64_t rows) {
  const cuuint64_t dims[4] = {64, rows, 4, 2};
  const cuuint64_t strides[3] = {mla::kDRow, 64, 256};
  const cuuint32_t box[4] = {64, 64, 2, 2};
  return make_map_u8(map, base, 4, dims, strides, box);
}
bool make_map_u8_rows(CUtensorMap* map, const void* base, uint64_t rows) {
  const cuuint64_t dims[1] = {rows};
  const cuuint64_t strides[1] = {1};   // not read for a rank-1 map
  const cuuint32_t box[1] = {64};
  return make_map_u8(map, base, 1, dims, strides, box);
}

// Number of CTA pairs of the decode kernel that can be resident at once on the current device.
int decode_cluster_slots() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 74;
  static int cached[64] = {0};
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaFuncSetAttribute(mla::decode_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           mla::kTcSmemBytes) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(mla::kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = mla::kTcSmemBytes;
    if (cudaOccupancyMaxActiveClusters(&n, mla::decode_tc_kernel<false>, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  if (n <= 0) n = device_sm_count() / 2;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

constexpr int kMaxSplits = 1024;

}  // namespace

extern "C" {

int32_t mla_decode_num_splits(int32_t batch, int32_t max_seq_len, int32_t num_splits) {
  if (num_splits > 0) return num_splits > kMaxSplits ? kMaxSplits : num_splits;
  if (batch <= 0 || max_seq_len <= 0) return 1;
  // Work ranges = CTA pairs.  The ranges split the batch's tiles evenly, so as many ranges as pairs
  // can be resident keep every SM busy; an upper bound on the tiles (every sequence at capacity)
  // keeps at least two tiles per range so each pair's start-up is amortised.  The plan itself uses
  // the true lengths on the device.
  const int slots = decode_cluster_slots();
  const long long tiles_max = static_cast<long long>(batch) * ((max_seq_len + mla::kTile - 1) / mla::kTile);
  long long p = (tiles_max + 1) / 2;
  if (p > slots) p = slots;
  if (p > kMaxSplits) p = kMaxSplits;
  return p < 1 ? 1 : static_cast<int32_t>(p);
}

size_t mla_decode_workspace_size(int32_t batch, int32_t max_seq_len, int32_t num_splits) {
  if (batch <= 0) return 0;
  return mla::ws_bytes(batch, mla_decode_num_splits(batch, max_seq_len, num_splits));
}

}  // extern "C"

namespace {

// The decode kernel and its combine over `rows` query rows: row b attends to the first
// lens[b] cached tokens of sequence b, or of sequence seq_map[b] when a map is given (chunked
// prefill).  Host checks shared by both entry points.
mla_status launch_attn(const mla_bf16* q_full, const void* cache, const int32_t* block_table,
                       const int32_t* lens, const int32_t* seq_map, mla_cache_desc desc, int32_t rows,
                       float softmax_scale, int32_t num_splits, void* workspace, size_t workspace_bytes,
                       mla_bf16* out_lat, float* lse, void* stream, const uint8_t* fp8_scales = nullptr) {
  const bool fp8 = fp8_scales != nullptr;
  if (rows < 0 || num_splits < 0) return MLA_ERR_INVALID_ARG;
  if (rows > mla::kMaxDecodeBatch) return MLA_ERR_UNSUPPORTED;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
  CacheView v;
  const mla_status st = check_cache(desc, cache, block_table, &v);
  if (st != MLA_OK) return st;
  if (rows == 0) return MLA_OK;
  if (seq_map == nullptr && rows > desc.num_seqs) return MLA_ERR_INVALID_ARG;
  // FP8: the scale bytes of a 64-row box are copied from row y, which must be a multiple of 16
  // (pages start at multiples of 64; a contiguous cache needs max_seq_len % 16 == 0).
  if (fp8 && (!aligned16(fp8_scales) || (desc.page_size == 0 && desc.max_seq_len % 16 != 0)))
    return MLA_ERR_INVALID_ARG;
  if (q_full == nullptr || lens == nullptr || out_lat == nullptr) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_full) || !aligned16(out_lat) || (lse != nullptr && !aligned16(lse))) return MLA_ERR_INVALID_ARG;
  const int capacity = cache_capacity(desc);
  const int P = mla_decode_num_splits(rows, capacity, num_splits);
  if (workspace == nullptr || !aligned16(workspace) || workspace_bytes < mla::ws_bytes(rows, P))
    return MLA_ERR_WORKSPACE;
  if (desc.num_rows >= (int64_t(1) << 31) || static_cast<int64_t>(rows) * mla::kHeads >= (int64_t(1) << 31))
    return MLA_ERR_UNSUPPORTED;
  cudaStream_t s = as_stream(stream);
  mla::DecodeTcArgs a;
  a.v = v;
  a.seq_lens = lens;
  a.batch = rows;
  a.capacity = capacity;
  a.P = P;
  a.scale_log2 = softmax_scale * mla::kLog2e;
  a.ws = mla::ws_carve(workspace, P);
  a.out_lat = reinterpret_cast<__nv_bfloat16*>(out_lat);
  a.lse = lse;
  a.cache = reinterpret_cast<const uint8_t*>(cache);
  a.row_bytes = fp8 ? mla::kDRow : 2 * mla::kDRow;
  a.seq_map = seq_map;
  CUtensorMap tka, tkb, tv, tq, tsc;
  if (!make_map_slabs(&tq, q_full, static_cast<uint64_t>(rows) * mla::kHeads, 9)) return MLA_ERR_CUDA;
  if (fp8) {
    if (!make_map_u8_slabs(&tka, cache, desc.num_rows, mla::kTcKSlabsA) ||
        !make_map_u8_slabs(&tkb, cache, desc.num_rows, mla::kTcKSlabsB) ||
        !make_map_u8_vbox(&tv, cache, desc.num_rows) || !make_map_u8_rows(&tsc, fp8_scales, desc.num_rows))
      return MLA_ERR_CUDA;
  } else {
    if (!make_map_slabs(&tka, cache, desc.num_rows, mla::kTcKSlabsA) ||
        !make_map_slabs(&tkb, cache, desc.num_rows, mla::kTcKSlabsB) || !make_map_vbox(&tv, cache, desc.num_rows))
      return MLA_ERR_CUDA;
    tsc = tq;   // unused by the bf16 instances
  }
  if (fp8 && seq_map != nullptr) return MLA_ERR_UNSUPPORTED;
  auto kernel = fp8 ? mla::decode_tc_kernel<false, true>
                    : (seq_map != nullptr ? mla::decode_tc_kernel<true> : mla::decode_tc_kernel<false>);
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, mla::kTcSmemBytes) != cudaSuccess)
    return MLA_ERR_CUDA;
  mla_status ls = launch_chained(kernel, dim3(2 * P), dim3(mla::tc_threads(fp8)),
                                 static_cast<size_t>(mla::kTcSmemBytes), s, tka, tkb, tv, tq, tsc, a);
  if (ls != MLA_OK) return ls;
  // Many rows (a prefill): each warp takes 8 heads of its row, so the plan is read by 8x fewer blocks.
  if (rows > 512)
    return launch_chained(mla::combine_kernel<8>, dim3(rows, mla::kHeads / 32), dim3(128), 0, s, a.ws, P,
                          reinterpret_cast<__nv_bfloat16*>(out_lat), lse);
  return launch_chained(mla::combine_kernel<1>, dim3(rows, mla::kHeads / 4), dim3(128), 0, s, a.ws, P,
                        reinterpret_cast<__nv_bfloat16*>(out_lat), lse);
}

}  // namespace
