/*
 * mla.h — C ABI of the B200 (sm_100a) library for DeepSeek-V2 Multi-head Latent Attention (MLA)
 * decode over the compressed latent KV cache, in its weight-absorbed form: (1) cache append,
 * (2) query absorption, (3) decode attention (split over work ranges, merged by a combine),
 * (4) value un-absorption, and beside them (1') the down-projection + append of new tokens,
 * (6) the output projection and (7) chunked-prefill attention.
 *
 * Sources (page title, section):
 *   [DR] 《DeepSeek-V2》深度解读报告 — §2.2 Low-Rank Key-Value Joint Compression,
 *        §2.3 Absorption, §2.4 Decoupled Rotary Position Embedding, §3.1 MLA 完整计算链路与参数核算,
 *        §3.3 (model width), §4.2 效率证据 (prompt throughput).
 *   [XD] DeepSeek-V2论文解读：MoE架构如何实现训练成本降42.5%与KV缓存压93.3% — §2.1.
 *
 * Fixed model dimensions ([DR] §3.1): n_h = 128 heads, d_h = 128, d_c = 512, d_R = 64.
 * One cached row per token per layer is [c^KV (512) | RoPE(k^R) (64)] = 576 bf16 = 1152 bytes.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library never allocates,
 *     frees or retains them.  bf16 values are passed as their 16-bit patterns (mla_bf16).
 *   - Every tensor pointer must be 16-byte aligned (TMA requirement); MLA_ERR_INVALID_ARG otherwise.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls only enqueue work on
 *     it: they return after host-side validation, never synchronise, and are safe to capture in a
 *     CUDA graph.  The return value reports host-side validation and launch errors only.
 *   - Data-dependent faults (a position beyond the cache capacity, a block id outside the pool,
 *     a bounded wait that gave up) are detected on the device: the offending row is skipped and
 *     a sticky device error word is set; read it with mla_get_device_error().  No kernel traps.
 */
#ifndef MLA_B200_H_
#define MLA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_N_HEADS 128
#define MLA_D_HEAD 128
#define MLA_D_LATENT 512
#define MLA_D_ROPE 64
#define MLA_D_ROW 576
#define MLA_PAGE_SIZE 64

typedef uint16_t mla_bf16; /* bfloat16 bit pattern */

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, inconsistent cache descriptor */
  MLA_ERR_UNSUPPORTED = 2, /* a size outside what the kernels support */
  MLA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than mla_decode_workspace_size() */
  MLA_ERR_CUDA = 4,        /* a CUDA runtime/driver call or kernel launch failed */
  MLA_ERR_DEVICE = 5       /* reported by mla_get_device_error(): a device-side check fired */
} mla_status;

/* Device error codes (bit flags) reported through mla_get_device_error(). */
#define MLA_DEVERR_POS_RANGE 0x1     /* append: position >= capacity, or seq id out of range */
#define MLA_DEVERR_BLOCK_RANGE 0x2   /* a block-table entry outside [0, num_blocks) */
#define MLA_DEVERR_SEQLEN_RANGE 0x4  /* decode: seq_len < 0 or > capacity */
#define MLA_DEVERR_WAIT_TIMEOUT 0x8  /* a bounded pipeline wait gave up; outputs of that CTA invalid */

/*
 * Layout of the latent cache of ONE layer ([DR] §2.4: (d_c + d_R) elements per token per layer).
 *   page_size == 0  (contiguous): cache is [num_seqs][max_seq_len][576]; row of (seq b, token t)
 *                   is b * max_seq_len + t.  block_table must be NULL.
 *   page_size == 64 (paged, PagedAttention-style block table, [XD] §2.1): cache is
 *                   [num_blocks][64][576]; row of (b, t) is block_table[b*max_blocks_per_seq + t/64]*64
 *                   + t%64.  Capacity per sequence is max_blocks_per_seq * 64.
 *   num_seqs: number of sequences the cache holds (contiguous: leading dimension of the buffer;
 *             paged: rows of block_table).  Sequence ids and decode batch indices must be below it.
 *   num_rows: total rows in the cache buffer (num_seqs*max_seq_len, or num_blocks*64); every row
 *             index the library forms is checked against it on the device.
 */
typedef struct {
  int32_t page_size;
  int32_t max_seq_len;
  int32_t max_blocks_per_seq;
  int32_t num_seqs;
  int64_t num_rows;
} mla_cache_desc;

/* Human-readable name of a status code (static string, never NULL). */
const char* mla_status_string(mla_status s);

/* Library ABI version (major * 100 + minor). */
int32_t mla_version(void);

/*
 * (1) Cache append — [DR] §2.4 (decoupled RoPE on the shared key branch) and §3.1 (c^KV and k^R
 *     are the only cached objects).
 * For each new token i in [0, n_tokens):
 *     row = [ c_new[i, 0:512] | RoPE(kr_new[i, 0:64], pos[i]) ]  written to the slot of
 *     (seq = seq_ids ? seq_ids[i] : i, token position pos[i]).
 * RoPE rotates interleaved pairs (x[2j], x[2j+1]) by pos * rope_base^(-2j/64), computed in fp64
 * and rounded once to bf16 (round-to-nearest-even).  c is copied bit-exactly.
 *   c_new   [n_tokens, 512] bf16     kr_new [n_tokens, 64] bf16 (before RoPE)
 *   seq_ids [n_tokens] int32 or NULL pos    [n_tokens] int32
 *   cache   per desc (written)       block_table [num_seqs, max_blocks_per_seq] int32 (paged) or NULL
 * n_tokens == 0 is a no-op.  Device checks: pos in [0, capacity) and the block id in range,
 * else the row is skipped and MLA_DEVERR_POS_RANGE / MLA_DEVERR_BLOCK_RANGE is set.
 */
mla_status mla_cache_append(const mla_bf16* c_new, const mla_bf16* kr_new, const int32_t* seq_ids,
                            const int32_t* pos, mla_bf16* cache, const int32_t* block_table,
                            mla_cache_desc desc, int32_t n_tokens, float rope_base, void* stream);

/*
 * (1-fp8) Cache append into an FP8 latent cache — [DR] §4.2 效率证据 (FP8 serving with the KV cache
 *     at about 6 bits per element; the pages give no format, this library's reading follows).
 * For each new token i, the row r = [c_new[i] (512) | RoPE(kr_new[i], pos[i]) (64)] is formed in
 * fp64 (the latent exactly, the key rotated in fp64 with no bf16 rounding) and stored as
 *     k = the smallest integer with max_j |r_j| <= 448 * 2^k   (0 for an all-zero row)
 *     scales[row] = k + 127                        (E8M0: the byte e stands for the scale 2^(e - 127))
 *     cache[row * 576 + j] = E4M3 code of fp32(r_j * 2^-k)   (OCP E4M3, round to nearest even,
 *                                                             saturating at +-448)
 * so r_j is approximated by code_value * 2^k, which is exact in bf16: 577 bytes per token, against
 * 1152 for the bf16 row.
 *   cache  [num_rows, 576] uint8 (E4M3 codes; contiguous or paged exactly as the bf16 cache, with
 *          the row index of the descriptor)              scales [num_rows] uint8 (E8M0, written)
 *   other arguments, checks and device errors as mla_cache_append.  cache 16-byte aligned.
 * Rows whose largest magnitude is below about 1e-33 lose their smallest codes when expanded to bf16.
 */
mla_status mla_cache_append_fp8(const mla_bf16* c_new, const mla_bf16* kr_new, const int32_t* seq_ids,
                                const int32_t* pos, uint8_t* cache, uint8_t* scales, const int32_t* block_table,
                                mla_cache_desc desc, int32_t n_tokens, float rope_base, void* stream);

/*
 * (1') Down-projection + cache append — [DR] §2.2 (c^KV = W_D^KV h_t), §3.1 (k^R, the shared
 *      64-wide key of the RoPE branch, is projected from h_t too; c^KV and k^R are the only cached
 *      objects), §2.4 (RoPE on that branch only), §3.3 (model width d = 5120).
 * For each new token i in [0, n_tokens):
 *     row = [ W_D^KV h[i] (512) | RoPE(W^KR h[i], pos[i]) (64) ]  written to the slot of
 *     (seq = seq_ids ? seq_ids[i] : i, token position pos[i])
 * i.e. the row mla_cache_append writes for c_new = W_D^KV h, kr_new = W^KR h, without the
 * round trip through memory.  Products in fp32 (exact for bf16), sums over d in fp32; the latent is
 * rounded once to bf16, the key rotated in fp64 from its fp32 sum and rounded once to bf16.
 *   h      [n_tokens, 5120] bf16          w_dkv [512, 5120] bf16 (output index first)
 *   w_kr   [64, 5120] bf16                seq_ids [n_tokens] int32 or NULL    pos [n_tokens] int32
 *   cache  per desc (written)             block_table per desc or NULL
 * n_tokens == 0 is a no-op; n_tokens must be <= 65536.  Device checks as mla_cache_append.  The
 * partial sums pass through a library-owned device buffer (6.8 MB, allocated when the library
 * loads): calls of this entry point on different streams must not overlap in time.
 */
mla_status mla_project_append(const mla_bf16* h, const mla_bf16* w_dkv, const mla_bf16* w_kr,
                              const int32_t* seq_ids, const int32_t* pos, mla_bf16* cache,
                              const int32_t* block_table, mla_cache_desc desc, int32_t n_tokens,
                              float rope_base, void* stream);

/*
 * (2) Query absorption — [DR] §2.3 (q.(W_UK c) = (q W_UK).c by associativity).
 *     q_full[b, h, 0:512]   = sum_j q_nope[b, h, j] * W_UK[h, j, :]        (tcgen05, fp32 accumulate)
 *     q_full[b, h, 512:576] = q_pe[b, h, :], rotated at q_pos[b] if q_pos != NULL
 *   q_nope [batch, 128, 128] bf16   q_pe [batch, 128, 64] bf16   q_pos [batch] int32 or NULL
 *   w_uk   [128, 128, 512] bf16 (head, d_h, d_c)                  q_full [batch, 128, 576] bf16 (written)
 * batch == 0 is a no-op; batch must be <= 65536.
 */
mla_status mla_absorb_q(const mla_bf16* q_nope, const mla_bf16* q_pe, const int32_t* q_pos,
                        const mla_bf16* w_uk, mla_bf16* q_full, int32_t batch, float rope_base,
                        void* stream);

/*
 * (1)+(2) in one launch: the cache append of n_tokens new tokens (exactly mla_cache_append's rows
 * and device checks) and the query absorption of batch queries (exactly mla_absorb_q's q_full),
 * for a decode step that appends the new tokens' rows and absorbs their queries together: one
 * kernel instead of two in the step's chain.  Arguments as in those two calls; n_tokens == 0 skips
 * the append, batch == 0 the absorption.
 */
mla_status mla_append_absorb(const mla_bf16* c_new, const mla_bf16* kr_new, const int32_t* seq_ids,
                             const int32_t* pos, mla_bf16* cache, const int32_t* block_table,
                             mla_cache_desc desc, int32_t n_tokens, const mla_bf16* q_nope,
                             const mla_bf16* q_pe, const int32_t* q_pos, const mla_bf16* w_uk,
                             mla_bf16* q_full, int32_t batch, float rope_base, void* stream);

/*
 * Number of work ranges P (one CTA pair each) the decode divides the batch's cached tokens into:
 * for num_splits == 0 (auto) as many as the device keeps resident, but at most one per two
 * 128-token tiles of batch x max_seq_len; num_splits itself when it is positive (clamped to
 * [1, 1024]).  Depends only on its arguments and the device.
 */
int32_t mla_decode_num_splits(int32_t batch, int32_t max_seq_len, int32_t num_splits);

/*
 * Bytes of workspace mla_decode_attn needs, with P = mla_decode_num_splits(batch, max_seq_len,
 * num_splits): range partials O [2P, 128, 512] fp32 and (m, l) [2P, 128] fp32 each, then the
 * plan table [batch + 2] int32 (per sequence its cost-line offset or first range, the total, the
 * plan kind; rounded up to 16 bytes).
 */
size_t mla_decode_workspace_size(int32_t batch, int32_t max_seq_len, int32_t num_splits);

/*
 * (3) Decode attention over the latent cache — [DR] §2.3/§2.4: score = scale * (q_abs.c + q_pe.k^R),
 *     the sum of the content and position channels; out_lat = softmax-weighted sum of c.
 * Split-KV flash decoding over P work ranges of 128-token tiles (T tiles in the batch, the last
 * tile of a sequence ragged), planned on the device from seq_lens: when every non-empty sequence
 * has at least T/P tiles, sequence b gets floor(P tiles_b / T) ranges that split its tiles evenly
 * (per-sequence plan); otherwise the tiles of the batch are laid end to end and range p takes
 * [floor(pT/P), floor((p+1)T/P)) (balanced plan), so a range may span several sequences and a
 * sequence several ranges.  Each part of a sequence a range covers keeps a running max m and sum
 * l (online softmax); a sequence covered by one range is finished by the decode kernel, the
 * others' unnormalised partials are merged by a combine in ascending range order:
 *     out_lat[b, h, :] = sum_r e^{m_r - M} O_r / sum_r e^{m_r - M} l_r,   M = max_r m_r
 *     lse[b, h]        = M + log(sum_r e^{m_r - M} l_r)                    (natural log)
 * The ranges depend only on seq_lens and P.
 *   q_full   [batch, 128, 576] bf16     cache / block_table per desc     seq_lens [batch] int32
 *   softmax_scale: e.g. 1/sqrt(192)     num_splits: work ranges P, 0 = auto, else forced
 *   workspace: >= mla_decode_workspace_size(batch, desc.max_seq_len or capacity, num_splits) bytes,
 *              16-byte aligned, contents need not be initialised (fully overwritten)
 *   out_lat  [batch, 128, 512] bf16 (written)    lse [batch, 128] fp32 (written) or NULL
 * The result for a sequence does not depend on the cache layout: paged and contiguous caches
 * holding the same rows give bit-identical outputs.  A sequence with seq_len == 0 yields
 * out_lat = 0 and lse = -inf.  seq_len > capacity sets MLA_DEVERR_SEQLEN_RANGE and is clamped.
 * batch must be <= 16384 (MLA_ERR_UNSUPPORTED otherwise).
 */
mla_status mla_decode_attn(const mla_bf16* q_full, const mla_bf16* cache, const int32_t* block_table,
                           const int32_t* seq_lens, mla_cache_desc desc, int32_t batch,
                           float softmax_scale, int32_t num_splits, void* workspace,
                           size_t workspace_bytes, mla_bf16* out_lat, float* lse, void* stream);

/*
 * (7) Chunked prefill attention, absorbed form — [DR] §4.2 (prompt throughput is measured beside
 *     generation) with the attention of (3): a chunk of new tokens of a sequence, appended to the
 *     cache first (mla_cache_append with their positions), each attends causally to the cached
 *     tokens up to and including itself.
 * Query row i (one new token) reads sequence q_seq[i] of the cache and attends to its first
 * q_len[i] tokens (q_len[i] = the token's position + 1 gives the causal mask; rows of later
 * tokens of the same chunk are not read).  Otherwise identical to mla_decode_attn with the query
 * rows in place of the batch: the same work ranges (planned from q_len), the same partials and
 * combine, the same outputs per row:
 *     out_lat[i, h, :] = sum_{t < q_len[i]} softmax_t(scale * q_full[i, h] . row(q_seq[i], t)) c_t
 *   q_full [n_queries, 128, 576] bf16   q_seq, q_len [n_queries] int32 (device)
 *   workspace >= mla_decode_workspace_size(n_queries, capacity, num_splits) bytes
 *   out_lat [n_queries, 128, 512] bf16 (written)   lse [n_queries, 128] fp32 (written) or NULL
 * Any number of rows may read the same sequence, and rows of several sequences may be mixed.
 * q_seq[i] outside [0, desc.num_seqs) sets MLA_DEVERR_BLOCK_RANGE and the row reads zeros;
 * q_len[i] > capacity sets MLA_DEVERR_SEQLEN_RANGE and is clamped.  n_queries <= 16384.
 */
mla_status mla_prefill_attn(const mla_bf16* q_full, const mla_bf16* cache, const int32_t* block_table,
                            const int32_t* q_seq, const int32_t* q_len, mla_cache_desc desc, int32_t n_queries,
                            float softmax_scale, int32_t num_splits, void* workspace, size_t workspace_bytes,
                            mla_bf16* out_lat, float* lse, void* stream);

/*
 * (3-fp8) Decode attention over an FP8 latent cache — [DR] §4.2 效率证据 (FP8 KV cache) with the
 *     attention of (3): every cached row is taken as code_value * 2^(scales[row] - 127), the rows
 *     mla_cache_append_fp8 writes, and attended exactly as mla_decode_attn attends bf16 rows (the
 *     decoded values are exact in bf16, so the result is that of mla_decode_attn on a bf16 cache
 *     holding them).
 *   cache  [num_rows, 576] uint8 E4M3 codes   scales [num_rows] uint8 E8M0 exponents (16-byte aligned)
 *   every other argument, output, workspace and error as mla_decode_attn (mla_decode_workspace_size
 *   applies unchanged).  A contiguous cache needs max_seq_len % 16 == 0 (the scale bytes of a
 *   64-row box are copied from a 16-byte boundary), else MLA_ERR_INVALID_ARG.
 */
mla_status mla_decode_attn_fp8(const mla_bf16* q_full, const uint8_t* cache, const uint8_t* scales,
                               const int32_t* block_table, const int32_t* seq_lens, mla_cache_desc desc,
                               int32_t batch, float softmax_scale, int32_t num_splits, void* workspace,
                               size_t workspace_bytes, mla_bf16* out_lat, float* lse, void* stream);

/*
 * Decode attention that allocates nothing and takes no workspace (the pages have no counterpart:
 * this is a deployment convenience of this library).
 * For callers that cannot obtain device memory at decode time, for example a plugin inside a
 * host engine that owns every device allocation, or a fixed-budget deployment that forbids
 * cudaMalloc after start-up.  Same arguments, result and checks as mla_decode_attn, except that
 * the range partials live in a library-owned static device buffer of MLA_NOALLOC_SCRATCH_BYTES
 * (48 MiB: room for the 2 x 74 partials of the auto plan on a 148-SM device) that every GPU which
 * loads the library holds until the process exits.
 *   - Returns MLA_ERR_WORKSPACE, launching nothing, when mla_decode_workspace_size(batch,
 *     capacity, num_splits) exceeds MLA_NOALLOC_SCRATCH_BYTES (use fewer ranges).
 *   - Every call looks up the buffer's device address for the calling thread's current context
 *     (cudaGetSymbolAddress: no allocation, about a microsecond of host time), so a host engine
 *     that runs the library under a context of its own, or re-creates a context after a device
 *     reset, gets that context's copy.  The first call in a context may load the library's device
 *     code there; make that first call before any stream capture.
 *   - All calls share the one buffer: calls whose kernels overlap on the GPU (different streams,
 *     no ordering between them) race and give wrong results.  The buffer keeps the last call's
 *     contents; nothing in it needs to start at zero (the kernels overwrite what they read).
 *   - Calls no allocation routine (cudaMalloc, cudaFree, or a library allocator).
 */
#define MLA_NOALLOC_SCRATCH_BYTES (48u * 1024u * 1024u)
mla_status mla_decode_attn_noalloc(const mla_bf16* q_full, const mla_bf16* cache, const int32_t* block_table,
                                   const int32_t* seq_lens, mla_cache_desc desc, int32_t batch,
                                   float softmax_scale, int32_t num_splits, mla_bf16* out_lat, float* lse,
                                   void* stream);
/* The size of that static buffer in bytes (MLA_NOALLOC_SCRATCH_BYTES as this build was compiled),
 * so that a binding need not restate the constant. */
size_t mla_noalloc_scratch_bytes(void);

/*
 * (4) Value un-absorption — [DR] §2.3 and [XD] §2.1 (W_UV applied after attention; folding
 *     W_O in is left to the caller).
 *     out[b, h, j] = sum_k out_lat[b, h, k] * W_UV[h, k, j]          (tcgen05, fp32 accumulate)
 *   out_lat [batch, 128, 512] bf16   w_uv [128, 512, 128] bf16 (head, d_c, d_h)
 *   out     [batch, 128, 128] bf16 (written)
 * batch == 0 is a no-op; batch must be <= 65536.
 */
mla_status mla_unabsorb_v(const mla_bf16* out_lat, const mla_bf16* w_uv, mla_bf16* out,
                          int32_t batch, void* stream);

/*
 * (6) Output projection — [DR] §2.3 (W_U^V belongs with the output projection W_O), §3.3 (model
 *     width d = 5120):  y[b] = W_O [ out[b, 0, :] | ... | out[b, 127, :] ]   (5120 <- 16384)
 * on the heads' outputs of mla_unabsorb_v, concatenated head-major.  Products in fp32 (exact for
 * bf16), sums over the 16384 inputs in fp32 (the same order on every call), one bf16 rounding of y.
 *   out [batch, 128, 128] bf16     w_o [5120, 16384] bf16 (output index first)     y [batch, 5120] bf16
 * batch == 0 is a no-op; batch must be <= 65536.  The partial sums pass through a library-owned
 * device buffer (23.5 MB, allocated when the library loads): calls of this entry point on different
 * streams must not overlap in time.
 */
mla_status mla_output_proj(const mla_bf16* out, const mla_bf16* w_o, mla_bf16* y, int32_t batch, void* stream);

/*
 * Self-test of the bounded waits every pipeline of this library uses (the pages have no
 * counterpart; this is failure detection without a fault): launches one CTA that waits on a
 * barrier nothing arrives on, with the wait loop of the pipelines and a limit of limit_us
 * (1 .. 2,000,000).  The wait must give up: result[0] = 1 if it completed (a broken wait),
 * 0 if it gave up; result[1] = microseconds waited.  Giving up sets MLA_DEVERR_WAIT_TIMEOUT with
 * wait site 0x7F (read and clear it with mla_get_device_error); the context stays usable.
 *   result: device int32[2] (written)
 */
mla_status mla_selftest_wait_timeout(uint32_t limit_us, int32_t* result, void* stream);

/*
 * Read and clear the sticky device error word of the current device: bits 0..7 are MLA_DEVERR_*
 * flags; when MLA_DEVERR_WAIT_TIMEOUT is set, bits 8..15 hold the id of the first pipeline wait
 * that gave up (a diagnostic for locating a protocol error).  Synchronises the device.
 * Returns MLA_OK with *code == 0 when no check fired.
 */
mla_status mla_get_device_error(int32_t* code);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H_ */
