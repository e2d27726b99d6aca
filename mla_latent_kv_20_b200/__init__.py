"""Python binding of libmla.so (the C ABI in include/mla.h): argument marshalling only.

Every step of the decode path runs in the library's CUDA kernels; PyTorch tensors are used
only as device buffers (their data pointers are passed through) and for the current stream.
There is no fallback: if the library is missing or fails to load, importing this package
raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla.so")

N_HEADS, D_HEAD, D_LATENT, D_ROPE, D_ROW, PAGE_SIZE = 128, 128, 512, 64, 576, 64

STATUS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_WORKSPACE",
          4: "MLA_ERR_CUDA", 5: "MLA_ERR_DEVICE"}
DEVERR_POS_RANGE, DEVERR_BLOCK_RANGE, DEVERR_SEQLEN_RANGE, DEVERR_WAIT_TIMEOUT = 1, 2, 4, 8


class MlaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


class CacheDesc(ctypes.Structure):
    _fields_ = [("page_size", ctypes.c_int32), ("max_seq_len", ctypes.c_int32),
                ("max_blocks_per_seq", ctypes.c_int32), ("num_seqs", ctypes.c_int32),
                ("num_rows", ctypes.c_int64)]


def contiguous_desc(num_seqs: int, max_seq_len: int) -> CacheDesc:
    return CacheDesc(0, max_seq_len, 0, num_seqs, num_seqs * max_seq_len)


def paged_desc(num_seqs: int, max_blocks_per_seq: int, num_blocks: int) -> CacheDesc:
    return CacheDesc(PAGE_SIZE, max_blocks_per_seq * PAGE_SIZE, max_blocks_per_seq, num_seqs,
                     num_blocks * PAGE_SIZE)


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python mla_latent_kv_20_b200/build.py` "
                          "(or __graft_entry__.build()); there is no non-CUDA fallback")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, F32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sigs = {
        "mla_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "mla_version": (I32, []),
        "mla_cache_append": (ctypes.c_int, [P, P, P, P, P, P, CacheDesc, I32, F32, P]),
        "mla_cache_append_fp8": (ctypes.c_int, [P, P, P, P, P, P, P, CacheDesc, I32, F32, P]),
        "mla_decode_attn_fp8": (ctypes.c_int, [P, P, P, P, P, CacheDesc, I32, F32, I32, P, SZ, P, P, P]),
        "mla_project_append": (ctypes.c_int, [P, P, P, P, P, P, P, CacheDesc, I32, F32, P]),
        "mla_output_proj": (ctypes.c_int, [P, P, P, I32, P]),
        "mla_append_absorb": (ctypes.c_int, [P, P, P, P, P, P, CacheDesc, I32, P, P, P, P, P, I32, F32, P]),
        "mla_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_uint32, P, P]),
        "mla_absorb_q": (ctypes.c_int, [P, P, P, P, P, I32, F32, P]),
        "mla_decode_num_splits": (I32, [I32, I32, I32]),
        "mla_decode_workspace_size": (SZ, [I32, I32, I32]),
        "mla_decode_attn": (ctypes.c_int, [P, P, P, P, CacheDesc, I32, F32, I32, P, SZ, P, P, P]),
        "mla_prefill_attn": (ctypes.c_int, [P, P, P, P, P, CacheDesc, I32, F32, I32, P, SZ, P, P, P]),
        "mla_unabsorb_v": (ctypes.c_int, [P, P, P, I32, P]),
        "mla_decode_attn_noalloc": (ctypes.c_int, [P, P, P, P, CacheDesc, I32, F32, I32, P, P, P]),
        "mla_noalloc_scratch_bytes": (SZ, []),
        "mla_get_device_error": (ctypes.c_int, [ctypes.POINTER(I32)]),
    }
    for name, (res, args) in sigs.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    return lib


lib = _load()


def _ptr(x):
    """Device pointer of a tensor (or an int address, or None -> NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, what: str):
    if status != 0:
        raise MlaError(status, what)


def status_string(s: int) -> str:
    return lib.mla_status_string(s).decode()


def cache_append(c_new, kr_new, pos, cache, desc: CacheDesc, *, seq_ids=None, block_table=None,
                 rope_base: float = 10000.0, stream=None, n_tokens: int | None = None):
    n = c_new.shape[0] if n_tokens is None else n_tokens
    _check(lib.mla_cache_append(_ptr(c_new), _ptr(kr_new), _ptr(seq_ids), _ptr(pos), _ptr(cache),
                                _ptr(block_table), desc, n, rope_base, _stream(stream)), "mla_cache_append")


def cache_append_fp8(c_new, kr_new, pos, cache, scales, desc: CacheDesc, *, seq_ids=None, block_table=None,
                     rope_base: float = 10000.0, stream=None, n_tokens: int | None = None):
    """mla_cache_append_fp8: rows as E4M3 codes (cache, uint8 [rows, 576]) with E8M0 row scales
    (scales, uint8 [rows])."""
    n = c_new.shape[0] if n_tokens is None else n_tokens
    _check(lib.mla_cache_append_fp8(_ptr(c_new), _ptr(kr_new), _ptr(seq_ids), _ptr(pos), _ptr(cache), _ptr(scales),
                                    _ptr(block_table), desc, n, rope_base, _stream(stream)), "mla_cache_append_fp8")


def project_append(h, w_dkv, w_kr, pos, cache, desc: CacheDesc, *, seq_ids=None, block_table=None,
                   rope_base: float = 10000.0, stream=None, n_tokens: int | None = None):
    n = h.shape[0] if n_tokens is None else n_tokens
    _check(lib.mla_project_append(_ptr(h), _ptr(w_dkv), _ptr(w_kr), _ptr(seq_ids), _ptr(pos), _ptr(cache),
                                  _ptr(block_table), desc, n, rope_base, _stream(stream)), "mla_project_append")


def append_absorb(c_new, kr_new, pos, cache, desc: CacheDesc, q_nope, q_pe, w_uk, q_full, *, seq_ids=None,
                  block_table=None, q_pos=None, rope_base: float = 10000.0, stream=None):
    """mla_cache_append and mla_absorb_q in one launch."""
    _check(lib.mla_append_absorb(_ptr(c_new), _ptr(kr_new), _ptr(seq_ids), _ptr(pos), _ptr(cache), _ptr(block_table),
                                 desc, c_new.shape[0], _ptr(q_nope), _ptr(q_pe), _ptr(q_pos), _ptr(w_uk), _ptr(q_full),
                                 q_nope.shape[0], rope_base, _stream(stream)), "mla_append_absorb")


def selftest_wait_timeout(limit_us: int, result, *, stream=None):
    """Run the bounded-wait self-test; result is a device int32[2] tensor (see mla.h)."""
    _check(lib.mla_selftest_wait_timeout(limit_us, _ptr(result), _stream(stream)), "mla_selftest_wait_timeout")


def output_proj(out, w_o, y, *, stream=None, batch: int | None = None):
    b = out.shape[0] if batch is None else batch
    _check(lib.mla_output_proj(_ptr(out), _ptr(w_o), _ptr(y), b, _stream(stream)), "mla_output_proj")


def absorb_q(q_nope, q_pe, w_uk, q_full, *, q_pos=None, rope_base: float = 10000.0, stream=None,
             batch: int | None = None):
    b = q_nope.shape[0] if batch is None else batch
    _check(lib.mla_absorb_q(_ptr(q_nope), _ptr(q_pe), _ptr(q_pos), _ptr(w_uk), _ptr(q_full), b, rope_base,
                            _stream(stream)), "mla_absorb_q")


def decode_num_splits(batch: int, max_seq_len: int, num_splits: int = 0) -> int:
    return lib.mla_decode_num_splits(batch, max_seq_len, num_splits)


def decode_workspace_size(batch: int, max_seq_len: int, num_splits: int = 0) -> int:
    return lib.mla_decode_workspace_size(batch, max_seq_len, num_splits)


def decode_attn(q_full, cache, seq_lens, desc: CacheDesc, workspace, out_lat, *, lse=None, block_table=None,
                softmax_scale: float = 1.0 / 192 ** 0.5, num_splits: int = 0, stream=None,
                batch: int | None = None, workspace_bytes: int | None = None):
    b = q_full.shape[0] if batch is None else batch
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(lib.mla_decode_attn(_ptr(q_full), _ptr(cache), _ptr(block_table), _ptr(seq_lens), desc, b,
                               softmax_scale, num_splits, _ptr(workspace), wb, _ptr(out_lat), _ptr(lse),
                               _stream(stream)), "mla_decode_attn")


def decode_attn_fp8(q_full, cache, scales, seq_lens, desc: CacheDesc, workspace, out_lat, *, lse=None,
                    block_table=None, softmax_scale: float = 1.0 / 192 ** 0.5, num_splits: int = 0, stream=None,
                    batch: int | None = None, workspace_bytes: int | None = None):
    """mla_decode_attn_fp8: decode over an FP8 cache (E4M3 codes + E8M0 row scales)."""
    b = q_full.shape[0] if batch is None else batch
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(lib.mla_decode_attn_fp8(_ptr(q_full), _ptr(cache), _ptr(scales), _ptr(block_table), _ptr(seq_lens), desc,
                                   b, softmax_scale, num_splits, _ptr(workspace), wb, _ptr(out_lat), _ptr(lse),
                                   _stream(stream)), "mla_decode_attn_fp8")


def prefill_attn(q_full, cache, q_seq, q_len, desc: CacheDesc, workspace, out_lat, *, lse=None,
                 block_table=None, softmax_scale: float = 1.0 / 192 ** 0.5, num_splits: int = 0, stream=None,
                 n_queries: int | None = None, workspace_bytes: int | None = None):
    """mla_prefill_attn: query row i (a new token of sequence q_seq[i]) attends to the first
    q_len[i] cached tokens of that sequence."""
    n = q_full.shape[0] if n_queries is None else n_queries
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(lib.mla_prefill_attn(_ptr(q_full), _ptr(cache), _ptr(block_table), _ptr(q_seq), _ptr(q_len), desc, n,
                                softmax_scale, num_splits, _ptr(workspace), wb, _ptr(out_lat), _ptr(lse),
                                _stream(stream)), "mla_prefill_attn")


NOALLOC_SCRATCH_BYTES = int(lib.mla_noalloc_scratch_bytes())   # the library's own constant


def decode_attn_noalloc(q_full, cache, seq_lens, desc: CacheDesc, out_lat, *, lse=None, block_table=None,
                        softmax_scale: float = 1.0 / 192 ** 0.5, num_splits: int = 0, stream=None,
                        batch: int | None = None):
    """mla_decode_attn without a workspace: for callers that cannot allocate device memory at
    decode time; range partials go to the library's static 48 MiB device buffer."""
    b = q_full.shape[0] if batch is None else batch
    _check(lib.mla_decode_attn_noalloc(_ptr(q_full), _ptr(cache), _ptr(block_table), _ptr(seq_lens), desc, b,
                                       softmax_scale, num_splits, _ptr(out_lat), _ptr(lse), _stream(stream)),
           "mla_decode_attn_noalloc")


def unabsorb_v(out_lat, w_uv, out, *, stream=None, batch: int | None = None):
    b = out_lat.shape[0] if batch is None else batch
    _check(lib.mla_unabsorb_v(_ptr(out_lat), _ptr(w_uv), _ptr(out), b, _stream(stream)), "mla_unabsorb_v")


def get_device_error() -> int:
    code = ctypes.c_int32(0)
    _check(lib.mla_get_device_error(ctypes.byref(code)), "mla_get_device_error")
    return code.value
