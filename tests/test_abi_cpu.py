"""C-ABI checks that need no GPU: the library builds and loads, exports every entry point that
include/mla.h declares, and its host-side validation returns the documented status codes
before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mla():
    import __graft_entry__
    __graft_entry__._build_module().build()
    import mla_latent_kv_20_b200 as m
    return m


def declared_functions():
    src = open(os.path.join(ROOT, "include", "mla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(mla_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_path():
    names = declared_functions()
    for n in ("mla_cache_append", "mla_absorb_q", "mla_decode_attn", "mla_prefill_attn", "mla_unabsorb_v",
              "mla_decode_workspace_size", "mla_get_device_error", "mla_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(mla):
    lib = ctypes.CDLL(mla.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings(mla):
    assert mla.status_string(0) == "MLA_OK"
    assert mla.status_string(3) == "MLA_ERR_WORKSPACE"
    assert mla.status_string(99) == "MLA_ERR_UNKNOWN"
    assert mla.lib.mla_version() >= 100


FAKE = 0x10000  # never dereferenced: validation fails first


@pytest.fixture
def host_only(mla):
    """The tests below pass never-dereferenced addresses and check that host validation refuses
    them before any device call.  They run only where no GPU is visible, so that a regression in
    the validation could never hand such an address to a kernel."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-validation test with placeholder addresses: runs only without a GPU")
    return mla


def test_append_validation(host_only):
    mla = host_only
    lib = mla.lib
    good = mla.contiguous_desc(4, 128)
    assert lib.mla_cache_append(FAKE, FAKE, None, FAKE, None, None, good, 4, 10000.0, None) == 1  # null cache
    assert lib.mla_cache_append(FAKE, FAKE, None, FAKE, FAKE + 8, None, good, 4, 10000.0, None) == 1  # misaligned
    assert lib.mla_cache_append(FAKE, FAKE, None, FAKE, FAKE, None, good, -1, 10000.0, None) == 1
    assert lib.mla_cache_append(FAKE, FAKE, None, FAKE, FAKE, None, good, 4, -1.0, None) == 1
    assert lib.mla_cache_append(FAKE, FAKE, None, FAKE, FAKE, None, good, 0, 10000.0, None) == 0   # no-op
    assert lib.mla_cache_append(FAKE, FAKE, None, FAKE, FAKE, None, good, 5, 10000.0, None) == 1   # > num_seqs
    bad_page = mla.CacheDesc(32, 128, 2, 4, 4 * 128)
    assert lib.mla_cache_append(FAKE, FAKE, None, FAKE, FAKE, FAKE, bad_page, 4, 10000.0, None) == 2
    paged_no_table = mla.paged_desc(4, 2, 8)
    assert lib.mla_cache_append(FAKE, FAKE, None, FAKE, FAKE, None, paged_no_table, 4, 10000.0, None) == 1
    contiguous_with_table = mla.contiguous_desc(4, 128)
    assert lib.mla_cache_append(FAKE, FAKE, None, FAKE, FAKE, FAKE, contiguous_with_table, 4, 10000.0, None) == 1
    too_few_rows = mla.CacheDesc(0, 128, 0, 4, 100)
    assert lib.mla_cache_append(FAKE, FAKE, None, FAKE, FAKE, None, too_few_rows, 1, 10000.0, None) == 1


def test_projection_validation(host_only):
    mla = host_only
    lib = mla.lib
    assert lib.mla_absorb_q(FAKE, FAKE, None, FAKE, FAKE, 0, 10000.0, None) == 0
    assert lib.mla_absorb_q(FAKE, FAKE, None, FAKE, FAKE, -1, 10000.0, None) == 1
    assert lib.mla_absorb_q(FAKE, FAKE, None, FAKE, FAKE, 70000, 10000.0, None) == 2
    assert lib.mla_absorb_q(None, FAKE, None, FAKE, FAKE, 4, 10000.0, None) == 1
    assert lib.mla_absorb_q(FAKE, FAKE, None, FAKE, FAKE + 2, 4, 10000.0, None) == 1
    assert lib.mla_absorb_q(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 0.0, None) == 1
    assert lib.mla_unabsorb_v(FAKE, FAKE, FAKE, 0, None) == 0
    assert lib.mla_unabsorb_v(FAKE, None, FAKE, 4, None) == 1
    assert lib.mla_unabsorb_v(FAKE, FAKE, FAKE + 4, 4, None) == 1


def test_decode_validation_and_workspace(host_only):
    mla = host_only
    lib = mla.lib
    d = mla.contiguous_desc(8, 4096)
    S = lib.mla_decode_num_splits(8, 4096, 16)
    assert S == 16 and lib.mla_decode_num_splits(8, 4096, 5000) == 1024
    need = lib.mla_decode_workspace_size(8, 4096, 16)
    assert need == 2 * 16 * 128 * (512 + 2) * 4 + 48     # partials of 16 ranges + the plan table [8 + 2], 16-B rounded
    # auto: at most one range per two 128-token tiles of batch x max_seq_len (the resident-pair
    # bound is 74 without a device to ask)
    assert lib.mla_decode_num_splits(1, 256, 0) == 1
    assert lib.mla_decode_num_splits(2, 1000, 0) == 8
    assert lib.mla_decode_num_splits(8, 4096, 0) == 74
    args = lambda ws, nbytes, scale=0.072, batch=8, splits=16, desc=d: (  # noqa: E731
        FAKE, FAKE, None, FAKE, desc, batch, scale, splits, ws, nbytes, FAKE, None, None)
    assert lib.mla_decode_attn(*args(FAKE, need - 16)) == 3           # workspace too small
    assert lib.mla_decode_attn(*args(None, need)) == 3                # workspace missing
    assert lib.mla_decode_attn(*args(FAKE, need, scale=0.0)) == 1     # bad scale
    assert lib.mla_decode_attn(*args(FAKE, need, batch=9)) == 1       # batch > num_seqs
    assert lib.mla_decode_attn(*args(FAKE, need, batch=0)) == 0       # empty batch is a no-op
    assert lib.mla_decode_attn(*args(FAKE, need, splits=-1)) == 1
    big = mla.contiguous_desc(16385, 64)
    assert lib.mla_decode_attn(*args(FAKE, 1 << 40, batch=16385, desc=big)) == 2   # batch beyond the plan's limit
    assert lib.mla_get_device_error(None) == 1


def test_prefill_validation(host_only):
    mla = host_only
    """Host checks of mla_prefill_attn (no kernel is launched on any of these paths): the query
    rows may outnumber the cache's sequences (several rows read one sequence), the map is required."""
    lib = mla.lib
    d = mla.contiguous_desc(2, 4096)
    need = lib.mla_decode_workspace_size(40, 4096, 16)
    args = lambda ws, nbytes, q_seq=FAKE, n=40, scale=0.072: (  # noqa: E731
        FAKE, FAKE, None, q_seq, FAKE, d, n, scale, 16, ws, nbytes, FAKE, None, None)
    assert lib.mla_prefill_attn(*args(FAKE, need - 16)) == 3          # workspace too small
    assert lib.mla_prefill_attn(*args(FAKE, need, q_seq=None)) == 1  # the row -> sequence map is required
    assert lib.mla_prefill_attn(*args(FAKE, need, scale=-1.0)) == 1
    assert lib.mla_prefill_attn(*args(FAKE, need, n=0)) == 0         # no rows: a no-op
    assert lib.mla_prefill_attn(*args(FAKE, need, n=16385)) == 2     # beyond the plan's limit


def test_wait_selftest_validates_arguments(host_only):
    mla = host_only
    """Host-side checks of the bounded-wait self-test (no launch, no GPU needed)."""
    import ctypes
    lib = ctypes.CDLL(mla.LIB_PATH)
    lib.mla_selftest_wait_timeout.restype = ctypes.c_int
    lib.mla_selftest_wait_timeout.argtypes = [ctypes.c_uint32, ctypes.c_void_p, ctypes.c_void_p]
    bogus = ctypes.c_void_p(16)
    assert lib.mla_selftest_wait_timeout(0, bogus, None) == 1           # MLA_ERR_INVALID_ARG
    assert lib.mla_selftest_wait_timeout(2000001, bogus, None) == 1
    assert lib.mla_selftest_wait_timeout(1000, None, None) == 1


def test_noalloc_scratch_size_and_refusal(host_only):
    """The static buffer's size as the header states it, as the library reports it and as the binding
    uses it agree; a problem whose partials exceed it is refused before any device call."""
    mla = host_only
    src = open(os.path.join(ROOT, "include", "mla.h")).read()
    m = re.search(r"#define\s+MLA_NOALLOC_SCRATCH_BYTES\s+\(([^)]*)\)", src)
    header_bytes = eval(m.group(1).replace("u", ""))   # e.g. "48u * 1024u * 1024u"
    assert header_bytes == mla.lib.mla_noalloc_scratch_bytes() == mla.NOALLOC_SCRATCH_BYTES
    d = mla.contiguous_desc(4, 131072)
    assert mla.decode_workspace_size(4, 131072, 1024) > mla.NOALLOC_SCRATCH_BYTES
    rc = mla.lib.mla_decode_attn_noalloc(FAKE, FAKE, None, FAKE, d, 4, ctypes.c_float(0.07), 1024, FAKE, None, None)
    assert rc == 3   # MLA_ERR_WORKSPACE
    assert mla.lib.mla_decode_attn_noalloc(FAKE, FAKE, None, FAKE, d, -1, ctypes.c_float(0.07), 0, FAKE, None,
                                           None) == 1
    assert mla.lib.mla_decode_attn_noalloc(FAKE, FAKE, None, FAKE, d, 0, ctypes.c_float(0.07), 0, FAKE, None,
                                           None) == 0   # empty batch: a no-op


def test_fp8_validation(host_only):
    """Host checks of the FP8 cache entry points (nothing is launched on these paths)."""
    mla = host_only
    lib = mla.lib
    d = mla.contiguous_desc(4, 128)
    assert lib.mla_cache_append_fp8(FAKE, FAKE, None, FAKE, FAKE, None, None, d, 4, 10000.0, None) == 1   # no scales
    assert lib.mla_cache_append_fp8(FAKE, FAKE, None, FAKE, FAKE, FAKE, None, d, 0, 10000.0, None) == 0   # no-op
    assert lib.mla_cache_append_fp8(FAKE, FAKE, None, FAKE, FAKE + 8, FAKE, None, d, 4, 10000.0, None) == 1
    need = lib.mla_decode_workspace_size(4, 128, 0)
    args = lambda desc, scales=FAKE, ws=FAKE, nbytes=need: (  # noqa: E731
        FAKE, FAKE, scales, None, FAKE, desc, 4, 0.072, 0, ws, nbytes, FAKE, None, None)
    assert lib.mla_decode_attn_fp8(*args(d, scales=None)) == 1               # scales are required
    assert lib.mla_decode_attn_fp8(*args(d, scales=FAKE + 4)) == 1           # scales 16-byte aligned
    assert lib.mla_decode_attn_fp8(*args(mla.contiguous_desc(4, 100))) == 1  # max_seq_len % 16 != 0
    assert lib.mla_decode_attn_fp8(*args(d, nbytes=need - 16)) == 3          # workspace too small
