"""Host-side checks of the C ABI without a GPU: the library loads, exports every
function include/csa.h declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from long_context_compressed_b200 import build
    build.build()
    return ctypes.CDLL(build.LIB)


def declared_functions():
    text = open(os.path.join(ROOT, "include", "csa.h"), encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


def test_header_declares_the_five_calls():
    names = declared_functions()
    for n in ("csa_compress", "csa_index_scores", "csa_topk", "sparse_attn", "hca_attn"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_binding_names_match_header():
    from long_context_compressed_b200 import csa
    assert sorted(csa.EXPORTED) == declared_functions()


def test_status_strings(lib):
    lib.csa_status_string.restype = ctypes.c_char_p
    assert lib.csa_status_string(0) == b"CSA_OK"
    assert b"INVALID" in lib.csa_status_string(1)
    assert lib.csa_version() == 101


def _vp(x=16):
    return ctypes.c_void_p(x)


def test_compress_rejects_bad_arguments(lib):
    f = lib.csa_compress
    f.restype = ctypes.c_int
    i64 = ctypes.c_int64
    p = _vp()
    # ratio must be 4 or 128
    assert f(p, p, p, p, None, None, 1, i64(64), 8, 5, 1, 1, p, None) == 1
    # carry given for one branch only
    assert f(p, p, p, p, p, None, 1, i64(64), 8, 4, 1, 1, p, None) == 1
    # channels not a multiple of 8
    assert f(p, p, p, p, None, None, 1, i64(64), 12, 4, 1, 1, p, None) == 1
    # misaligned pointer
    assert f(_vp(18), p, p, p, None, None, 1, i64(64), 8, 4, 1, 1, p, None) == 1
    # HCA with a b branch
    assert f(p, p, p, None, None, None, 1, i64(256), 128, 128, 1, 1, p, None) == 1
    # bad dtype code
    assert f(p, p, p, p, None, None, 1, i64(64), 8, 4, 7, 1, p, None) == 1
    # nothing to do is OK and launches nothing
    assert f(p, p, p, p, None, None, 0, i64(64), 8, 4, 1, 1, p, None) == 0
    assert f(p, p, p, p, None, None, 1, i64(3), 8, 4, 1, 1, p, None) == 0


def test_topk_rejects_bad_arguments(lib):
    f = lib.csa_topk
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    p = 16
    assert f(p, p, 1, 1, 100, 0, p, None, 0, None) == 1           # k < 1
    assert f(p, p, 1, 1, 100, 4096, p, None, 0, None) == 1        # k > max
    assert f(p, p, 1, 1, (1 << 20) + 1, 8, p, None, 0, None) == 2  # N too large
    # long rows need a workspace of csa_topk_workspace_size bytes
    lib.csa_topk_workspace_size.restype = ctypes.c_size_t
    lib.csa_topk_workspace_size.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int]
    need = lib.csa_topk_workspace_size(1, 1, 262144, 1024)
    assert need > 262144 * 8
    assert f(p, p, 1, 1, 262144, 1024, p, None, 0, None) == 1
    assert f(p, p, 1, 1, 262144, 1024, p, 16, need - 1, None) == 1
    assert lib.csa_topk_workspace_size(4096, 1, 32768, 512) == 0   # row-resident path needs none


def test_index_and_attention_reject_bad_arguments(lib):
    f = lib.csa_index_scores
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
    p = 16
    assert f(p, None, p, p, None, 2, p, 1, 1, 100, p, None) == 1   # e4m3 without scales
    assert f(p, None, p, p, None, 9, p, 1, 1, 100, p, None) == 1   # bad dtype
    assert f(p, None, None, p, None, 1, p, 1, 1, 100, p, None) == 1  # no head weights
    fx = lib.csa_index_scores_ex
    fx.restype = ctypes.c_int
    fx.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint,
                                           ctypes.c_void_p]
    assert fx(p, None, p, p, None, 1, p, 1, 1, 100, p, None, 2, None) == 1   # unknown flag bit
    assert fx(p, None, p, p, None, 2, p, 1, 1, 100, p, None, 1, None) == 1   # keys ready, e4m3 without scales
    g = lib.sparse_attn
    g.restype = ctypes.c_int
    g.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    # bf16 supports D in {128, 256, 512} and H <= 128
    assert g(p, p, p, p, 128, p, p, p, 8, 0.1, 1, 1, 16, 96, 100, 1, p, None, 0, None) == 2
    assert g(p, p, p, p, 128, p, p, p, 8, 0.1, 1, 1, 256, 512, 100, 1, p, None, 0, None) == 2
    # NaN scale, negative k
    assert g(p, p, p, p, 128, p, p, p, 8, float("nan"), 1, 1, 16, 128, 100, 1, p, None, 0, None) == 1
    assert g(p, p, p, p, 128, p, p, p, -1, 0.1, 1, 1, 16, 128, 100, 1, p, None, 0, None) == 1


def test_index_topk_host_checks(lib):
    """csa_index_topk: unsupported dtypes, k and N past the fused path's limits, a missing or
    short workspace, and the workspace size of the prefill shape (it holds the fallback's
    score matrix besides the candidate lists)."""
    sz = lib.csa_index_topk_workspace_size
    sz.restype = ctypes.c_size_t
    sz.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int]
    need = sz(1, 4096, 32768, 512, 1)
    assert need >= 4096 * 32768 * 4 + 4096 * 8192 * 8
    assert sz(0, 4, 100, 8, 1) == 0
    f = lib.csa_index_topk
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    p, ws = 16, 256
    assert f(p, None, p, p, None, 0, p, 1, 4, 1000, 64, p, None, ws, 1 << 30, None) == 2   # fp32
    assert f(p, None, p, p, None, 4, p, 1, 4, 1000, 64, p, None, ws, 1 << 30, None) == 2   # mxfp4
    assert f(p, None, p, p, None, 1, p, 1, 4, 1000, 2048, p, None, ws, 1 << 30, None) == 2  # k > 1024
    assert f(p, None, p, p, None, 1, p, 1, 4, 40000, 64, p, None, ws, 1 << 30, None) == 2  # N > 32768
    assert f(p, None, p, p, None, 2, p, 1, 4, 1000, 64, p, None, ws, 1 << 30, None) == 1   # e4m3, no scales
    assert f(p, None, p, p, None, 1, p, 1, 4, 1000, 0, p, None, ws, 1 << 30, None) == 1    # k = 0
    assert f(p, None, p, p, None, 1, p, 1, 4, 1000, 64, p, None, None, 0, None) == 1       # no workspace
    assert f(p, None, p, p, None, 1, p, 1, 4, 1000, 64, p, None, ws, 64, None) == 1        # too small
    assert f(p, None, p, p, None, 1, p, 1, 4, 1000, 64, p, None, 16, 1 << 30, None) == 1   # misaligned


def test_kv8_storage_host_checks(lib):
    """Mixed-precision entries: 608 bytes at D = 512, nothing else; bad arguments rejected."""
    eb = lib.csa_kv8_entry_bytes
    eb.restype = ctypes.c_longlong
    eb.argtypes = [ctypes.c_int]
    assert eb(512) == 608 and eb(128) == 0 and eb(256) == 0
    q = lib.csa_quantize_kv8
    q.restype = ctypes.c_int
    q.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    p = 16
    assert q(p, 4, 256, p, None) == 2            # D other than 512
    assert q(None, 4, 512, p, None) == 1         # null source
    assert q(p, 4, 512, 8, None) == 1            # misaligned destination
    assert q(p, -1, 512, p, None) == 1
    assert q(p, 0, 512, p, None) == 0            # nothing to do
    g = lib.sparse_attn
    g.restype = ctypes.c_int
    g.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    # CSA_BF16_KV8 (3) needs D = 512 and H <= 128; an unknown dtype is invalid
    assert g(p, p, p, p, 128, p, p, p, 8, 0.1, 1, 1, 16, 256, 100, 3, p, None, 0, None) == 2
    assert g(p, p, p, p, 128, p, p, p, 8, 0.1, 1, 1, 256, 512, 100, 3, p, None, 0, None) == 2
    assert g(p, p, p, p, 128, p, p, p, 8, 0.1, 1, 1, 16, 512, 100, 4, p, None, 0, None) == 1


def test_hadamard_quantizer_host_checks(lib):
    """The rotated quantiser takes rows of 32, 64, 128 or 256 F32 / BF16 values only."""
    f = lib.csa_quantize_e4m3_hadamard
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p]
    p = 16
    for cols in (0, 16, 96, 512, 1024):
        assert f(p, 1, 4, cols, p, p, None) == 1, cols
    assert f(p, 2, 4, 128, p, p, None) == 1          # e4m3 input
    assert f(p, 1, -1, 128, p, p, None) == 1
    assert f(None, 1, 4, 128, p, p, None) == 1
    assert f(p, 1, 4, 128, None, p, None) == 1
    assert f(p + 8, 1, 4, 128, p, p, None) == 1      # x not 16-byte aligned
    assert f(p, 1, 4, 128, p + 4, p, None) == 1      # codes not 16-byte aligned
    for cols in (32, 64, 128, 256):
        assert f(p, 1, 0, cols, p, p, None) == 0     # nothing to do


def test_mxfp4_quantizer_host_checks(lib):
    f = lib.csa_quantize_mxfp4
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p]
    p = 16
    for cols in (0, 16, 48, 96, 512):
        assert f(p, 1, 4, cols, 0, p, p, None) == 1, cols
    assert f(p, 2, 4, 128, 0, p, p, None) == 1          # e4m3 input
    assert f(p, 1, -1, 128, 1, p, p, None) == 1
    assert f(None, 1, 4, 128, 1, p, p, None) == 1
    assert f(p, 1, 4, 128, 1, p, None, None) == 1
    assert f(p + 8, 1, 4, 128, 0, p, p, None) == 1      # x not 16-byte aligned
    assert f(p, 1, 4, 128, 0, p + 8, p, None) == 1      # codes not 16-byte aligned
    for cols in (32, 64, 128, 256):
        assert f(p, 1, 0, cols, 1, p, p, None) == 0


def test_n_valid_and_bounded_wait_host_checks(lib):
    """csa_n_valid: ratio >= 1, 0 <= lo <= hi, non-null pointers; csa_test_bounded_wait:
    a limit between 1 us and 1 s.  Rejected calls launch nothing."""
    f = lib.csa_n_valid
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                  ctypes.c_void_p]
    p = 16
    assert f(p, 4, 0, 0, 10, p, None) == 1            # ratio 0
    assert f(p, 4, 4, 5, 3, p, None) == 1             # hi < lo
    assert f(p, 4, 4, -1, 3, p, None) == 1            # negative lo
    assert f(p, -1, 4, 0, 3, p, None) == 1            # negative count
    assert f(None, 4, 4, 0, 3, p, None) == 1          # null q_pos
    assert f(p, 4, 4, 0, 3, None, None) == 1          # null output
    assert f(p, 4, 4, 0, 1 << 32, p, None) == 1       # range beyond int32
    assert f(None, 0, 4, 0, 3, None, None) == 0       # nothing to do
    g = lib.csa_test_bounded_wait
    g.restype = ctypes.c_int
    g.argtypes = [ctypes.c_int, ctypes.c_longlong, ctypes.c_void_p]
    for bad in (0, 999, 10 ** 9 + 1, -5):
        assert g(0, bad, None) == 1
