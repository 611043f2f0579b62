"""CPU oracle for the CSA / HCA hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never calls it and
shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, single-threaded, double
accumulation); this module compiles it with gcc on first use and marshals
numpy arrays through ctypes, looping over the batch dimension.  Sources are
cited in ``oracle.c``:

  [HA] "DeepSeek-V4 混合注意力：从压缩记忆到百万上下文": §4.1 compressor, §4.2 indexer,
       §5 HCA compressor and dense attention, §6 SWA and attention sink,
       §7 call chain.
  [P1] "揭秘DeepSeek-V4-Pro-MXFP4稀疏注意力：哈希索引与DSA如何撑起1M超长上下文？"
  [P2] "解密DeepSeek-V4-Flash-NVFP4的混合注意力机制：压缩稀疏注意力如何提升长文本处理能力"

Parity status: every function here is pinned by a ``-m "not gpu"`` test
(tests/test_oracle_pins.py) except the FP8 *recall* statistic, which the pages
do not fix ("parity unpinned" for recall only; the e4m3 codec, the FP8 score
definition, the Hadamard rotation of the index vectors, the MXFP4 codec of the FP4
index operands, the partial RoPE and the mixed-precision KV storage codec are pinned).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_vp = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, no fast-math, no FMA contraction).

    With CSA_ORACLE_SANITIZE=1 in the environment the library is built with AddressSanitizer
    and UndefinedBehaviorSanitizer instead (liboracle_san.so); the process then needs the
    sanitizer runtimes preloaded, e.g.
    LD_PRELOAD="$(gcc -print-file-name=libasan.so):$(gcc -print-file-name=libubsan.so)"
    ASAN_OPTIONS=detect_leaks=0 UBSAN_OPTIONS=halt_on_error=1 CSA_ORACLE_SANITIZE=1 \
        python -m pytest tests/test_oracle_pins.py"""
    lib, flags = _LIB, ["-O2"]
    if os.environ.get("CSA_ORACLE_SANITIZE"):
        lib = os.path.join(_HERE, "liboracle_san.so")
        flags = ["-O1", "-g", "-fsanitize=address,undefined", "-fno-omit-frame-pointer"]
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(_SRC):
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *flags, "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, lib)
    return lib


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
    lib.oracle_compress_csa.argtypes = [_f32p, _f32p, _f32p, _f32p, _vp, _vp, i64, i32, i32, _f64p, _f64p]
    lib.oracle_compress_hca.argtypes = [_f32p, _f32p, i64, i32, i32, _f64p, _f64p]
    lib.oracle_n_visible.argtypes = [i64, i32, i64]
    lib.oracle_n_visible.restype = i64
    lib.oracle_index_scores.argtypes = [_f32p, _f32p, _f32p, _i32p, i32, i64, i32, i32, _f64p, _f64p]
    lib.oracle_index_scores_e4m3.argtypes = [_u8p, _f32p, _f32p, _u8p, _f32p, _i32p, i32, i64, i32, i32,
                                             _f64p, _f64p]
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = dbl
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_quantize_rows_e4m3.argtypes = [_f32p, i64, i32, _u8p, _f32p]
    lib.oracle_hadamard_rotate.argtypes = [_f64p, i64, i32, _f64p]
    lib.oracle_rope.argtypes = [_f64p, _i64p, i64, i32, dbl, i32, _f64p]
    lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e2m1_decode.restype = dbl
    lib.oracle_e2m1_encode.argtypes = [dbl]
    lib.oracle_e2m1_encode.restype = ctypes.c_uint8
    lib.oracle_quantize_rows_mxfp4.argtypes = [_f32p, i64, i32, _u8p, _u8p]
    lib.oracle_mxfp4_dequantize.argtypes = [_u8p, _u8p, i64, i32, _f32p]
    lib.oracle_quantize_rows_e4m3_hadamard.argtypes = [_f32p, i64, i32, _u8p, _f32p]
    lib.oracle_sparse_attn_partial.argtypes = [_f32p, _f32p, _f32p, i64, i32, _i64p, _i32p, i32, dbl, i32,
                                               i32, i32, i32, i64, _f64p, _f64p, _f64p]
    lib.oracle_attn_combine.argtypes = [i32, i32, i32, i32, _f64p, _f64p, _f64p, _f32p, _f64p]
    lib.oracle_kv8_entry_bytes.argtypes = [i32]
    lib.oracle_kv8_entry_bytes.restype = i64
    lib.oracle_kv8_quantize.argtypes = [_f32p, i64, i32, _u8p]
    lib.oracle_kv8_dequantize.argtypes = [_u8p, i64, i32, _f32p]
    lib.oracle_topk.argtypes = [_f32p, _i32p, i32, i64, i32, _i32p]
    lib.oracle_sparse_attn.argtypes = [_f32p, _f32p, _f32p, i64, i32, _i64p, _f32p, _i32p, i32, dbl, i32,
                                       i32, i32, i32, i64, _f64p, _f64p]
    lib.oracle_hca_attn.argtypes = [_f32p, _f32p, _f32p, i64, i32, _i64p, _f32p, i32, dbl, i32,
                                    i32, i32, i32, i64, _f64p, _f64p]
    for name in ("oracle_compress_csa", "oracle_compress_hca", "oracle_index_scores",
                 "oracle_index_scores_e4m3", "oracle_quantize_rows_e4m3", "oracle_hadamard_rotate",
                 "oracle_quantize_rows_e4m3_hadamard", "oracle_quantize_rows_mxfp4", "oracle_mxfp4_dequantize",
                 "oracle_rope",
                 "oracle_kv8_quantize",
                 "oracle_kv8_dequantize", "oracle_sparse_attn_partial", "oracle_attn_combine", "oracle_topk",
                 "oracle_sparse_attn", "oracle_hca_attn"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle: {what} rejected its arguments")


# --------------------------------------------------------------------------- compressor
def compress_csa(Ca, Cb, Za, Zb, prev_Cb=None, prev_Zb=None, m: int = 4, with_mag: bool = False):
    """[HA] §4.1 overlapped 2m-position softmax pooling.  Inputs [B, L, c] (or [L, c]);
    optional carry prev_* [B, m, c].  Returns [B, L//m, c] float64 (and the magnitude)."""
    lib = _load()
    Ca, Cb, Za, Zb = (_f32(x) for x in (Ca, Cb, Za, Zb))
    squeeze = Ca.ndim == 2
    if squeeze:
        Ca, Cb, Za, Zb = (x[None] for x in (Ca, Cb, Za, Zb))
        prev_Cb = None if prev_Cb is None else _f32(prev_Cb)[None]
        prev_Zb = None if prev_Zb is None else _f32(prev_Zb)[None]
    B, L, c = Ca.shape
    out = np.empty((B, L // m, c), np.float64)
    mag = np.empty_like(out)
    for b in range(B):
        pc = None if prev_Cb is None else np.ascontiguousarray(_f32(prev_Cb)[b])
        pz = None if prev_Zb is None else np.ascontiguousarray(_f32(prev_Zb)[b])
        ob, mb = np.empty((L // m, c), np.float64), np.empty((L // m, c), np.float64)
        rc = lib.oracle_compress_csa(np.ascontiguousarray(Ca[b]), np.ascontiguousarray(Cb[b]),
                                     np.ascontiguousarray(Za[b]), np.ascontiguousarray(Zb[b]),
                                     None if pc is None else pc.ctypes.data,
                                     None if pz is None else pz.ctypes.data,
                                     L, c, m, ob, mb)
        _check(rc, "compress_csa")
        out[b], mag[b] = ob, mb
    if squeeze:
        out, mag = out[0], mag[0]
    return (out, mag) if with_mag else out


def compress_hca(C, Z, m: int = 128, with_mag: bool = False):
    """[HA] §5 non-overlapped m-position softmax pooling.  [B, L, c] -> [B, L//m, c]."""
    lib = _load()
    C, Z = _f32(C), _f32(Z)
    squeeze = C.ndim == 2
    if squeeze:
        C, Z = C[None], Z[None]
    B, L, c = C.shape
    out = np.empty((B, L // m, c), np.float64)
    mag = np.empty_like(out)
    for b in range(B):
        ob, mb = np.empty((L // m, c), np.float64), np.empty((L // m, c), np.float64)
        _check(lib.oracle_compress_hca(np.ascontiguousarray(C[b]), np.ascontiguousarray(Z[b]),
                                       L, c, m, ob, mb), "compress_hca")
        out[b], mag[b] = ob, mb
    if squeeze:
        out, mag = out[0], mag[0]
    return (out, mag) if with_mag else out


def n_visible(q_pos, m: int, N: int):
    """Number of complete compressed entries visible at each absolute position."""
    lib = _load()
    q = np.asarray(q_pos, np.int64)
    flat = [lib.oracle_n_visible(int(t), m, N) for t in q.reshape(-1)]
    return np.asarray(flat, np.int32).reshape(q.shape)


# --------------------------------------------------------------------------- indexer
def index_scores(qI, w, kI, n_valid, with_mag: bool = False):
    """[HA] §4.2.  qI [B,T,Hi,d], w [B,T,Hi], kI [B,N,d], n_valid [B,T] -> [B,T,N] float64."""
    lib = _load()
    qI, w, kI = _f32(qI), _f32(w), _f32(kI)
    nv = np.ascontiguousarray(np.asarray(n_valid, np.int32))
    B, T, Hi, d = qI.shape
    N = kI.shape[1]
    out = np.empty((B, T, N), np.float64)
    mag = np.empty_like(out)
    for b in range(B):
        ob, mb = np.empty((T, N), np.float64), np.empty((T, N), np.float64)
        _check(lib.oracle_index_scores(np.ascontiguousarray(qI[b]), np.ascontiguousarray(w[b]),
                                       np.ascontiguousarray(kI[b]), np.ascontiguousarray(nv[b]),
                                       T, N, Hi, d, ob, mb), "index_scores")
        out[b], mag[b] = ob, mb
    return (out, mag) if with_mag else out


def index_scores_e4m3(q8, q_scale, w, k8, k_scale, n_valid, with_mag: bool = False):
    """[HA] §4.2 on dequantised e4m3 codes.  q8 [B,T,Hi,d] u8, q_scale [B,T,Hi],
    k8 [B,N,d] u8, k_scale [B,N] -> [B,T,N] float64."""
    lib = _load()
    q8 = np.ascontiguousarray(np.asarray(q8, np.uint8))
    k8 = np.ascontiguousarray(np.asarray(k8, np.uint8))
    q_scale, w, k_scale = _f32(q_scale), _f32(w), _f32(k_scale)
    nv = np.ascontiguousarray(np.asarray(n_valid, np.int32))
    B, T, Hi, d = q8.shape
    N = k8.shape[1]
    out = np.empty((B, T, N), np.float64)
    mag = np.empty_like(out)
    for b in range(B):
        ob, mb = np.empty((T, N), np.float64), np.empty((T, N), np.float64)
        _check(lib.oracle_index_scores_e4m3(np.ascontiguousarray(q8[b]), np.ascontiguousarray(q_scale[b]),
                                            np.ascontiguousarray(w[b]), np.ascontiguousarray(k8[b]),
                                            np.ascontiguousarray(k_scale[b]), np.ascontiguousarray(nv[b]),
                                            T, N, Hi, d, ob, mb), "index_scores_e4m3")
        out[b], mag[b] = ob, mb
    return (out, mag) if with_mag else out


def e4m3_decode(codes):
    lib = _load()
    c = np.asarray(codes, np.uint8)
    return np.asarray([lib.oracle_e4m3_decode(int(b)) for b in c.reshape(-1)], np.float64).reshape(c.shape)


def e4m3_encode(x):
    lib = _load()
    a = np.asarray(x, np.float32)
    return np.asarray([lib.oracle_e4m3_encode(float(v)) for v in a.reshape(-1)], np.uint8).reshape(a.shape)


def quantize_rows_e4m3(x):
    """Per-row e4m3 quantisation (scale = amax/448 in fp32).  x [..., cols] -> (codes u8, scale f32)."""
    lib = _load()
    x = _f32(x)
    cols = x.shape[-1]
    rows = x.size // cols
    codes = np.empty(x.shape, np.uint8)
    scale = np.empty(x.shape[:-1], np.float32)
    _check(lib.oracle_quantize_rows_e4m3(x, rows, cols, codes, scale), "quantize_rows_e4m3")
    return codes, scale


def hadamard_rotate(x):
    """Orthonormal Sylvester Walsh-Hadamard rotation of the last axis ([P1], Indexer
    paragraph).  x [..., n], n a power of two -> float64 [..., n]."""
    lib = _load()
    x = np.ascontiguousarray(np.asarray(x, np.float64))
    n = x.shape[-1]
    y = np.empty(x.shape, np.float64)
    _check(lib.oracle_hadamard_rotate(x, x.size // n if n else 0, n, y), "hadamard_rotate")
    return y


def quantize_rows_e4m3_hadamard(x):
    """Rotate each row, round to fp32, then quantize_rows_e4m3.  x [..., n] -> (codes u8, scale f32)."""
    lib = _load()
    x = _f32(x)
    n = x.shape[-1]
    codes = np.empty(x.shape, np.uint8)
    scale = np.empty(x.shape[:-1], np.float32)
    _check(lib.oracle_quantize_rows_e4m3_hadamard(x, x.size // n, n, codes, scale), "quantize_rows_e4m3_hadamard")
    return codes, scale


def e2m1_decode(codes):
    """FP4 E2M1 code (low nibble) -> value."""
    lib = _load()
    c = np.asarray(codes, np.uint8)
    return np.asarray([lib.oracle_e2m1_decode(int(b)) for b in c.reshape(-1)], np.float64).reshape(c.shape)


def e2m1_encode(x):
    """Nearest E2M1 code (ties to the even mantissa, saturating at 6)."""
    lib = _load()
    a = np.asarray(x, np.float64)
    return np.asarray([lib.oracle_e2m1_encode(float(v)) for v in a.reshape(-1)], np.uint8).reshape(a.shape)


def quantize_rows_mxfp4(x, hadamard: bool = False):
    """MXFP4 of the last axis ([HA] §4.2 FP4 index QK; OCP MX reading): x [..., n], n a
    multiple of 32 -> (codes u8 [..., n] one E2M1 code per byte, scale u8 [..., n/32] E8M0).
    hadamard=True quantises the Walsh-Hadamard-rotated rows, rounded to fp32 first."""
    lib = _load()
    x = _f32(x)
    if hadamard:
        x = hadamard_rotate(x).astype(np.float32)
    n = x.shape[-1]
    codes = np.empty(x.shape, np.uint8)
    scale = np.empty(x.shape[:-1] + (n // 32 if n % 32 == 0 else 0,), np.uint8)
    _check(lib.oracle_quantize_rows_mxfp4(x, x.size // n if n else 0, n, codes, scale), "quantize_rows_mxfp4")
    return codes, scale


def mxfp4_dequantize(codes, scale):
    """codes [..., n], scale [..., n/32] -> float32 [..., n], exactly code * 2^(scale-127)."""
    lib = _load()
    c = np.ascontiguousarray(np.asarray(codes, np.uint8))
    s = np.ascontiguousarray(np.asarray(scale, np.uint8))
    n = c.shape[-1]
    out = np.empty(c.shape, np.float32)
    _check(lib.oracle_mxfp4_dequantize(c, s, c.size // n, n, out), "mxfp4_dequantize")
    return out


def rope(x, pos, theta: float, inverse: bool = False):
    """Partial RoPE of the last 64 dims ([HA] §6; RoFormer pairs (2i, 2i+1), angle
    pos * theta^(-2i/64)).  x [..., D] (taken as float64), pos broadcastable to
    x.shape[:-1] (int) -> float64 [..., D].  inverse turns the other way."""
    lib = _load()
    x = np.ascontiguousarray(np.asarray(x, np.float64))
    D = x.shape[-1]
    p = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, np.int64), x.shape[:-1]).reshape(-1))
    y = np.empty(x.shape, np.float64)
    _check(lib.oracle_rope(x, p, x.size // D if D else 0, D, float(theta), int(inverse), y), "rope")
    return y


def compressed_entry_positions(N: int, m: int):
    """Position of compressed entry i for RoPE: i * m, the first token of its own block
    (a reading: the pages do not say which token an entry stands for)."""
    return np.arange(N, dtype=np.int64) * m


def sparse_attn_rope(q, kv, swa_kv, swa_pos0, q_pos, sink, idx, scale, theta: float, m: int,
                     window: int = 128, kv_pos=None):
    """sparse_attn with the partial RoPE of [HA] §6 around it: the query rotated at its
    position, memory entry i at compressed_entry_positions (or kv_pos [B, N]), SWA row j at
    its token position swa_pos0 + j; attention on the rotated rows (rounded to fp32 for
    the attention definition); the output's last 64 dims turned back at the query's
    position.  Shapes as sparse_attn -> float64 [B, T, H, D]."""
    q = np.asarray(q, np.float64)
    B, T, H, D = q.shape
    N, W = np.asarray(kv).shape[1], np.asarray(swa_kv).shape[1]
    q_pos = np.asarray(q_pos, np.int64)
    if kv_pos is None:
        kv_pos = np.broadcast_to(compressed_entry_positions(N, m), (B, N))
    swa_pos = np.asarray(swa_pos0, np.int64).reshape(B, 1) + np.arange(W, dtype=np.int64)
    qr = rope(q, q_pos[:, :, None], theta)
    kvr = rope(kv, kv_pos, theta)
    swar = rope(swa_kv, swa_pos, theta)
    o = sparse_attn(qr, kvr, swar, swa_pos0, q_pos, sink, idx, scale, window)
    return rope(o, q_pos[:, :, None], theta, inverse=True)


def kv8_entry_bytes(D: int) -> int:
    """Bytes of one mixed-precision compressed entry (FP8 dims, BF16 RoPE dims, scales)."""
    return int(_load().oracle_kv8_entry_bytes(int(D)))


def kv8_quantize(kv):
    """Mixed-precision storage of compressed entries ([HA] §4.2 storage precision):
    kv [..., D] (BF16 values) -> entries [..., kv8_entry_bytes(D)] uint8."""
    lib = _load()
    x = _f32(kv)
    D = x.shape[-1]
    rows = x.size // D
    out = np.empty(x.shape[:-1] + (kv8_entry_bytes(D),), np.uint8)
    _check(lib.oracle_kv8_quantize(x, rows, D, out), "kv8_quantize")
    return out


def kv8_dequantize(entries, D: int):
    """entries [..., kv8_entry_bytes(D)] uint8 -> kv [..., D] float32 (exact values)."""
    lib = _load()
    e = np.ascontiguousarray(np.asarray(entries, np.uint8))
    eb = kv8_entry_bytes(D)
    assert e.shape[-1] == eb
    rows = e.size // eb
    out = np.empty(e.shape[:-1] + (D,), np.float32)
    _check(lib.oracle_kv8_dequantize(e, rows, D, out), "kv8_dequantize")
    return out


# --------------------------------------------------------------------------- top-k
def topk(scores, n_valid, k: int):
    """Full-sort top-k.  scores [B,T,N] float32, n_valid [B,T] -> idx [B,T,k] int32."""
    lib = _load()
    s = _f32(scores)
    nv = np.ascontiguousarray(np.asarray(n_valid, np.int32))
    B, T, N = s.shape
    out = np.empty((B, T, k), np.int32)
    for b in range(B):
        ob = np.empty((T, k), np.int32)
        _check(lib.oracle_topk(np.ascontiguousarray(s[b]), np.ascontiguousarray(nv[b]), T, N, k, ob), "topk")
        out[b] = ob
    return out


# --------------------------------------------------------------------------- attention
def sparse_attn(q, kv, swa_kv, swa_pos0, q_pos, sink, idx, scale, window: int = 128, with_mag: bool = False):
    """[HA] §6-§7 / [P2] sparse_attn.  q [B,T,H,D], kv [B,N,D], swa_kv [B,W,D], swa_pos0 [B],
    q_pos [B,T], sink [H], idx [B,T,k] -> out [B,T,H,D] float64."""
    lib = _load()
    q, kv, swa_kv, sink = _f32(q), _f32(kv), _f32(swa_kv), _f32(sink)
    idx = np.ascontiguousarray(np.asarray(idx, np.int32))
    q_pos = np.ascontiguousarray(np.asarray(q_pos, np.int64))
    swa_pos0 = np.asarray(swa_pos0, np.int64).reshape(-1)
    B, T, H, D = q.shape
    N, W, k = kv.shape[1], swa_kv.shape[1], idx.shape[2]
    out = np.empty((B, T, H, D), np.float64)
    mag = np.empty_like(out)
    for b in range(B):
        ob, mb = np.empty((T, H, D), np.float64), np.empty((T, H, D), np.float64)
        _check(lib.oracle_sparse_attn(np.ascontiguousarray(q[b]), np.ascontiguousarray(kv[b]),
                                      np.ascontiguousarray(swa_kv[b]), int(swa_pos0[b]), W,
                                      np.ascontiguousarray(q_pos[b]), sink, np.ascontiguousarray(idx[b]),
                                      k, float(scale), window, T, H, D, N, ob, mb), "sparse_attn")
        out[b], mag[b] = ob, mb
    return (out, mag) if with_mag else out


def sparse_attn_partial(q, kv, swa_kv, swa_pos0, q_pos, idx, scale, window: int = 128, with_swa: bool = True):
    """Attention pieces over one row set without the sink: (m [B,T,H], l [B,T,H], o [B,T,H,D]),
    m = max z, l = sum e^(z - m), o = sum e^(z - m) row / l.  The SWA rows count only if
    with_swa; the memory rows are kv[idx] for idx in [0, N)."""
    lib = _load()
    q, kv, swa_kv = _f32(q), _f32(kv), _f32(swa_kv)
    B, T, H, D = q.shape
    N, W, k = kv.shape[1], swa_kv.shape[1], idx.shape[2]
    idx = np.ascontiguousarray(np.asarray(idx, np.int32))
    s0 = np.asarray(swa_pos0, np.int64).reshape(B)
    qp = np.ascontiguousarray(np.asarray(q_pos, np.int64))
    m = np.empty((B, T, H)); l = np.empty((B, T, H)); o = np.empty((B, T, H, D))
    for b in range(B):
        mb, lb, ob = np.empty((T, H)), np.empty((T, H)), np.empty((T, H, D))
        _check(lib.oracle_sparse_attn_partial(np.ascontiguousarray(q[b]), np.ascontiguousarray(kv[b]),
                                              np.ascontiguousarray(swa_kv[b]), int(s0[b]), W if with_swa else 0,
                                              np.ascontiguousarray(qp[b]), np.ascontiguousarray(idx[b]), k,
                                              float(scale), window, T, H, D, N, mb, lb, ob), "sparse_attn_partial")
        m[b], l[b], o[b] = mb, lb, ob
    return m, l, o


def attn_combine(m, l, o, sink):
    """Pieces of G disjoint row sets (m, l [G,B,T,H]; o [G,B,T,H,D]) -> attention output
    [B,T,H,D] with the sink added once."""
    lib = _load()
    m, l, o = (np.ascontiguousarray(np.asarray(a, np.float64)) for a in (m, l, o))
    G, B, T, H, D = o.shape
    sk = _f32(sink)
    out = np.empty((B, T, H, D))
    for b in range(B):
        ob = np.empty((T, H, D))
        _check(lib.oracle_attn_combine(G, T, H, D, np.ascontiguousarray(m[:, b]), np.ascontiguousarray(l[:, b]),
                                       np.ascontiguousarray(o[:, b]), sk, ob), "attn_combine")
        out[b] = ob
    return out


def hca_attn(q, kv, swa_kv, swa_pos0, q_pos, sink, scale, ratio: int = 128, window: int = 128,
             with_mag: bool = False):
    """[HA] §5 dense MQA over every complete summary plus the SWA rows."""
    lib = _load()
    q, kv, swa_kv, sink = _f32(q), _f32(kv), _f32(swa_kv), _f32(sink)
    q_pos = np.ascontiguousarray(np.asarray(q_pos, np.int64))
    swa_pos0 = np.asarray(swa_pos0, np.int64).reshape(-1)
    B, T, H, D = q.shape
    N, W = kv.shape[1], swa_kv.shape[1]
    out = np.empty((B, T, H, D), np.float64)
    mag = np.empty_like(out)
    for b in range(B):
        ob, mb = np.empty((T, H, D), np.float64), np.empty((T, H, D), np.float64)
        _check(lib.oracle_hca_attn(np.ascontiguousarray(q[b]), np.ascontiguousarray(kv[b]),
                                   np.ascontiguousarray(swa_kv[b]), int(swa_pos0[b]), W,
                                   np.ascontiguousarray(q_pos[b]), sink, ratio, float(scale), window,
                                   T, H, D, N, ob, mb), "hca_attn")
        out[b], mag[b] = ob, mb
    return (out, mag) if with_mag else out
