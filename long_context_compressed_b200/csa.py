"""ctypes binding of libcsa.so (the C ABI in include/csa.h), same entry-point names.

Argument marshalling only: shapes and dtype codes are read off torch tensors,
device pointers and the current CUDA stream are passed through, and a non-zero
status raises ``CsaError``.  Every step of the computation runs in the CUDA
kernels of libcsa.so; there is no other implementation behind these names.
Importing this module fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m long_context_compressed_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

CSA_OK, CSA_ERR_INVALID, CSA_ERR_UNSUPPORTED, CSA_ERR_CUDA, CSA_ERR_TIMEOUT = range(5)
CSA_F32, CSA_BF16, CSA_E4M3, CSA_BF16_KV8, CSA_MXFP4 = 0, 1, 2, 3, 4
CSA_INDEX_KEYS_READY = 1
KV8_DIMS, KV8_BYTES = 512, 608   # mixed-precision compressed entry: 448 e4m3 dims, 64 bf16 RoPE dims, 7 scales
INDEX_HEADS, INDEX_DIM, SWA_WINDOW, MAX_TOPK = 64, 128, 128, 2048

_vp, _i32, _i64, _sz, _f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float

_SIGS = {
    "csa_status_string": ([_i32], ctypes.c_char_p),
    "csa_version": ([], _i32),
    "csa_n_valid": ([_vp, _i64, _i32, _i64, _i64, _vp, _vp], _i32),
    "csa_compress": ([_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _i32, _vp, _vp], _i32),
    "csa_compress_index_keys": ([_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i64, _i64, _vp, _vp, _vp,
                                 _vp], _i32),
    "csa_quantize_e4m3": ([_vp, _i32, _i64, _i32, _vp, _vp, _vp], _i32),
    "csa_quantize_e4m3_hadamard": ([_vp, _i32, _i64, _i32, _vp, _vp, _vp], _i32),
    "csa_quantize_mxfp4": ([_vp, _i32, _i64, _i32, _i32, _vp, _vp, _vp], _i32),
    "csa_mxfp4_sf128_bytes": ([_i64, _i64], _sz),
    "csa_quantize_mxfp4_sf128": ([_vp, _i32, _i64, _i64, _i32, _vp, _vp, _vp], _i32),
    "csa_kv8_entry_bytes": ([_i32], ctypes.c_longlong),
    "csa_quantize_kv8": ([_vp, _i64, _i32, _vp, _vp], _i32),
    "csa_index_scores": ([_vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i64, _vp, _vp, _vp], _i32),
    "csa_index_scores_ex": ([_vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i64, _vp, _vp, ctypes.c_uint, _vp],
                            _i32),
    "csa_index_topk_workspace_size": ([_i32, _i32, _i64, _i32, _i32], _sz),
    "csa_index_topk": ([_vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i64, _i32, _vp, _vp, _vp, _sz, _vp], _i32),
    "csa_select_workspace_size": ([_i32, _i64], _sz),
    "csa_score_histogram": ([_vp, _vp, _i32, _i64, _vp, _sz, _vp], _i32),
    "csa_topk_select": ([_vp, _vp, _i32, _i64, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _sz, _vp], _i32),
    "csa_topk_noalloc": ([_vp, _vp, _i32, _i32, _i64, _i32, _vp, _vp], _i32),
    "csa_index_rerank": ([_vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i64, _i32, _vp, _vp, _vp], _i32),
    "csa_topk_workspace_size": ([_i32, _i32, _i64, _i32], _sz),
    "csa_topk": ([_vp, _vp, _i32, _i32, _i64, _i32, _vp, _vp, _sz, _vp], _i32),
    "csa_attn_workspace_size": ([_i32, _i32, _i32, _i32, _i64, _i32], _sz),
    "sparse_attn": ([_vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _i32, _f32, _i32, _i32, _i32, _i32, _i64, _i32,
                     _vp, _vp, _sz, _vp], _i32),
    "hca_attn": ([_vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32, _f32, _i32, _i32, _i32, _i32, _i64, _i32,
                  _vp, _vp, _sz, _vp], _i32),
    "csa_rope": ([_vp, _i32, _i32, _i64, _i32, _vp, _i64, ctypes.c_double, _i32, _vp, _vp], _i32),
    "sparse_attn_rope": ([_vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _i32, _f32, ctypes.c_double, _i32, _i32, _i32,
                          _i32, _i64, _i32, _vp, _vp, _sz, _vp], _i32),
    "hca_attn_rope": ([_vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32, _f32, ctypes.c_double, _i32, _i32, _i32, _i32,
                       _i64, _i32, _vp, _vp, _sz, _vp], _i32),
    "sparse_attn_partial": ([_vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32, _f32, _i32, _i32, _i32, _i32, _i64, _i32,
                             _vp, _vp, _vp, _sz, _vp], _i32),
    "csa_attn_combine": ([_vp, _i64, _vp, _i64, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp], _i32),
    "csa_shard_select_workspace_size": ([_i32, _i32, _i32], _sz),
    "csa_shard_pack": ([_vp, _vp, _i64, _i64, _i64, _vp, _vp], _i32),
    "csa_shard_select": ([_vp, _i32, _i32, _i32, _vp, _vp, _sz, _vp], _i32),
    "csa_shard_remap": ([_vp, _i64, _i64, _i64, _i64, _vp, _vp], _i32),
    "csa_launch_count": ([], ctypes.c_ulonglong),
    "csa_poll_status": ([_vp], _i32),
    "csa_test_bounded_wait": ([_i32, ctypes.c_longlong, _vp], _i32),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

EXPORTED = tuple(_SIGS)


class CsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {_lib.csa_status_string(status).decode()}")
        self.status = status


def _check(status: int, where: str):
    if status != CSA_OK:
        raise CsaError(status, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return CSA_F32
    if t.dtype == torch.bfloat16:
        return CSA_BF16
    if t.dtype == torch.uint8:
        return CSA_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors must be contiguous CUDA tensors")
    return t.data_ptr()


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def csa_status_string(status: int) -> str:
    return _lib.csa_status_string(status).decode()


def csa_version() -> int:
    return _lib.csa_version()


def csa_n_valid(q_pos, ratio: int, lo: int = 0, hi: int = 0, *, out=None, stream=None):
    """Visible compressed entries per query, q_pos [...] int64 -> n_valid [...] int32, computed by
    the library (entries [lo, hi) held here; pass hi = N for a whole sequence)."""
    if out is None:
        out = torch.empty(q_pos.shape, dtype=torch.int32, device=q_pos.device)
    _check(_lib.csa_n_valid(_ptr(q_pos), q_pos.numel(), int(ratio), int(lo), int(hi), _ptr(out), _stream(stream)),
           "csa_n_valid")
    return out


def csa_compress(C_a, C_b=None, Z_a=None, Z_b=None, prev_Cb=None, prev_Zb=None, *, ratio=4, out=None,
                 out_dtype=None, stream=None):
    """Compressor.  ratio 4: C_a, C_b, Z_a, Z_b [B, L, c] (+ carry [B, 4, c]); ratio 128: C_a = C,
    Z_a = Z, C_b = Z_b = None.  Returns out [B, L // ratio, c]."""
    B, L, c = C_a.shape
    if out is None:
        out = torch.empty((B, L // ratio, c), dtype=out_dtype or C_a.dtype, device=C_a.device)
    _check(_lib.csa_compress(_ptr(C_a), _ptr(C_b), _ptr(Z_a), _ptr(Z_b), _ptr(prev_Cb), _ptr(prev_Zb), B, L, c,
                             ratio, _dtype_code(C_a), _dtype_code(out), _ptr(out), _stream(stream)), "csa_compress")
    return out


def csa_compress_index_keys(C_a, C_b, Z_a, Z_b, prev_Cb, prev_Zb, kI, *, pos0: int, k8=None, k_scale=None,
                            hadamard: bool = True, stream=None):
    """New index-key entries of raw rows C_a, C_b, Z_a, Z_b [B, L, 128] (+ carry [B, 4, 128]) into
    rows pos0 .. pos0 + L/4 - 1 of the caches kI [B, Ncap, 128] bf16 and, if given, k8 [B, Ncap, 128]
    uint8 e4m3 / k_scale [B, Ncap] fp32 (Hadamard-rotated before the quantisation when `hadamard`)."""
    B, L, c = C_a.shape
    _check(_lib.csa_compress_index_keys(_ptr(C_a), _ptr(C_b), _ptr(Z_a), _ptr(Z_b), _ptr(prev_Cb), _ptr(prev_Zb), B, L,
                                        _dtype_code(C_a), int(bool(hadamard)), kI.shape[1], int(pos0), _ptr(kI),
                                        _ptr(k8), _ptr(k_scale), _stream(stream)), "csa_compress_index_keys")
    return kI


def csa_quantize_mxfp4(x, codes=None, scales=None, stream=None, hadamard=False):
    """MXFP4 of x [..., cols] -> (codes uint8 [..., cols/2] two E2M1 values per byte,
    scales uint8 [..., cols/32] E8M0); hadamard=True rotates the rows first."""
    cols = x.shape[-1]
    rows = x.numel() // cols
    if codes is None:
        codes = torch.empty(x.shape[:-1] + (cols // 2,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1] + (cols // 32,), dtype=torch.uint8, device=x.device)
    _check(_lib.csa_quantize_mxfp4(_ptr(x), _dtype_code(x), rows, cols, int(bool(hadamard)), _ptr(codes),
                                   _ptr(scales), _stream(stream)), "csa_quantize_mxfp4")
    return codes, scales


def csa_quantize_e4m3(x, codes=None, scale=None, stream=None, hadamard=False):
    """Per-row e4m3 quantisation of x [..., cols] -> (codes uint8 [..., cols], scale fp32 [...]).
    hadamard=True quantises the Walsh-Hadamard-rotated rows instead (csa_quantize_e4m3_hadamard;
    give queries and keys the same setting)."""
    cols = x.shape[-1]
    rows = x.numel() // cols
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    name = "csa_quantize_e4m3_hadamard" if hadamard else "csa_quantize_e4m3"
    _check(getattr(_lib, name)(_ptr(x), _dtype_code(x), rows, cols, _ptr(codes), _ptr(scale), _stream(stream)),
           name)
    return codes, scale


def csa_index_scores(qI, w, kI, n_valid, *, q_scale=None, k_scale=None, scores=None, select_ws=None,
                     mxfp4: bool = False, keys_ready: bool = False, stream=None):
    """Indexer scores.  qI [B, T, 64, 128] (fp32 | bf16 | uint8 e4m3 codes), w [B, T, 64] fp32,
    kI [B, N, 128] same dtype, n_valid [B, T] int32 -> scores [B, T, N] fp32.  With select_ws
    (T == 1) the per-row score histogram for csa_topk_select is accumulated there.
    mxfp4=True: qI [B, T, 64, 64] / kI [B, N, 64] packed E2M1 codes and q_scale / k_scale their
    tensor-core-layout scales (csa_quantize_mxfp4_sf128).  keys_ready=True: the caller states the
    launch just before this call on the stream does not write kI / k_scale
    (CSA_INDEX_KEYS_READY): the first key tiles then load while that launch finishes."""
    B, T = qI.shape[0], qI.shape[1]
    N = kI.shape[1]
    if scores is None:
        scores = torch.empty((B, T, N), dtype=torch.float32, device=qI.device)
    dt = CSA_MXFP4 if mxfp4 else _dtype_code(qI)
    _check(_lib.csa_index_scores_ex(_ptr(qI), _ptr(q_scale), _ptr(w), _ptr(kI), _ptr(k_scale), dt,
                                    _ptr(n_valid), B, T, N, _ptr(scores), _ptr(select_ws),
                                    CSA_INDEX_KEYS_READY if keys_ready else 0, _stream(stream)),
           "csa_index_scores")
    return scores


def index_topk_workspace(B: int, T: int, N: int, k: int, dtype, device="cuda") -> torch.Tensor:
    """A csa_index_topk workspace (256-byte aligned; no initial contents needed)."""
    n = int(_lib.csa_index_topk_workspace_size(B, T, N, k, dtype))
    buf = torch.empty(max(n, 16) + 256, dtype=torch.uint8, device=device)
    off = (-buf.data_ptr()) % 256
    return buf[off:off + max(n, 16)]


def csa_index_topk(qI, w, kI, n_valid, k: int, *, q_scale=None, k_scale=None, idx=None, workspace=None,
                   failed_rows=None, stream=None):
    """Indexer scores and their top-k without the score matrix: idx [B, T, k] int32 equal to
    csa_topk(csa_index_scores(...), n_valid, k).  qI [B, T, 64, 128] bf16 (or uint8 e4m3 codes
    with q_scale / k_scale), kI [B, N, 128].  failed_rows: optional int32 [1] device tensor that
    receives the number of rows that took the fallback."""
    B, T = qI.shape[0], qI.shape[1]
    N = kI.shape[1]
    dt = _dtype_code(qI)
    if idx is None:
        idx = torch.empty((B, T, k), dtype=torch.int32, device=qI.device)
    if workspace is None:
        workspace = index_topk_workspace(B, T, N, k, dt, qI.device)
    _check(_lib.csa_index_topk(_ptr(qI), _ptr(q_scale), _ptr(w), _ptr(kI), _ptr(k_scale), dt, _ptr(n_valid), B, T,
                               N, k, _ptr(idx), _ptr(failed_rows), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream)),
           "csa_index_topk")
    return idx


def csa_mxfp4_sf128_bytes(batches: int, rows_per_batch: int) -> int:
    """Bytes of the tensor-core-layout scales of `batches` x `rows_per_batch` MXFP4 rows."""
    return int(_lib.csa_mxfp4_sf128_bytes(batches, rows_per_batch))


def csa_quantize_mxfp4_sf128(x, batches: int, *, hadamard: bool = True, codes=None, sf=None, stream=None):
    """MXFP4 index operands with the scales in the tensor-core layout: x [..., 128] (fp32 | bf16) whose
    rows form `batches` equal batches -> (codes uint8 [..., 64], sf uint8 [csa_mxfp4_sf128_bytes])."""
    rows = x.numel() // 128
    rpb = rows // batches
    if codes is None:
        codes = torch.empty(x.shape[:-1] + (64,), dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.zeros(max(16, csa_mxfp4_sf128_bytes(batches, rpb)), dtype=torch.uint8, device=x.device)
    _check(_lib.csa_quantize_mxfp4_sf128(_ptr(x), _dtype_code(x), batches, rpb, int(bool(hadamard)), _ptr(codes),
                                         _ptr(sf), _stream(stream)), "csa_quantize_mxfp4_sf128")
    return codes, sf


def csa_select_workspace_size(B: int, N: int) -> int:
    return int(_lib.csa_select_workspace_size(B, N))


def select_workspace(B: int, N: int, device="cuda") -> torch.Tensor:
    """A zero-filled csa_topk_select workspace (the library keeps it ready between call pairs)."""
    return torch.zeros(max(16, csa_select_workspace_size(B, N)), dtype=torch.uint8, device=device)


def csa_score_histogram(scores, n_valid, workspace, stream=None):
    """Accumulate the per-row score histogram of scores [B, (1,) N] into a select workspace."""
    B, N = scores.shape[0], scores.shape[-1]
    _check(_lib.csa_score_histogram(_ptr(scores), _ptr(n_valid), B, N, _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)),
           "csa_score_histogram")


def csa_topk_select(scores, n_valid, k: int, workspace, *, kc=None, qI=None, w=None, kI=None, idx=None,
                    idx_scores=None, stream=None):
    """Decode top-k from the histogram csa_index_scores(select_ws=workspace) accumulated.
    scores [B, 1, N] (or [B, N]), n_valid [B, 1] -> idx [B, 1, k].  With qI/w/kI (full precision)
    the candidates of the kc-th score's bin are rescored exactly and the best k kept.
    idx_scores (optional, fp32 with idx's shape) receives the score that ranked each entry."""
    B, N = scores.shape[0], scores.shape[-1]
    if idx is None:
        idx = torch.empty((B, 1, k), dtype=torch.int32, device=scores.device)
    kc = k if kc is None else kc
    dt = _dtype_code(qI) if qI is not None else CSA_F32
    _check(_lib.csa_topk_select(_ptr(scores), _ptr(n_valid), B, N, k, kc, _ptr(qI), _ptr(w), _ptr(kI), dt, _ptr(idx),
                                _ptr(idx_scores), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream)),
           "csa_topk_select")
    return idx


def csa_index_rerank(qI, w, kI, cand, k: int, *, cand_scores=None, idx=None, stream=None):
    """Exact rescoring of candidates cand [B, T, kc] (ascending, -1 padded) with full-precision
    qI / kI (fp32 or bf16), then the k best -> idx [B, T, k] int32 (ascending, -1 padded)."""
    B, T, kc = cand.shape
    N = kI.shape[1]
    if cand_scores is None:
        cand_scores = torch.empty((B, T, kc), dtype=torch.float32, device=qI.device)
    if idx is None:
        idx = torch.empty((B, T, k), dtype=torch.int32, device=qI.device)
    _check(_lib.csa_index_rerank(_ptr(qI), _ptr(w), _ptr(kI), _dtype_code(qI), _ptr(cand), kc, B, T, N, k,
                                 _ptr(cand_scores), _ptr(idx), _stream(stream)), "csa_index_rerank")
    return idx


def csa_topk_workspace_size(B: int, T: int, N: int, k: int) -> int:
    return int(_lib.csa_topk_workspace_size(B, T, N, k))


def topk_workspace(B: int, T: int, N: int, k: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace of the size csa_topk needs (the library keeps it zeroed)."""
    n = max(16, csa_topk_workspace_size(B, T, N, k))
    return torch.zeros(n, dtype=torch.uint8, device=device)


def csa_topk(scores, n_valid, k: int, *, idx=None, workspace=None, stream=None):
    """Top-k indices per row of scores [B, T, N] -> idx [B, T, k] int32 (ascending, -1 padded)."""
    B, T, N = scores.shape
    if idx is None:
        idx = torch.empty((B, T, k), dtype=torch.int32, device=scores.device)
    if workspace is None:
        workspace = topk_workspace(B, T, N, k, scores.device)
    _check(_lib.csa_topk(_ptr(scores), _ptr(n_valid), B, T, N, k, _ptr(idx), _ptr(workspace),
                         workspace.numel() * workspace.element_size(), _stream(stream)), "csa_topk")
    return idx


NOALLOC_SCRATCH_BYTES = 16 << 20


def csa_topk_noalloc(scores, n_valid, k: int, *, idx=None, stream=None):
    """csa_topk for callers that cannot allocate device memory: the scratch is the library's own
    16 MiB device array (no workspace argument, no allocation inside the call).  Calls that could
    overlap on the GPU race on that array.  Raises CsaError (CSA_ERR_UNSUPPORTED) when the rows
    need more scratch than the array holds."""
    B, T, N = scores.shape
    if idx is None:
        idx = torch.empty((B, T, k), dtype=torch.int32, device=scores.device)
    rc = _lib.csa_topk_noalloc(_ptr(scores), _ptr(n_valid), B, T, N, k, _ptr(idx), _stream(stream))
    if rc == CSA_ERR_UNSUPPORTED and csa_topk_workspace_size(B, T, N, k) > NOALLOC_SCRATCH_BYTES:
        raise CsaError(rc, f"csa_topk_noalloc: {csa_topk_workspace_size(B, T, N, k)} bytes of scratch needed, "
                           f"the static array holds {NOALLOC_SCRATCH_BYTES}")
    _check(rc, "csa_topk_noalloc")
    return idx


def csa_attn_workspace_size(B: int, T: int, H: int, D: int, rows_per_query: int, dtype: int = CSA_BF16) -> int:
    return int(_lib.csa_attn_workspace_size(B, T, H, D, rows_per_query, dtype))


def attn_workspace(B, T, H, D, rows_per_query, dtype=CSA_BF16, device="cuda"):
    n = max(16, csa_attn_workspace_size(B, T, H, D, rows_per_query, dtype))
    return torch.empty(n, dtype=torch.uint8, device=device)


def quantize_kv8(kv, entries=None, stream=None):
    """Mixed-precision storage of compressed entries (FP8 dims, BF16 RoPE dims):
    kv [..., 512] bf16 -> entries [..., 608] uint8 (layout in include/csa.h)."""
    assert kv.dtype == torch.bfloat16 and kv.shape[-1] == KV8_DIMS
    kv = kv.contiguous()
    rows = kv.numel() // KV8_DIMS
    if entries is None:
        entries = torch.empty(kv.shape[:-1] + (KV8_BYTES,), dtype=torch.uint8, device=kv.device)
    _check(_lib.csa_quantize_kv8(_ptr(kv), rows, KV8_DIMS, _ptr(entries), _stream(stream)), "csa_quantize_kv8")
    return entries


def _attn_dtype(q, kv) -> int:
    # uint8 kv of 608-byte rows: quantize_kv8 entries (bf16 q, swa_kv and out)
    if kv.dtype == torch.uint8:
        assert q.dtype == torch.bfloat16 and kv.shape[-1] == KV8_BYTES
        return CSA_BF16_KV8
    return _dtype_code(q)


def sparse_attn(q, kv, swa_kv, swa_pos0, q_pos, sink, idx, scale: float, *, rope_theta: float = 0.0, out=None,
                workspace=None, stream=None):
    """CSA core attention.  q [B,T,H,D], kv [B,N,D] (or [B,N,608] uint8 quantize_kv8 entries), swa_kv [B,W,D],
    swa_pos0 [B] int64, q_pos [B,T] int64, sink [H] fp32, idx [B,T,k] int32 -> out [B,T,H,D].
    rope_theta > 0: sparse_attn_rope (q turned at q_pos inside, output turned back; rows as stored)."""
    B, T, H, D = q.shape
    N, W, k = kv.shape[1], swa_kv.shape[1], idx.shape[2]
    dt = _attn_dtype(q, kv)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = attn_workspace(B, T, H, D, min(W, SWA_WINDOW) + k, dt, q.device)
    args = (_ptr(q), _ptr(kv), _ptr(swa_kv), _ptr(swa_pos0), W, _ptr(q_pos), _ptr(sink), _ptr(idx), k, float(scale))
    tail = (B, T, H, D, N, dt, _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream(stream))
    if rope_theta:
        _check(_lib.sparse_attn_rope(*args, float(rope_theta), *tail), "sparse_attn_rope")
    else:
        _check(_lib.sparse_attn(*args, *tail), "sparse_attn")
    return out


def hca_attn(q, kv, swa_kv, swa_pos0, q_pos, sink, scale: float, *, ratio: int = 128, rope_theta: float = 0.0,
             out=None, workspace=None, stream=None):
    """HCA core attention: dense over kv[b, :min(N, (pos+1)//ratio)] plus the SWA rows
    (rope_theta > 0: hca_attn_rope)."""
    B, T, H, D = q.shape
    N, W = kv.shape[1], swa_kv.shape[1]
    dt = _attn_dtype(q, kv)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = attn_workspace(B, T, H, D, min(W, SWA_WINDOW) + N, dt, q.device)
    args = (_ptr(q), _ptr(kv), _ptr(swa_kv), _ptr(swa_pos0), W, _ptr(q_pos), _ptr(sink), ratio, float(scale))
    tail = (B, T, H, D, N, dt, _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream(stream))
    if rope_theta:
        _check(_lib.hca_attn_rope(*args, float(rope_theta), *tail), "hca_attn_rope")
    else:
        _check(_lib.hca_attn(*args, *tail), "hca_attn")
    return out


def csa_rope(x, theta: float, *, stride: int = 1, pos_base=None, inverse: bool = False, out=None, stream=None):
    """Partial RoPE of rows x [B, R, D] (fp32 | bf16): dims D-64.. turned at position
    pos_base[b] + r * stride (pos_base [B] int64 or None for 0) -> out (pass out=x for in place)."""
    B, R, D = x.shape
    if out is None:
        out = torch.empty_like(x)
    _check(_lib.csa_rope(_ptr(x), _dtype_code(x), B, R, D, _ptr(pos_base), int(stride), float(theta), int(inverse),
                         _ptr(out), _stream(stream)), "csa_rope")
    return out


def sparse_attn_partial(q, kv, swa_kv, swa_pos0, q_pos, idx, scale: float, *, with_swa: bool = True, out=None,
                        ml=None, workspace=None, stream=None):
    """sparse_attn over these rows without the sink -> (out [B,T,H,D] bf16, ml [B,T,H,2] fp32 (m, l))."""
    B, T, H, D = q.shape
    N, W, k = kv.shape[1], swa_kv.shape[1], idx.shape[2]
    dt = _attn_dtype(q, kv)
    if out is None:
        out = torch.empty_like(q)
    if ml is None:
        ml = torch.empty((B, T, H, 2), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = attn_workspace(B, T, H, D, min(W, SWA_WINDOW) + k, dt, q.device)
    _check(_lib.sparse_attn_partial(_ptr(q), _ptr(kv), _ptr(swa_kv), _ptr(swa_pos0), W if with_swa else 0,
                                    _ptr(q_pos), _ptr(idx), k, float(scale), B, T, H, D, N, dt, _ptr(out), _ptr(ml),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
           "sparse_attn_partial")
    return out, ml


def attn_combine(parts, ml, sink, out=None, stream=None):
    """parts [G,B,T,H,D] bf16 and ml [G,B,T,H,2] fp32 (stacked) -> out [B,T,H,D] bf16, the sink added once."""
    G, B, T, H, D = parts.shape
    if out is None:
        out = torch.empty(parts.shape[1:], dtype=parts.dtype, device=parts.device)
    _check(_lib.csa_attn_combine(_ptr(parts), parts[0].numel() * 2, _ptr(ml), ml[0].numel() * 4, _ptr(sink), G, B,
                                 T, H, D, _ptr(out), _stream(stream)), "csa_attn_combine")
    return out


def attn_combine_packed(gathered, shape, sink, out=None, stream=None):
    """gathered [G, nbytes] uint8, each row one shard's packed (output, (m, l)) buffer of
    pack_partial_views(shape) -> out [B,T,H,D] bf16."""
    G = gathered.shape[0]
    B, T, H, D = shape
    rows = B * T * H
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, device=gathered.device)
    stride = gathered.shape[1]
    base = gathered.data_ptr()
    _check(_lib.csa_attn_combine(base, stride, base + rows * D * 2, stride, _ptr(sink), G, B, T, H, D, _ptr(out),
                                 _stream(stream)), "csa_attn_combine")
    return out


def pack_partial_views(shape, device):
    """One uint8 buffer holding a partial output [B,T,H,D] bf16 followed by its (m, l)
    [B,T,H,2] fp32 -> (buffer, out view, ml view)."""
    B, T, H, D = shape
    ob = B * T * H * D * 2
    buf = torch.empty(ob + B * T * H * 8, dtype=torch.uint8, device=device)
    return buf, buf[:ob].view(torch.bfloat16).view(B, T, H, D), buf[ob:].view(torch.float32).view(B, T, H, 2)


def shard_pack(scores, loc, ns: int, lo: int, pairs=None, stream=None):
    """Winners (scores [..], local indices [..], same shape) -> pairs [.., 2] int32 (score bits, global index)."""
    if pairs is None:
        pairs = torch.empty(tuple(loc.shape) + (2,), dtype=torch.int32, device=loc.device)
    _check(_lib.csa_shard_pack(_ptr(scores), _ptr(loc), loc.numel(), int(ns), int(lo), _ptr(pairs), _stream(stream)),
           "csa_shard_pack")
    return pairs


def shard_select(pairs, k: int, idx=None, workspace=None, stream=None):
    """Gathered pairs [G,B,kk,2] int32 (csa_shard_pack) -> global top-k indices [B,k] (ties to the lower index)."""
    G, B, kk = pairs.shape[0], pairs.shape[1], pairs.shape[2]
    if idx is None:
        idx = torch.empty((B, k), dtype=torch.int32, device=pairs.device)
    if workspace is None:
        workspace = torch.empty(int(_lib.csa_shard_select_workspace_size(G, B, kk)), dtype=torch.uint8,
                                device=pairs.device)
    _check(_lib.csa_shard_select(_ptr(pairs), G, B, kk, _ptr(idx), _ptr(workspace), workspace.numel(),
                                 _stream(stream)), "csa_shard_select")
    return idx


def shard_remap(idx_in, lo: int, hi: int, add: int = 0, out=None, stream=None):
    """out = idx_in - lo + add where lo <= idx_in < hi, else -1 (int32, any shape)."""
    if out is None:
        out = torch.empty_like(idx_in)
    _check(_lib.csa_shard_remap(_ptr(idx_in), idx_in.numel(), int(lo), int(hi), int(add), _ptr(out),
                                _stream(stream)), "csa_shard_remap")
    return out


def csa_launch_count() -> int:
    """Kernels enqueued by libcsa.so in this process so far."""
    return int(_lib.csa_launch_count())


def csa_poll_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return int(_lib.csa_poll_status(_stream(stream)))


def csa_test_bounded_wait(complete: bool, limit_ns: int, stream=None) -> None:
    """Enqueue the bounded-wait check: a kernel waits on a barrier that completes only if
    `complete`; if the limit runs out it records CSA_ERR_TIMEOUT (read by csa_poll_status)."""
    _check(_lib.csa_test_bounded_wait(int(bool(complete)), int(limit_ns), _stream(stream)), "csa_test_bounded_wait")
