"""Thin ctypes binding of libattn.so (include/attn.h): argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; this module only
allocates output tensors with PyTorch, passes raw pointers, sizes and the current CUDA
stream, and turns status codes into exceptions.  There is no fallback: if the library or
a GPU is missing, calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libattn.so")

ATTN_OK = 0
ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_CUDA = 1, 2, 3
ATTN_ERR_BUDGET, ATTN_ERR_TIMEOUT, ATTN_ERR_INJECTED = 4, 5, 6
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "CUDA error", 4: "budget", 5: "timeout",
          6: "injected"}
ATTN_BF16, ATTN_FP8_E4M3, ATTN_F32, ATTN_INT8, ATTN_INT4 = 0, 1, 2, 3, 4
_KV_NAMES = {"bf16": ATTN_BF16, "fp8": ATTN_FP8_E4M3, "int8": ATTN_INT8, "int4": ATTN_INT4}


def _kv_kind(k, D: int, kv_dtype: str | None) -> int:
    """Cache element kind: explicit ("bf16", "fp8", "int8", "int4"), else from the tensor: int8 ->
    INT8 codes; uint8 rows of D/2 bytes -> packed INT4 codes; uint8 / float8_e4m3fn rows of D -> E4M3
    codes; otherwise bf16."""
    if kv_dtype is not None:
        if kv_dtype not in _KV_NAMES:
            raise ValueError(f"kv_dtype must be one of {sorted(_KV_NAMES)}, not {kv_dtype!r}")
        return _KV_NAMES[kv_dtype]
    if k.dtype == torch.int8:
        return ATTN_INT8
    if k.dtype == torch.uint8 and k.shape[-1] * 2 == D:
        return ATTN_INT4
    if k.dtype in (torch.uint8, torch.float8_e4m3fn):
        return ATTN_FP8_E4M3
    return ATTN_BF16

EXPORTS = [
    "attn_prefill", "attn_decode_workspace_bytes", "attn_decode_num_splits", "attn_decode_splitkv",
    "attn_decode_splitkv_noalloc", "attn_decode_paged", "attn_prefill_varlen", "attn_decode_multi", "attn_decode_multi_workspace_bytes",
    "attn_merge_lse", "attn_stream_plan", "attn_stream_task", "attn_chunked_stream", "attn_status_string",
    "attn_last_cuda_error", "attn_device_status", "attn_set_wait_limit_ns", "attn_debug_wait_probe",
    "attn_debug_inject", "attn_debug_exp2",
]


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} (status {status})")


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("D", ctypes.c_int),
                ("scale", ctypes.c_float)]


class StreamPlan(ctypes.Structure):
    _fields_ = [("q_block", ctypes.c_longlong), ("kv_chunk", ctypes.c_longlong), ("n_tasks", ctypes.c_longlong),
                ("device_bytes", ctypes.c_longlong)]


class StreamStats(ctypes.Structure):
    _fields_ = [("plan", StreamPlan), ("h2d_bytes", ctypes.c_longlong), ("d2h_bytes", ctypes.c_longlong),
                ("ms_total", ctypes.c_double), ("ms_compute", ctypes.c_double), ("ms_device", ctypes.c_double),
                ("ms_compute_busy", ctypes.c_double), ("ms_h2d", ctypes.c_double), ("ms_d2h", ctypes.c_double)]


_lib = None


def _expect(name, t, dtypes, shape):
    """The library reads or writes exactly prod(shape) elements of one of `dtypes` at t's address,
    row-major with no gaps.  A tensor of another type, shape or layout would be misread, or written
    past its end on the device: refuse it.  None passes (optional outputs)."""
    if t is None:
        return
    if not isinstance(dtypes, tuple):
        dtypes = (dtypes,)
    if t.dtype not in dtypes or tuple(t.shape) != tuple(int(x) for x in shape) or not t.is_contiguous():
        want = "/".join(str(d).replace("torch.", "") for d in dtypes)
        raise ValueError(f"{name}: expected a contiguous {want} tensor of shape {tuple(int(x) for x in shape)}, "
                         f"got {str(t.dtype).replace('torch.', '')} {tuple(t.shape)}"
                         f"{'' if t.is_contiguous() else ' (not contiguous)'}")


_ONE_BYTE = (torch.uint8, torch.int8, torch.float8_e4m3fn)


def _check_kv_rows(k, v, D: int, kind: int, k_scale=None, v_scale=None):
    """The library reads rows of D elements (D/2 bytes for packed INT4) and one float32 scale per
    (token, KV head) with strides it derives from the dimensions, so a cache or scale tensor of
    another shape, type or layout would be misread: refuse it."""
    row = D // 2 if kind == ATTN_INT4 else D
    for name, t in (("k", k), ("v", v)):
        if t.shape[-1] != row or not t.is_contiguous():
            raise ValueError(f"{name}: expected a contiguous cache with rows of {row} elements for this "
                             f"element type, got shape {tuple(t.shape)}")
        ok = t.dtype == torch.bfloat16 if kind == ATTN_BF16 else t.dtype in _ONE_BYTE
        if not ok:
            raise ValueError(f"{name}: a {'bf16' if kind == ATTN_BF16 else 'one-byte code'} cache was expected "
                             f"for this element kind, got {t.dtype}")
    if tuple(v.shape) != tuple(k.shape):
        raise ValueError(f"v: expected the shape of k {tuple(k.shape)}, got {tuple(v.shape)}")
    for name, t in (("k_scale", k_scale), ("v_scale", v_scale)):
        if t is not None and (tuple(t.shape) != tuple(k.shape[:-1]) or t.dtype != torch.float32
                              or not t.is_contiguous()):
            raise ValueError(f"{name}: expected contiguous float32 {tuple(k.shape[:-1])}, got "
                             f"{t.dtype} {tuple(t.shape)}")


def _check_decode_io(q, kv_lens, o, lse, ws, q_shape, n_seq):
    """Decode inputs and outputs: q bf16 [B, (n_q,) Hq, D], kv_lens int32 [B], o bf16 of q's shape,
    lse float32 of q's shape without D, the workspace contiguous (its byte size is passed on)."""
    B = q_shape[0]
    _expect("q", q, torch.bfloat16, q_shape)
    _expect("kv_lens", kv_lens, torch.int32, (B,))
    _expect("o", o, torch.bfloat16, q_shape)
    _expect("lse", lse, torch.float32, q_shape[:-1])
    if n_seq is not None and n_seq != B:
        raise ValueError(f"k/v: expected {B} sequences (the batch of q), got {n_seq}")
    if ws is not None and not ws.is_contiguous():
        raise ValueError("ws: expected a contiguous workspace")


def lib() -> ctypes.CDLL:
    """Load libattn.so (built in-tree by exact_long_context_tmem_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m exact_long_context_tmem_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, ll, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t, ctypes.c_float
    L.attn_prefill.argtypes = [vp, vp, vp, vp, i, vp, Dims, i, i, i, ll, ll, ctypes.POINTER(ll), vp]
    L.attn_prefill.restype = i
    L.attn_decode_workspace_bytes.argtypes = [Dims, i, i]
    L.attn_decode_workspace_bytes.restype = sz
    L.attn_decode_num_splits.argtypes = [Dims, i, i]
    L.attn_decode_num_splits.restype = i
    L.attn_decode_splitkv.argtypes = [vp, vp, vp, i, vp, vp, vp, i, Dims, i, vp, vp, vp, sz, vp]
    L.attn_decode_splitkv.restype = i
    L.attn_decode_splitkv_noalloc.argtypes = [vp, vp, vp, i, vp, vp, vp, i, Dims, i, vp, vp, vp]
    L.attn_decode_splitkv_noalloc.restype = i
    L.attn_decode_paged.argtypes = [vp, vp, vp, i, vp, vp, vp, i, i, i, vp, Dims, i, vp, vp, vp, sz, vp]
    L.attn_decode_paged.restype = i
    L.attn_prefill_varlen.argtypes = [vp, vp, vp, vp, i, vp, Dims, vp, vp, i, i, i, i, vp]
    L.attn_prefill_varlen.restype = i
    L.attn_decode_multi_workspace_bytes.argtypes = [Dims, i, i, i]
    L.attn_decode_multi_workspace_bytes.restype = sz
    L.attn_decode_multi.argtypes = [vp, vp, vp, i, vp, vp, vp, i, i, Dims, i, vp, vp, vp, sz, vp]
    L.attn_decode_multi.restype = i
    L.attn_merge_lse.argtypes = [vp, vp, i, ll, i, vp, i, vp, i, vp]
    L.attn_merge_lse.restype = i
    L.attn_stream_plan.argtypes = [Dims, ll, i, ll, sz, ctypes.POINTER(StreamPlan)]
    L.attn_stream_plan.restype = i
    L.attn_stream_task.argtypes = [ctypes.POINTER(StreamPlan), ll, i, ll, ctypes.POINTER(ll), ctypes.POINTER(ll)]
    L.attn_stream_task.restype = i
    L.attn_chunked_stream.argtypes = [vp, vp, vp, vp, vp, Dims, ll, i, ll, sz, vp, vp, ctypes.POINTER(StreamStats)]
    L.attn_chunked_stream.restype = i
    L.attn_status_string.argtypes = [i]
    L.attn_status_string.restype = ctypes.c_char_p
    L.attn_last_cuda_error.argtypes = []
    L.attn_last_cuda_error.restype = i
    L.attn_device_status.argtypes = [i, ctypes.POINTER(i)]
    L.attn_device_status.restype = i
    L.attn_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    L.attn_set_wait_limit_ns.restype = i
    L.attn_debug_wait_probe.argtypes = [ctypes.c_ulonglong]
    L.attn_debug_wait_probe.restype = i
    L.attn_debug_inject.argtypes = [i, ll]
    L.attn_debug_inject.restype = i
    L.attn_debug_exp2.argtypes = [vp, vp, ll, i, vp]
    L.attn_debug_exp2.restype = i
    _ = f
    _lib = L
    return L


def _check(status: int, what: str):
    if status != ATTN_OK:
        raise AttnError(status, what)


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dims(B, Hq, Hkv, D, scale):
    return Dims(int(B), int(Hq), int(Hkv), int(D), float(scale))


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("device tensors expected (the library runs on the GPU only)")


def _bshd_strides(name, t, dtypes, shape):
    """Element strides (batch, token, head) of a [B, S, H, D] view whose D elements are contiguous,
    as attn_prefill takes them; the view may be a slice of a larger tensor (fused QKV, a subset of
    heads, a [B, H, S, D] tensor transposed)."""
    if t.dtype not in dtypes or tuple(t.shape) != tuple(shape):
        want = "/".join(str(d).replace("torch.", "") for d in dtypes)
        raise ValueError(f"{name}: expected a {want} tensor of shape {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")
    if t.shape[-1] > 1 and t.stride(-1) != 1:
        raise ValueError(f"{name}: the last (D) dimension must be contiguous, got strides {t.stride()}")
    return [t.stride(0), t.stride(1), t.stride(2)]


def attn_prefill(q, k, v, *, causal: bool = True, scale: float | None = None, q_pos0: int = 0, kv_pos0: int = 0,
                 o=None, lse=None, out_dtype=torch.bfloat16, want_lse: bool = True, stream=None):
    """q [B,S,Hq,D], k/v [B,T,Hkv,D] bf16 CUDA tensors -> (o [B,S,Hq,D], lse [B,S,Hq] float32).

    q, k, v and a caller-supplied o may be strided views (D contiguous, every other stride a
    multiple of 16 bytes): they are read and written in place through attn_prefill's strides."""
    _need_cuda(q, k, v, o, lse)
    B, S, Hq, D = q.shape
    T, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    if o is None:
        o = torch.empty((B, S, Hq, D), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, S, Hq), dtype=torch.float32, device=q.device)
    _expect("lse", lse, torch.float32, (B, S, Hq))
    bf = (torch.bfloat16,)
    st_all = (_bshd_strides("q", q, bf, (B, S, Hq, D)) + _bshd_strides("k", k, bf, (B, T, Hkv, D)) +
              _bshd_strides("v", v, bf, (B, T, Hkv, D)) +
              _bshd_strides("o", o, (torch.bfloat16, torch.float32), (B, S, Hq, D)))
    packed = all(t.is_contiguous() for t in (q, k, v, o))
    strides = None if packed else (ctypes.c_longlong * 12)(*st_all)
    od = ATTN_F32 if o.dtype == torch.float32 else ATTN_BF16
    st = lib().attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(o), od, _ptr(lse), _dims(B, Hq, Hkv, D, scale), S, T,
                            int(bool(causal)), int(q_pos0), int(kv_pos0), strides, _stream(stream))
    _check(st, "attn_prefill")
    return o, lse


def attn_decode_workspace_bytes(B, Hq, Hkv, D, Tmax, num_splits=0, scale=1.0) -> int:
    return int(lib().attn_decode_workspace_bytes(_dims(B, Hq, Hkv, D, scale), int(Tmax), int(num_splits)))


def attn_decode_num_splits(B, Hq, Hkv, D, Tmax, num_splits=0, scale=1.0) -> int:
    return int(lib().attn_decode_num_splits(_dims(B, Hq, Hkv, D, scale), int(Tmax), int(num_splits)))


def attn_decode_splitkv(q, k, v, kv_lens, *, k_scale=None, v_scale=None, scale: float | None = None,
                        num_splits: int = 0, o=None, lse=None, ws=None, want_lse: bool = True, stream=None,
                        kv_dtype: str | None = None):
    """q [B,Hq,D] bf16; k/v [B,Tmax,Hkv,D] bf16, uint8 E4M3 codes or int8 codes, or [B,Tmax,Hkv,D/2]
    uint8 packed INT4 codes (+ float32 scales [B,Tmax,Hkv] for every coded cache); kv_lens int32
    [B] on the device -> (o [B,Hq,D] bf16, lse [B,Hq] float32)."""
    _need_cuda(q, k, v, kv_lens, k_scale, v_scale, o, lse, ws)
    B, Hq, D = q.shape
    Tmax, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    kind = _kv_kind(k, D, kv_dtype)
    _check_kv_rows(k, v, D, kind, k_scale, v_scale)
    _check_decode_io(q, kv_lens, o, lse, ws, (B, Hq, D), k.shape[0])
    dims = _dims(B, Hq, Hkv, D, scale)
    if o is None:
        o = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    need = int(lib().attn_decode_workspace_bytes(dims, int(Tmax), int(num_splits)))
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    st = lib().attn_decode_splitkv(_ptr(q), _ptr(k), _ptr(v), kind, _ptr(k_scale),
                                   _ptr(v_scale), _ptr(kv_lens), int(Tmax), dims, int(num_splits), _ptr(o),
                                   _ptr(lse), _ptr(ws), ws_bytes, _stream(stream))
    _check(st, "attn_decode_splitkv")
    return o, lse


def attn_prefill_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, *, causal: bool = True,
                        scale: float | None = None, o=None, lse=None, want_lse: bool = True,
                        out_dtype=torch.bfloat16, stream=None):
    """Packed batch: q [total_q,Hq,D], k/v [total_k,Hkv,D] bf16; cu_seqlens_q/k int32 [B+1] on the
    device -> (o [total_q,Hq,D], lse [total_q,Hq] float32)."""
    _need_cuda(q, k, v, cu_seqlens_q, cu_seqlens_k, o, lse)
    total_q, Hq, D = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    B = cu_seqlens_q.shape[0] - 1
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    _expect("q", q, torch.bfloat16, (total_q, Hq, D))
    _expect("k", k, torch.bfloat16, (total_k, Hkv, D))
    _expect("v", v, torch.bfloat16, (total_k, Hkv, D))
    _expect("cu_seqlens_q", cu_seqlens_q, torch.int32, (B + 1,))
    _expect("cu_seqlens_k", cu_seqlens_k, torch.int32, (B + 1,))
    _expect("o", o, (torch.bfloat16, torch.float32), (total_q, Hq, D))
    _expect("lse", lse, torch.float32, (total_q, Hq))
    if o is None:
        o = torch.empty((total_q, Hq, D), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((total_q, Hq), dtype=torch.float32, device=q.device)
    od = ATTN_F32 if o.dtype == torch.float32 else ATTN_BF16
    st = lib().attn_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), od, _ptr(lse), _dims(B, Hq, Hkv, D, scale),
                                   _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), int(total_q), int(total_k),
                                   int(max_seqlen_q), int(bool(causal)), _stream(stream))
    _check(st, "attn_prefill_varlen")
    return o, lse


def attn_decode_multi(q, k, v, kv_lens, *, k_scale=None, v_scale=None, scale: float | None = None,
                      num_splits: int = 0, o=None, lse=None, ws=None, want_lse: bool = True, stream=None,
                      kv_dtype: str | None = None):
    """q [B,n_q,Hq,D] bf16 (n_q new tokens per sequence, already in the cache); k/v as for
    attn_decode_splitkv -> (o [B,n_q,Hq,D] bf16, lse [B,n_q,Hq] float32)."""
    _need_cuda(q, k, v, kv_lens, k_scale, v_scale, o, lse, ws)
    B, n_q, Hq, D = q.shape
    Tmax, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    kind = _kv_kind(k, D, kv_dtype)
    _check_kv_rows(k, v, D, kind, k_scale, v_scale)
    _check_decode_io(q, kv_lens, o, lse, ws, (B, n_q, Hq, D), k.shape[0])
    dims = _dims(B, Hq, Hkv, D, scale)
    if o is None:
        o = torch.empty((B, n_q, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, n_q, Hq), dtype=torch.float32, device=q.device)
    need = int(lib().attn_decode_multi_workspace_bytes(dims, int(Tmax), int(n_q), int(num_splits)))
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    st = lib().attn_decode_multi(_ptr(q), _ptr(k), _ptr(v), kind, _ptr(k_scale),
                                 _ptr(v_scale), _ptr(kv_lens), int(Tmax), int(n_q), dims, int(num_splits), _ptr(o),
                                 _ptr(lse), _ptr(ws), ws_bytes, _stream(stream))
    _check(st, "attn_decode_multi")
    return o, lse


def attn_decode_paged(q, k_pool, v_pool, page_table, kv_lens, *, k_scale=None, v_scale=None,
                      scale: float | None = None, num_splits: int = 0, o=None, lse=None, ws=None,
                      want_lse: bool = True, stream=None, kv_dtype: str | None = None):
    """q [B,Hq,D] bf16; k_pool/v_pool [num_pages, page_size, Hkv, D] bf16, uint8 E4M3 or int8 codes,
    or [num_pages, page_size, Hkv, D/2] packed INT4 codes (+ float32 scale pools
    [num_pages, page_size, Hkv] for every coded cache); page_table int32 [B, max_pages] and
    kv_lens int32 [B] on the device -> (o [B,Hq,D] bf16, lse [B,Hq] float32)."""
    _need_cuda(q, k_pool, v_pool, page_table, kv_lens, k_scale, v_scale, o, lse, ws)
    B, Hq, D = q.shape
    num_pages, page_size, Hkv = k_pool.shape[0], k_pool.shape[1], k_pool.shape[2]
    if page_table.dim() != 2:
        raise ValueError(f"page_table: expected int32 [B, max_pages], got shape {tuple(page_table.shape)}")
    max_pages = page_table.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    kind = _kv_kind(k_pool, D, kv_dtype)
    _check_kv_rows(k_pool, v_pool, D, kind, k_scale, v_scale)
    _check_decode_io(q, kv_lens, o, lse, ws, (B, Hq, D), None)
    _expect("page_table", page_table, torch.int32, (B, max_pages))
    dims = _dims(B, Hq, Hkv, D, scale)
    if o is None:
        o = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    need = int(lib().attn_decode_workspace_bytes(dims, int(max_pages * page_size), int(num_splits)))
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    st = lib().attn_decode_paged(_ptr(q), _ptr(k_pool), _ptr(v_pool), kind,
                                 _ptr(k_scale), _ptr(v_scale), _ptr(page_table), int(max_pages), int(page_size),
                                 int(num_pages), _ptr(kv_lens), dims, int(num_splits), _ptr(o), _ptr(lse), _ptr(ws),
                                 ws_bytes, _stream(stream))
    _check(st, "attn_decode_paged")
    return o, lse


NOALLOC_SCRATCH_BYTES = 4 << 20


def attn_decode_splitkv_noalloc(q, k, v, kv_lens, *, k_scale=None, v_scale=None, scale: float | None = None,
                                num_splits: int = 0, o=None, lse=None, want_lse: bool = True, stream=None,
                                kv_dtype: str | None = None):
    """attn_decode_splitkv without a workspace: the split partials live in the library's static
    device scratch array (see include/attn.h).  For callers that cannot allocate device memory;
    the outputs o and lse may be passed in preallocated."""
    _need_cuda(q, k, v, kv_lens, k_scale, v_scale, o, lse)
    B, Hq, D = q.shape
    Tmax, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    kind = _kv_kind(k, D, kv_dtype)
    _check_kv_rows(k, v, D, kind, k_scale, v_scale)
    _check_decode_io(q, kv_lens, o, lse, None, (B, Hq, D), k.shape[0])
    if o is None:
        o = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    st = lib().attn_decode_splitkv_noalloc(_ptr(q), _ptr(k), _ptr(v), kind,
                                           _ptr(k_scale), _ptr(v_scale), _ptr(kv_lens), int(Tmax),
                                           _dims(B, Hq, Hkv, D, scale), int(num_splits), _ptr(o), _ptr(lse),
                                           _stream(stream))
    _check(st, "attn_decode_splitkv_noalloc")
    return o, lse


def attn_merge_lse(o_parts, lse_parts, *, o_out=None, lse_out=None, accumulate: bool = False,
                   out_dtype=torch.float32, stream=None):
    """o_parts float32 [P,R,D], lse_parts float32 [P,R] -> (o_out [R,D], lse_out [R])."""
    _need_cuda(o_parts, lse_parts, o_out, lse_out)
    P, R, D = o_parts.shape
    _expect("o_parts", o_parts, torch.float32, (P, R, D))
    _expect("lse_parts", lse_parts, torch.float32, (P, R))
    _expect("o_out", o_out, (torch.float32, torch.bfloat16), (R, D))
    _expect("lse_out", lse_out, torch.float32, (R,))
    if o_out is None:
        o_out = torch.empty((R, D), dtype=out_dtype, device=o_parts.device)
    if lse_out is None:
        lse_out = torch.empty((R,), dtype=torch.float32, device=o_parts.device)
    od = ATTN_F32 if o_out.dtype == torch.float32 else ATTN_BF16
    st = lib().attn_merge_lse(_ptr(o_parts), _ptr(lse_parts), int(P), int(R), int(D), _ptr(o_out), od,
                              _ptr(lse_out), int(bool(accumulate)), _stream(stream))
    _check(st, "attn_merge_lse")
    return o_out, lse_out


def attn_stream_plan(B, Hq, Hkv, D, S, *, causal=True, chunk_tokens=0, budget_bytes=16 * 10**9, scale=None):
    plan = StreamPlan()
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    st = lib().attn_stream_plan(_dims(B, Hq, Hkv, D, scale), int(S), int(bool(causal)), int(chunk_tokens),
                                int(budget_bytes), ctypes.byref(plan))
    _check(st, "attn_stream_plan")
    return plan


def attn_stream_task(plan: StreamPlan, S: int, causal: bool, idx: int):
    q0, k0 = ctypes.c_longlong(), ctypes.c_longlong()
    st = lib().attn_stream_task(ctypes.byref(plan), int(S), int(bool(causal)), int(idx), ctypes.byref(q0),
                                ctypes.byref(k0))
    _check(st, "attn_stream_task")
    return q0.value, k0.value


def attn_chunked_stream(q_h, k_h, v_h, *, causal=True, chunk_tokens=0, budget_bytes=16 * 10**9, scale=None,
                        o_h=None, lse_h=None, want_lse=True, compute_stream=None, copy_stream=None):
    """Host (ideally pinned) bf16 q_h [B,S,Hq,D], k_h/v_h [B,S,Hkv,D] -> host (o_h, lse_h, stats)."""
    for t in (q_h, k_h, v_h):
        if t.is_cuda:
            raise ValueError("attn_chunked_stream takes host tensors")
    B, S, Hq, D = q_h.shape
    Hkv = k_h.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    for t in (o_h, lse_h):
        if t is not None and t.is_cuda:
            raise ValueError("attn_chunked_stream takes host tensors")
    _expect("q_h", q_h, torch.bfloat16, (B, S, Hq, D))
    _expect("k_h", k_h, torch.bfloat16, (B, S, Hkv, D))
    _expect("v_h", v_h, torch.bfloat16, (B, S, Hkv, D))
    _expect("o_h", o_h, torch.bfloat16, (B, S, Hq, D))
    _expect("lse_h", lse_h, torch.float32, (B, S, Hq))
    if o_h is None:
        o_h = torch.empty((B, S, Hq, D), dtype=torch.bfloat16, pin_memory=True)
    if lse_h is None and want_lse:
        lse_h = torch.empty((B, S, Hq), dtype=torch.float32, pin_memory=True)
    stats = StreamStats()
    cs = None if compute_stream is None else _stream(compute_stream)
    xs = None if copy_stream is None else _stream(copy_stream)
    st = lib().attn_chunked_stream(_ptr(q_h), _ptr(k_h), _ptr(v_h), _ptr(o_h), _ptr(lse_h),
                                   _dims(B, Hq, Hkv, D, scale), int(S), int(bool(causal)), int(chunk_tokens),
                                   int(budget_bytes), cs, xs, ctypes.byref(stats))
    _check(st, "attn_chunked_stream")
    return o_h, lse_h, stats


def attn_device_status(reset: bool = False):
    site = ctypes.c_int(0)
    st = lib().attn_device_status(int(bool(reset)), ctypes.byref(site))
    return st, site.value


def attn_set_wait_limit_ns(ns: int):
    _check(lib().attn_set_wait_limit_ns(int(ns)), "attn_set_wait_limit_ns")


def attn_debug_wait_probe(limit_ns: int) -> int:
    return int(lib().attn_debug_wait_probe(int(limit_ns)))


def attn_debug_inject(what: int, nth: int):
    _check(lib().attn_debug_inject(int(what), int(nth)), "attn_debug_inject")


def attn_debug_exp2(x, mode: int = 0, stream=None):
    """Device exp2 of a float32 CUDA tensor: mode 0 = FMA-pipe polynomial, 1 = MUFU ex2.approx."""
    _need_cuda(x)
    x = x.contiguous()
    y = torch.empty_like(x)
    _check(lib().attn_debug_exp2(_ptr(x), _ptr(y), x.numel(), int(mode), _stream(stream)), "attn_debug_exp2")
    return y


def attn_status_string(status: int) -> str:
    return lib().attn_status_string(int(status)).decode()
