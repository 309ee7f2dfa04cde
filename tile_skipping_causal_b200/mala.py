"""Python binding of libmala.so (argument marshalling only).

Every function here fills the C structs of include/mala.h from torch CUDA
tensors, allocates outputs/workspace with torch (device memory only), and
calls the library on the current torch stream. All computation happens in
the library's CUDA kernels; there is no fallback: if the library is missing
or the device is not a CUDA device, these functions raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libmala.so")

MALA_OK, MALA_ERR_INVALID_ARG, MALA_ERR_UNSUPPORTED, MALA_ERR_WORKSPACE, MALA_ERR_CUDA, \
    MALA_ERR_TIMEOUT = range(6)
MALA_BF16, MALA_FP32, MALA_FP8_E4M3 = 0, 1, 2
MALA_CAUSAL, MALA_DECODE = 0, 1

_i64x3 = ctypes.c_int64 * 3


class FwdArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("keep_mask", ctypes.c_void_p),
        ("batch", ctypes.c_int64), ("heads_q", ctypes.c_int64), ("heads_kv", ctypes.c_int64),
        ("seqlen_q", ctypes.c_int64), ("seqlen_k", ctypes.c_int64), ("head_dim", ctypes.c_int64),
        ("q_stride", _i64x3), ("k_stride", _i64x3), ("v_stride", _i64x3), ("o_stride", _i64x3),
        ("q_to_kv", ctypes.c_void_p), ("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32),
        ("tau", ctypes.c_float), ("dtype", ctypes.c_int32), ("mode", ctypes.c_int32),
        ("stats", ctypes.c_void_p), ("cu_seqlens_q", ctypes.c_void_p), ("cu_seqlens_k", ctypes.c_void_p),
        ("group_vote", ctypes.c_int32), ("wait_limit_ns", ctypes.c_int64),
    ]


class BwdArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("o", ctypes.c_void_p), ("dout", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("keep_mask", ctypes.c_void_p), ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p),
        ("dv", ctypes.c_void_p), ("bwd_keep_mask", ctypes.c_void_p),
        ("batch", ctypes.c_int64), ("heads_q", ctypes.c_int64), ("heads_kv", ctypes.c_int64),
        ("seqlen_q", ctypes.c_int64), ("seqlen_k", ctypes.c_int64), ("head_dim", ctypes.c_int64),
        ("q_stride", _i64x3), ("k_stride", _i64x3), ("v_stride", _i64x3), ("o_stride", _i64x3),
        ("do_stride", _i64x3), ("dq_stride", _i64x3), ("dk_stride", _i64x3), ("dv_stride", _i64x3),
        ("q_to_kv", ctypes.c_void_p), ("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32),
        ("tau", ctypes.c_float), ("dtype", ctypes.c_int32), ("stats", ctypes.c_void_p),
        ("cu_seqlens_q", ctypes.c_void_p), ("cu_seqlens_k", ctypes.c_void_p),
        ("wait_limit_ns", ctypes.c_int64),
    ]


class DecodeArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("keep_mask", ctypes.c_void_p),
        ("batch", ctypes.c_int64), ("heads_q", ctypes.c_int64), ("heads_kv", ctypes.c_int64),
        ("seqlen_k", ctypes.c_int64), ("head_dim", ctypes.c_int64),
        ("q_stride", _i64x3), ("k_stride", _i64x3), ("v_stride", _i64x3), ("o_stride", _i64x3),
        ("q_to_kv", ctypes.c_void_p), ("block_k", ctypes.c_int32), ("tau", ctypes.c_float),
        ("dtype", ctypes.c_int32), ("num_splits", ctypes.c_int32), ("stats", ctypes.c_void_p),
        ("kv_dtype", ctypes.c_int32), ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float),
        ("group_vote", ctypes.c_int32), ("wait_limit_ns", ctypes.c_int64),
    ]


# symbols declared in include/mala.h
EXPORTS = (
    "mala_fwd", "mala_fwd_workspace_size", "mala_bwd", "mala_bwd_workspace_size",
    "mala_decode", "mala_decode_workspace_size", "mala_status_string",
    "mala_last_error_message", "mala_check_device_error", "mala_version",
    "mala_decode_noalloc",
)

# size of the library's built-in decode scratch buffer (include/mala.h)
DECODE_NOALLOC_SCRATCH_BYTES = 4 << 20

_lib = None


class MalaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{_status_name(code)}: {msg}")
        self.code = code


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmala.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m tile_skipping_causal_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.mala_fwd.argtypes = [ctypes.POINTER(FwdArgs), vp, sz, vp]
    lib.mala_fwd.restype = ctypes.c_int
    lib.mala_fwd_workspace_size.argtypes = [ctypes.POINTER(FwdArgs)]
    lib.mala_fwd_workspace_size.restype = sz
    lib.mala_bwd.argtypes = [ctypes.POINTER(BwdArgs), vp, sz, vp]
    lib.mala_bwd.restype = ctypes.c_int
    lib.mala_bwd_workspace_size.argtypes = [ctypes.POINTER(BwdArgs)]
    lib.mala_bwd_workspace_size.restype = sz
    lib.mala_decode.argtypes = [ctypes.POINTER(DecodeArgs), vp, sz, vp]
    lib.mala_decode.restype = ctypes.c_int
    lib.mala_decode_workspace_size.argtypes = [ctypes.POINTER(DecodeArgs)]
    lib.mala_decode_workspace_size.restype = sz
    lib.mala_status_string.argtypes = [ctypes.c_int]
    lib.mala_status_string.restype = ctypes.c_char_p
    lib.mala_last_error_message.argtypes = []
    lib.mala_last_error_message.restype = ctypes.c_char_p
    lib.mala_check_device_error.argtypes = [vp]
    lib.mala_check_device_error.restype = ctypes.c_int
    lib.mala_version.argtypes = []
    lib.mala_version.restype = ctypes.c_char_p
    lib.mala_decode_noalloc.argtypes = [ctypes.POINTER(DecodeArgs), vp]
    lib.mala_decode_noalloc.restype = ctypes.c_int
    _lib = lib
    return lib


def _status_name(code: int) -> str:
    try:
        return load_library().mala_status_string(code).decode()
    except Exception:
        return f"status {code}"


def _check(code: int):
    if code != MALA_OK:
        raise MalaError(code, load_library().mala_last_error_message().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _strides(t: torch.Tensor):
    if t.stride(-1) != 1:
        raise ValueError("last dimension must be contiguous")
    return _i64x3(t.stride(0), t.stride(1), t.stride(2))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MALA_BF16
    if t.dtype == torch.float32:
        return MALA_FP32
    raise ValueError(f"unsupported dtype {t.dtype}")


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _head_map(q_to_kv: Optional[Sequence[int]]):
    if q_to_kv is None:
        return None, None
    arr = (ctypes.c_int32 * len(q_to_kv))(*[int(x) for x in q_to_kv])
    return arr, ctypes.cast(arr, ctypes.c_void_p)


def _keep_for_stream(ws: Optional[torch.Tensor], stream) -> None:
    """A workspace allocated on torch's current stream but used on another
    must not be handed out again before that stream is done with it."""
    if ws is not None and stream is not None:
        ws.record_stream(stream)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("MALA kernels take CUDA tensors only")


def mask_words(n_tiles: int) -> int:
    return (n_tiles + 31) // 32


def unpack_mask(words: torch.Tensor, n_tiles: int) -> np.ndarray:
    """uint32 bit-set rows (stored as int32) -> bool array [..., n_tiles]."""
    w = words.detach().cpu().numpy().view(np.uint32)
    bits = (w[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1
    return bits.reshape(*w.shape[:-1], -1)[..., :n_tiles].astype(bool)


def pack_mask(mask: np.ndarray) -> np.ndarray:
    """bool [..., n_tiles] -> uint32 words [..., ceil(n/32)] (as int32)."""
    n = mask.shape[-1]
    nw = mask_words(n)
    pad = np.zeros(mask.shape[:-1] + (nw * 32,), dtype=np.uint32)
    pad[..., :n] = mask
    w = (pad.reshape(*mask.shape[:-1], nw, 32) << np.arange(32, dtype=np.uint32)).sum(-1, dtype=np.uint64)
    return w.astype(np.uint32).view(np.int32)


def fwd_args(q, k, v, o, lse, keep_mask, tau, block_q, block_k, stats=None, q_to_kv_ptr=None):
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    a = FwdArgs()
    a.q, a.k, a.v, a.o = _ptr(q), _ptr(k), _ptr(v), _ptr(o)
    a.lse, a.keep_mask = _ptr(lse), _ptr(keep_mask)
    a.batch, a.heads_q, a.heads_kv = B, Hq, Hkv
    a.seqlen_q, a.seqlen_k, a.head_dim = Nq, Nk, d
    a.q_stride, a.k_stride, a.v_stride, a.o_stride = _strides(q), _strides(k), _strides(v), _strides(o)
    a.q_to_kv = q_to_kv_ptr
    a.block_q, a.block_k = block_q, block_k
    a.tau = float(tau)
    a.dtype = _dtype_code(q)
    a.mode = MALA_CAUSAL
    a.stats = _ptr(stats)
    return a


def _packed(cu_seqlens_q, cu_seqlens_k, block_q, block_k):
    """Host int32 offset arrays of packed sequences -> (arrays, number of
    sequences, packed query blocks, largest key-block count)."""
    cq = np.ascontiguousarray(np.asarray(cu_seqlens_q, dtype=np.int32))
    ck = np.ascontiguousarray(np.asarray(cu_seqlens_k, dtype=np.int32))
    if cq.shape != ck.shape or cq.ndim != 1 or cq.size < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must be 1-D arrays of equal length >= 2")
    lq, lk = np.diff(cq.astype(np.int64)), np.diff(ck.astype(np.int64))
    QB = int((-(-lq // block_q)).sum())
    KB = max(1, int((-(-lk // block_k)).max()))
    return cq, ck, cq.size - 1, QB, KB


def mala_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, tau: float,
             block_q: int = 128, block_k: int = 128, *, o=None, lse=None, keep_mask=None,
             with_mask: bool = True, stats=None, q_to_kv=None, stream=None,
             cu_seqlens_q=None, cu_seqlens_k=None, group_vote: bool = False, wait_limit_ns: int = 0):
    """MALA forward/prefill. q [B, N_q, Hq, d], k/v [B, N_k, Hkv, d] (bf16 or
    fp32, scale folded into q; N_q <= N_k, bottom-right aligned). Returns
    (o, lse [B, Hq, N_q] fp32, keep_mask words [B, Hq, nQB, ceil(nKB/32)]
    int32 or None).

    Packed sequences: cu_seqlens_q / cu_seqlens_k (host int32 offsets, one
    more than the number of sequences) with q [1, total_q, Hq, d] and k, v
    [1, total_k, Hkv, d]; lse is then [Hq, total_q] and keep_mask
    [Hq, packed query blocks, ceil(largest key-block count / 32)].

    group_vote: one decision per (query block, key tile) for the query heads
    of a KV head (a tile is skipped only when every row of every head passes
    the test; bf16, 128 x 128 tiles, default head map, at most 8 heads per
    group).

    wait_limit_ns: limit of every device-side wait (0 = the library's 2 s);
    small values only serve tests of the timeout path."""
    lib = load_library()
    _require_cuda(q, k, v)
    B, N, Hq, d = q.shape
    nQB, nKB = -(-N // block_q), -(-k.shape[1] // block_k)
    packed = None
    if cu_seqlens_q is not None or cu_seqlens_k is not None:
        if q.shape[0] != 1 or k.shape[0] != 1:
            raise ValueError("packed sequences take q, k, v with a batch dimension of 1")
        packed = _packed(cu_seqlens_q, cu_seqlens_k, block_q, block_k)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        shape = (Hq, N) if packed else (B, Hq, N)
        lse = torch.empty(shape, dtype=torch.float32, device=q.device)
    if keep_mask is None and with_mask:
        shape = (Hq, packed[3], mask_words(packed[4])) if packed else (B, Hq, nQB, mask_words(nKB))
        keep_mask = torch.empty(shape, dtype=torch.int32, device=q.device)
    keep_alive, hm = _head_map(q_to_kv)
    a = fwd_args(q, k, v, o, lse, keep_mask, tau, block_q, block_k, stats, hm)
    a.group_vote = 1 if group_vote else 0
    a.wait_limit_ns = int(wait_limit_ns)
    if packed:
        a.batch = packed[2]
        a.cu_seqlens_q = packed[0].ctypes.data
        a.cu_seqlens_k = packed[1].ctypes.data
    ws_n = lib.mala_fwd_workspace_size(ctypes.byref(a))
    ws = torch.empty(ws_n, dtype=torch.uint8, device=q.device) if ws_n else None
    _check(lib.mala_fwd(ctypes.byref(a), _ptr(ws), ws_n, _stream(stream)))
    _keep_for_stream(ws, stream)
    del keep_alive, packed
    return o, lse, keep_mask


def mala_bwd(q, k, v, o, do, lse, tau: float, keep_mask=None, block_q: int = 128,
             block_k: int = 128, *, dq=None, dk=None, dv=None, bwd_keep_mask=None,
             with_bwd_mask: bool = False, stats=None, q_to_kv=None, stream=None,
             cu_seqlens_q=None, cu_seqlens_k=None, wait_limit_ns: int = 0):
    """MALA backward. Returns (dq, dk, dv, bwd_keep_mask or None). Packed
    sequences as for mala_fwd (the same cu_seqlens; lse and keep_mask in
    mala_fwd's packed layouts). wait_limit_ns as for mala_fwd."""
    lib = load_library()
    _require_cuda(q, k, v, o, do, lse)
    B, N, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    nQB, nKB = -(-N // block_q), -(-Nk // block_k)
    packed = None
    if cu_seqlens_q is not None or cu_seqlens_k is not None:
        if q.shape[0] != 1 or k.shape[0] != 1:
            raise ValueError("packed sequences take q, k, v with a batch dimension of 1")
        packed = _packed(cu_seqlens_q, cu_seqlens_k, block_q, block_k)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if bwd_keep_mask is None and with_bwd_mask:
        shape = (Hq, packed[3], mask_words(packed[4])) if packed else (B, Hq, nQB, mask_words(nKB))
        bwd_keep_mask = torch.empty(shape, dtype=torch.int32, device=q.device)
    keep_alive, hm = _head_map(q_to_kv)
    a = BwdArgs()
    a.q, a.k, a.v, a.o, a.dout = _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do)
    a.lse, a.keep_mask = _ptr(lse), _ptr(keep_mask)
    a.dq, a.dk, a.dv, a.bwd_keep_mask = _ptr(dq), _ptr(dk), _ptr(dv), _ptr(bwd_keep_mask)
    a.batch, a.heads_q, a.heads_kv = B, Hq, Hkv
    a.seqlen_q, a.seqlen_k, a.head_dim = N, Nk, d
    a.q_stride, a.k_stride, a.v_stride, a.o_stride = _strides(q), _strides(k), _strides(v), _strides(o)
    a.do_stride, a.dq_stride, a.dk_stride, a.dv_stride = _strides(do), _strides(dq), _strides(dk), _strides(dv)
    a.q_to_kv = hm
    a.block_q, a.block_k = block_q, block_k
    a.tau = float(tau)
    a.dtype = _dtype_code(q)
    a.stats = _ptr(stats)
    a.wait_limit_ns = int(wait_limit_ns)
    if packed:
        a.batch = packed[2]
        a.cu_seqlens_q = packed[0].ctypes.data
        a.cu_seqlens_k = packed[1].ctypes.data
    ws_n = lib.mala_bwd_workspace_size(ctypes.byref(a))
    if ws_n == 0:
        _check(lib.mala_bwd(ctypes.byref(a), None, 0, _stream(stream)))   # reports the argument error
    ws = torch.empty(ws_n, dtype=torch.uint8, device=q.device)
    _check(lib.mala_bwd(ctypes.byref(a), _ptr(ws), ws_n, _stream(stream)))
    _keep_for_stream(ws, stream)
    del keep_alive, packed
    return dq, dk, dv, bwd_keep_mask


def _decode_cache(a, k, v, k_scale, v_scale):
    """Cache element type: bf16, or e4m3 codes with their scales."""
    fp8 = (k.dtype == torch.float8_e4m3fn, v.dtype == torch.float8_e4m3fn)
    if fp8[0] != fp8[1]:
        raise ValueError("k and v caches must have the same element type")
    a.kv_dtype = MALA_FP8_E4M3 if fp8[0] else MALA_BF16
    a.k_scale, a.v_scale = float(k_scale), float(v_scale)


def _decode_call(q, k, v, tau, block_k, num_splits, o, lse, keep_mask, with_mask, stats, q_to_kv,
                 k_scale, v_scale, group_vote, wait_limit_ns=0):
    """Output tensors and the filled argument struct of a decode call (plus
    the objects that must outlive the call)."""
    _require_cuda(q, k, v)
    B, _, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    nKB = -(-Nk // block_k)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if lse is None else lse
    if keep_mask is None and with_mask:
        keep_mask = torch.empty((B, Hq, mask_words(nKB)), dtype=torch.int32, device=q.device)
    keep_alive, hm = _head_map(q_to_kv)
    a = DecodeArgs()
    a.q, a.k, a.v, a.o = _ptr(q), _ptr(k), _ptr(v), _ptr(o)
    a.lse, a.keep_mask = _ptr(lse), _ptr(keep_mask)
    a.batch, a.heads_q, a.heads_kv, a.seqlen_k, a.head_dim = B, Hq, Hkv, Nk, d
    a.q_stride, a.k_stride, a.v_stride, a.o_stride = _strides(q), _strides(k), _strides(v), _strides(o)
    a.q_to_kv = hm
    a.block_k = block_k
    a.tau = float(tau)
    a.dtype = _dtype_code(q)
    a.num_splits = int(num_splits)
    a.stats = _ptr(stats)
    _decode_cache(a, k, v, k_scale, v_scale)
    a.group_vote = 1 if group_vote else 0
    a.wait_limit_ns = int(wait_limit_ns)
    return o, lse, keep_mask, a, keep_alive


def mala_decode(q, k, v, tau: float, block_k: int = 128, num_splits: int = 0, *, o=None,
                lse=None, keep_mask=None, with_mask: bool = True, stats=None, q_to_kv=None,
                stream=None, workspace=None, k_scale: float = 1.0, v_scale: float = 1.0,
                group_vote: bool = False, wait_limit_ns: int = 0):
    """Single-token decoding. q [B, 1, Hq, d] bf16; k/v cache [B, Nk, Hkv, d]
    in bf16, or torch.float8_e4m3fn codes whose values are code * k_scale and
    code * v_scale. group_vote: one decision per key tile for all query heads
    of a KV head (a tile is skipped only when every head passes the test).
    wait_limit_ns as for mala_fwd. Returns (o, lse [B, Hq], keep_mask words
    [B, Hq, ceil(T/32)] or None, num_splits used)."""
    lib = load_library()
    o, lse, keep_mask, a, keep_alive = _decode_call(q, k, v, tau, block_k, num_splits, o, lse, keep_mask,
                                                    with_mask, stats, q_to_kv, k_scale, v_scale, group_vote,
                                                    wait_limit_ns)
    ws_n = lib.mala_decode_workspace_size(ctypes.byref(a))
    own_ws = workspace is None or workspace.numel() < ws_n
    if own_ws:
        workspace = torch.empty(ws_n, dtype=torch.uint8, device=q.device) if ws_n else None
    _check(lib.mala_decode(ctypes.byref(a), _ptr(workspace), ws_n, _stream(stream)))
    if own_ws:
        _keep_for_stream(workspace, stream)
    del keep_alive
    return o, lse, keep_mask, int(a.num_splits)


def mala_decode_noalloc(q, k, v, tau: float, block_k: int = 128, num_splits: int = 0, *, o=None,
                        lse=None, keep_mask=None, with_mask: bool = True, stats=None, q_to_kv=None,
                        stream=None, k_scale: float = 1.0, v_scale: float = 1.0,
                        group_vote: bool = False):
    """mala_decode without a workspace: the library keeps the split partials
    in its own built-in device buffer (for callers that cannot allocate;
    calls that overlap on the GPU race on that buffer). Returns the same
    tuple as :func:`mala_decode`."""
    lib = load_library()
    o, lse, keep_mask, a, keep_alive = _decode_call(q, k, v, tau, block_k, num_splits, o, lse, keep_mask,
                                                    with_mask, stats, q_to_kv, k_scale, v_scale, group_vote)
    _check(lib.mala_decode_noalloc(ctypes.byref(a), _stream(stream)))
    del keep_alive
    return o, lse, keep_mask, int(a.num_splits)


def check_device_error(stream=None):
    """Synchronise and raise if a kernel recorded a device-side failure."""
    _check(load_library().mala_check_device_error(_stream(stream)))
