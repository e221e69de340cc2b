"""QSA forward pass on B200: a thin Python binding over libqsa.so (include/qsa.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (device memory and streams come from
PyTorch); each call enqueues on the current torch stream unless one is given.
The first call fails loudly (ImportError) if the CUDA library has not been
built; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Iterable, Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqsa.so")

(QSA_OK, QSA_ERR_INVALID_ARG, QSA_ERR_UNSUPPORTED, QSA_ERR_WORKSPACE, QSA_ERR_CUDA, QSA_ERR_TIMEOUT,
 QSA_ERR_BAD_INDEX) = range(7)
QSA_DTYPE_F32, QSA_DTYPE_BF16 = 0, 1
(QSA_OP_COMPRESS, QSA_OP_INDEX, QSA_OP_SELECT, QSA_OP_ATTN, QSA_OP_FORWARD, QSA_OP_FORWARD_LOWMEM,
 QSA_OP_ATTN_UNION, QSA_OP_FORWARD_PREFIXED) = range(8)


class qsa_config_t(ctypes.Structure):
    _fields_ = [("r", ctypes.c_int32), ("budget_tokens", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("n_kv_groups", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("idx_heads", ctypes.c_int32),
                ("idx_dim", ctypes.c_int32), ("rope_fraction", ctypes.c_float),
                ("rope_base", ctypes.c_double), ("softmax_scale", ctypes.c_float),
                ("dtype", ctypes.c_int)]


class qsa_segment_t(ctypes.Structure):
    _fields_ = [("q_offset", ctypes.c_int32), ("q_len", ctypes.c_int32),
                ("pos0", ctypes.c_int32), ("slot", ctypes.c_int32)]


class qsa_prefix_t(ctypes.Structure):
    _fields_ = [("slot", ctypes.c_int32), ("blocks", ctypes.c_int32)]


class qsa_cache_t(ctypes.Structure):
    _fields_ = [("k_idx", ctypes.c_void_p), ("khat", ctypes.c_void_p), ("k", ctypes.c_void_p),
                ("v", ctypes.c_void_p), ("n_slots", ctypes.c_int32), ("n_cap", ctypes.c_int64)]


class QSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libqsa.so not built at {LIB_PATH}; run block_sparse_attention_22_b200/build.py "
                          "or __graft_entry__.build()")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    C = ctypes.POINTER(qsa_config_t)
    K = ctypes.POINTER(qsa_cache_t)
    S = ctypes.POINTER(qsa_segment_t)
    sig = {
        "qsa_compress_keys": [C, K, P, P, P, I32, P],
        "qsa_index_scores": [C, K, S, I32, I32, P, P, P, I64, P],
        "qsa_select_topk": [C, S, I32, I32, P, I64, P, P, P, SZ, P],
        "qsa_sparse_attn_fwd": [C, K, S, I32, I32, P, P, P, P, P, P, SZ, P],
        "qsa_sparse_attn_fwd_union": [C, K, S, I32, I32, P, P, P, P, P, P, SZ, P],
        "qsa_sparse_attn_bwd": [C, K, S, I32, I32, P, P, P, P, P, P, P, P, P, P],
        "qsa_forward": [C, K, S, I32, I32, P, P, P, P, P, P, P, P, SZ, P],
        "qsa_forward_lowmem": [C, K, S, I32, I32, P, P, P, P, P, P, P, P, SZ, P],
        "qsa_forward_prefixed": [C, K, S, ctypes.POINTER(qsa_prefix_t), I32, I32, P, P, P, P, P, P, P, P, SZ, P],
        "qsa_device_status": [P],
        "qsa_select_fallbacks": [P, ctypes.POINTER(ctypes.c_int64)],
        "qsa_selftest_wait_timeout": [P],
        "qsa_select_topk_noalloc": [C, S, I32, I32, P, I64, P, P, P],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.qsa_workspace_size.argtypes = [C, S, I32, I32, ctypes.c_int]
    lib.qsa_workspace_size.restype = SZ
    lib.qsa_status_string.argtypes = [ctypes.c_int]
    lib.qsa_status_string.restype = ctypes.c_char_p
    lib.qsa_version.restype = I32
    lib.qsa_launch_count.restype = I64
    return lib


_LIB = None


def get_lib():
    """The loaded libqsa.so (loaded on first use)."""
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def status_string(status: int) -> str:
    return get_lib().qsa_status_string(status).decode()


def _check(status: int, where: str):
    if status != QSA_OK:
        raise QSAError(status, where)


def make_config(shape, softmax_scale: float = 0.0) -> qsa_config_t:
    """qsa_config_t from a synth.Shape-like object."""
    return qsa_config_t(shape.r, shape.budget_tokens, shape.n_heads, shape.n_groups, shape.head_dim,
                        shape.idx_heads, shape.idx_dim, shape.rope_fraction, shape.rope_base,
                        softmax_scale, QSA_DTYPE_BF16 if shape.dtype == "bf16" else QSA_DTYPE_F32)


def make_segments(segs: Iterable[Sequence[int]]):
    """Array of qsa_segment_t from (q_offset, q_len, pos0, slot) tuples."""
    segs = list(segs)
    arr = (qsa_segment_t * max(1, len(segs)))()
    for i, (off, n, p0, slot) in enumerate(segs):
        arr[i] = qsa_segment_t(off, n, p0, slot)
    return arr, len(segs)


def make_prefixes(prefixes: Iterable[Sequence[int]]):
    """Array of qsa_prefix_t from (slot, blocks) pairs, one per segment."""
    prefixes = list(prefixes)
    arr = (qsa_prefix_t * max(1, len(prefixes)))()
    for i, (slot, blocks) in enumerate(prefixes):
        arr[i] = qsa_prefix_t(slot, blocks)
    return arr


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def make_cache(k_idx, khat, k, v) -> qsa_cache_t:
    """Caches: k_idx [slots,N,dI], khat [slots,N/r,dI], k/v [slots,G,N,D] (CUDA tensors)."""
    return qsa_cache_t(_ptr(k_idx), _ptr(khat), _ptr(k), _ptr(v), k.shape[0], k.shape[2])


def _stream(stream) -> int:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def workspace_size(cfg, segs, n_tokens: int, op: int) -> int:
    arr, n = segs
    return int(get_lib().qsa_workspace_size(ctypes.byref(cfg), arr, n, n_tokens, op))


def qsa_compress_keys(cfg, cache, slots, blk_begin, blk_end, stream=None):
    n = len(slots)
    s = (ctypes.c_int32 * max(1, n))(*slots)
    b0 = (ctypes.c_int64 * max(1, n))(*blk_begin)
    b1 = (ctypes.c_int64 * max(1, n))(*blk_end)
    _check(get_lib().qsa_compress_keys(ctypes.byref(cfg), ctypes.byref(cache), s, b0, b1, n, _stream(stream)),
           "qsa_compress_keys")


def qsa_index_scores(cfg, cache, segs, n_tokens, q_idx, w, scores, ld_scores, stream=None):
    arr, n = segs
    _check(get_lib().qsa_index_scores(ctypes.byref(cfg), ctypes.byref(cache), arr, n, n_tokens, _ptr(q_idx),
                                _ptr(w), _ptr(scores), ld_scores, _stream(stream)), "qsa_index_scores")


def qsa_select_topk(cfg, segs, n_tokens, scores, ld_scores, sel, nsel, workspace=None, stream=None):
    arr, n = segs
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(get_lib().qsa_select_topk(ctypes.byref(cfg), arr, n, n_tokens, _ptr(scores), ld_scores, _ptr(sel),
                               _ptr(nsel), _ptr(workspace), ws_bytes, _stream(stream)), "qsa_select_topk")


def qsa_select_topk_noalloc(cfg, segs, n_tokens, scores, ld_scores, sel, nsel, stream=None):
    """qsa_select_topk with its scratch in the library's static device array
    (no workspace argument; for callers that cannot allocate device memory)."""
    arr, n = segs
    _check(get_lib().qsa_select_topk_noalloc(ctypes.byref(cfg), arr, n, n_tokens, _ptr(scores), ld_scores,
                                             _ptr(sel), _ptr(nsel), _stream(stream)), "qsa_select_topk_noalloc")


def qsa_sparse_attn_fwd(cfg, cache, segs, n_tokens, q, sel, nsel, o, lse=None, workspace=None,
                        stream=None):
    arr, n = segs
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(get_lib().qsa_sparse_attn_fwd(ctypes.byref(cfg), ctypes.byref(cache), arr, n, n_tokens, _ptr(q),
                                   _ptr(sel), _ptr(nsel), _ptr(o), _ptr(lse), _ptr(workspace), ws_bytes,
                                   _stream(stream)), "qsa_sparse_attn_fwd")


def qsa_sparse_attn_fwd_union(cfg, cache, segs, n_tokens, q, sel, nsel, o, lse=None, workspace=None,
                              stream=None):
    """qsa_sparse_attn_fwd on tiles of neighbouring queries that gather the union
    of their kept blocks once (workspace: QSA_OP_ATTN_UNION; bf16 only)."""
    arr, n = segs
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(get_lib().qsa_sparse_attn_fwd_union(ctypes.byref(cfg), ctypes.byref(cache), arr, n, n_tokens,
                                               _ptr(q), _ptr(sel), _ptr(nsel), _ptr(o), _ptr(lse),
                                               _ptr(workspace), ws_bytes, _stream(stream)),
           "qsa_sparse_attn_fwd_union")


def qsa_sparse_attn_bwd(cfg, cache, segs, n_tokens, q, o, lse, dout, sel, nsel, dq, dk, dv, stream=None):
    """Backward of qsa_sparse_attn_fwd: writes dq (fp32 [T,H,D]); adds into dk, dv
    (fp32, laid out like the K/V caches)."""
    arr, n = segs
    _check(get_lib().qsa_sparse_attn_bwd(ctypes.byref(cfg), ctypes.byref(cache), arr, n, n_tokens, _ptr(q),
                                         _ptr(o), _ptr(lse), _ptr(dout), _ptr(sel), _ptr(nsel), _ptr(dq),
                                         _ptr(dk), _ptr(dv), _stream(stream)), "qsa_sparse_attn_bwd")


def qsa_forward(cfg, cache, segs, n_tokens, q, q_idx, w, o, lse=None, sel=None, nsel=None,
                workspace=None, stream=None):
    arr, n = segs
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(get_lib().qsa_forward(ctypes.byref(cfg), ctypes.byref(cache), arr, n, n_tokens, _ptr(q), _ptr(q_idx),
                           _ptr(w), _ptr(o), _ptr(lse), _ptr(sel), _ptr(nsel), _ptr(workspace), ws_bytes,
                           _stream(stream)), "qsa_forward")


def qsa_forward_lowmem(cfg, cache, segs, n_tokens, q, q_idx, w, o, lse=None, sel=None, nsel=None,
                       workspace=None, stream=None):
    """qsa_forward without the score matrix (workspace: QSA_OP_FORWARD_LOWMEM)."""
    arr, n = segs
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(get_lib().qsa_forward_lowmem(ctypes.byref(cfg), ctypes.byref(cache), arr, n, n_tokens, _ptr(q),
                                        _ptr(q_idx), _ptr(w), _ptr(o), _ptr(lse), _ptr(sel), _ptr(nsel),
                                        _ptr(workspace), ws_bytes, _stream(stream)), "qsa_forward_lowmem")


def qsa_forward_prefixed(cfg, cache, segs, prefixes, n_tokens, q, q_idx, w, o, lse=None, sel=None, nsel=None,
                         workspace=None, stream=None):
    """qsa_forward for sequences that share cached prefixes: prefixes is the
    make_prefixes() array, one (slot, blocks) per segment (workspace:
    QSA_OP_FORWARD_PREFIXED)."""
    arr, n = segs
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(get_lib().qsa_forward_prefixed(ctypes.byref(cfg), ctypes.byref(cache), arr, prefixes, n, n_tokens,
                                          _ptr(q), _ptr(q_idx), _ptr(w), _ptr(o), _ptr(lse), _ptr(sel), _ptr(nsel),
                                          _ptr(workspace), ws_bytes, _stream(stream)), "qsa_forward_prefixed")


def qsa_device_status(stream=None):
    _check(get_lib().qsa_device_status(_stream(stream)), "qsa_device_status")


def device_status(stream=None) -> int:
    """Status code of qsa_device_status (reads and clears the device error word)."""
    return int(get_lib().qsa_device_status(_stream(stream)))


def select_fallbacks(stream=None) -> int:
    """Rows whose selection took the exact fallback since the last call (reads and clears)."""
    n = ctypes.c_int64(0)
    _check(get_lib().qsa_select_fallbacks(_stream(stream), ctypes.byref(n)), "qsa_select_fallbacks")
    return int(n.value)


def qsa_selftest_wait_timeout(stream=None):
    """Enqueue the bounded-wait diagnostic (a wait that runs out after ~0.1 s)."""
    _check(get_lib().qsa_selftest_wait_timeout(_stream(stream)), "qsa_selftest_wait_timeout")


def launch_count() -> int:
    """Kernels the library has enqueued so far in this process."""
    return int(get_lib().qsa_launch_count())


def version() -> int:
    return int(get_lib().qsa_version())
