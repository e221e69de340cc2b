"""Python entry to the CPU oracle (TEST INFRASTRUCTURE).

Only the tests, __graft_entry__.smoke() and bench.py's cpu_baseline /
reference leg may import this package.  The product path (the package
block_sparse_attention_22_b200 and its CUDA library) never does.

Thin ctypes wrappers over oracle/qsa_oracle.c; every array is a contiguous
numpy array (fp32 inputs, fp64 outputs, int32/int64 indices).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

from . import build as _build

HERE = os.path.dirname(os.path.abspath(__file__))


class RefConfig(ctypes.Structure):
    _fields_ = [
        ("r", ctypes.c_int32),
        ("budget_tokens", ctypes.c_int32),
        ("n_heads", ctypes.c_int32),
        ("n_groups", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("idx_heads", ctypes.c_int32),
        ("idx_dim", ctypes.c_int32),
        ("rope_dims", ctypes.c_int32),
        ("rope_base", ctypes.c_double),
        ("softmax_scale", ctypes.c_double),
        ("round_bf16", ctypes.c_int32),
    ]


def config(r=4, budget_tokens=2048, n_heads=24, n_groups=2, head_dim=256, idx_heads=4,
           idx_dim=128, rope_dims=None, rope_base=1e7, softmax_scale=None, round_bf16=True):
    if rope_dims is None:
        rope_dims = int(idx_dim * 0.25)
        rope_dims -= rope_dims % 2
    if softmax_scale is None:
        softmax_scale = 1.0 / np.sqrt(head_dim)
    return RefConfig(r, budget_tokens, n_heads, n_groups, head_dim, idx_heads, idx_dim,
                     rope_dims, float(rope_base), float(softmax_scale), int(bool(round_bf16)))


def config_from_shape(shape) -> RefConfig:
    """Oracle config from a synth.Shape-like object."""
    return config(shape.r, shape.budget_tokens, shape.n_heads, shape.n_groups, shape.head_dim,
                  shape.idx_heads, shape.idx_dim, shape.rope_dims, shape.rope_base,
                  1.0 / np.sqrt(shape.head_dim), shape.dtype == "bf16")


_LIBS = {}

_F = ctypes.POINTER(ctypes.c_float)
_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)
_I64 = ctypes.POINTER(ctypes.c_int64)
_C = ctypes.POINTER(RefConfig)


def _lib(acc="f64"):
    name = "libqsa_oracle.so" if acc == "f64" else "libqsa_oracle_f32.so"
    if name not in _LIBS:
        # QSA_ORACLE_LIB / QSA_ORACLE_LIB_F32: another build of qsa_oracle.c (the
        # planted-mistake tests load deliberately wrong builds through these)
        override = os.environ.get("QSA_ORACLE_LIB" if acc == "f64" else "QSA_ORACLE_LIB_F32")
        if override:
            path = override
        else:
            _build.build()
            path = os.path.join(HERE, name)
        lib = ctypes.CDLL(path)
        lib.qsa_ref_round_bf16.argtypes = [ctypes.c_double]
        lib.qsa_ref_round_bf16.restype = ctypes.c_double
        lib.qsa_ref_rope_theta.argtypes = [_C, ctypes.c_int]
        lib.qsa_ref_rope_theta.restype = ctypes.c_double
        lib.qsa_ref_rope_cos_sin.argtypes = [_C, ctypes.c_int64, _F, _F]
        lib.qsa_ref_rope_vec.argtypes = [_C, _F, ctypes.c_int64, _F]
        lib.qsa_ref_compress_keys.argtypes = [_C, _F, ctypes.c_int64, ctypes.c_int64, _F]
        lib.qsa_ref_index_scores.argtypes = [_C, _F, _F, ctypes.c_int64, _F, _D]
        lib.qsa_ref_select.argtypes = [_C, _D, ctypes.c_int64, _I32]
        lib.qsa_ref_select.restype = ctypes.c_int
        lib.qsa_ref_attend.argtypes = [_C, _F, _F, _F, ctypes.c_int64, ctypes.c_int64, _I32,
                                       ctypes.c_int, _D, _D]
        lib.qsa_ref_attend_bwd.argtypes = [_C, _F, _F, _F, ctypes.c_int64, ctypes.c_int64, _I32,
                                           ctypes.c_int, _F, _D, _D, _D]
        lib.qsa_ref_forward.argtypes = [_C, _F, _F, _F, _I64, ctypes.c_int64, _F, _F, _F,
                                        ctypes.c_int64, _I32, _I32, _D, _D, ctypes.c_int]
        lib.qsa_ref_acc_bits.restype = ctypes.c_int
        _LIBS[name] = lib
    return _LIBS[name]


def _f32(a):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    return a, a.ctypes.data_as(_F)


def _p(a, t):
    return a.ctypes.data_as(t)


def round_bf16(x: float, acc="f64") -> float:
    return _lib(acc).qsa_ref_round_bf16(float(x))


def rope_theta(cfg: RefConfig, i: int) -> float:
    return _lib().qsa_ref_rope_theta(ctypes.byref(cfg), i)


def rope_cos_sin(cfg: RefConfig, pos: int):
    half = cfg.rope_dims // 2
    c = np.zeros(max(half, 1), np.float32)
    s = np.zeros(max(half, 1), np.float32)
    _lib().qsa_ref_rope_cos_sin(ctypes.byref(cfg), pos, _p(c, _F), _p(s, _F))
    return c[:half], s[:half]


def rope_vec(cfg: RefConfig, x, pos: int, acc="f64") -> np.ndarray:
    x, px = _f32(x)
    out = np.zeros_like(x)
    _lib(acc).qsa_ref_rope_vec(ctypes.byref(cfg), px, pos, _p(out, _F))
    return out


def compress_keys(cfg: RefConfig, k_idx, b0: int, b1: int, acc="f64") -> np.ndarray:
    """k^ for blocks [b0, b1) of one sequence; k_idx is [n, idx_dim]."""
    k_idx, pk = _f32(k_idx)
    out = np.zeros((max(b1 - b0, 0), cfg.idx_dim), np.float32)
    _lib(acc).qsa_ref_compress_keys(ctypes.byref(cfg), pk, b0, b1, _p(out, _F))
    return out


def index_scores(cfg: RefConfig, q_idx, w, t: int, khat, acc="f64") -> np.ndarray:
    """Scores of the query at position t against blocks [0, t // r)."""
    q_idx, pq = _f32(q_idx)
    w, pw = _f32(w)
    khat, pk = _f32(khat)
    bt = t // cfg.r
    assert khat.shape[0] >= bt
    out = np.zeros(max(bt, 1), np.float64)
    _lib(acc).qsa_ref_index_scores(ctypes.byref(cfg), pq, pw, t, pk, _p(out, _D))
    return out[:bt]


def select(cfg: RefConfig, scores, t: int, acc="f64"):
    """(sel[S] ascending, -1 padded; nsel) for the query at position t."""
    S = cfg.budget_tokens // cfg.r
    bt = t // cfg.r
    s = np.ascontiguousarray(np.asarray(scores, dtype=np.float64))
    if s.size < max(bt, 1):
        s = np.concatenate([s, np.zeros(max(bt, 1) - s.size)])
    sel = np.zeros(S, np.int32)
    n = _lib(acc).qsa_ref_select(ctypes.byref(cfg), _p(s, _D), t, _p(sel, _I32))
    return sel, n


def attend(cfg: RefConfig, q, k, v, t: int, sel, nsel: int, acc="f64"):
    """Attention of one query; k, v are the sequence's [G, ld, D] caches."""
    q, pq = _f32(q)
    k, pk = _f32(k)
    v, pv = _f32(v)
    sel = np.ascontiguousarray(np.asarray(sel, dtype=np.int32))
    o = np.zeros((cfg.n_heads, cfg.head_dim), np.float64)
    lse = np.zeros(cfg.n_heads, np.float64)
    _lib(acc).qsa_ref_attend(ctypes.byref(cfg), pq, pk, pv, k.shape[1], t, _p(sel, _I32), nsel,
                             _p(o, _D), _p(lse, _D))
    return o, lse


def attend_bwd(cfg: RefConfig, q, k, v, t: int, sel, nsel: int, dout, dk=None, dv=None, acc="f64"):
    """Backward of one query's attention for the loss sum(dout * o): returns dq
    [H, D]; adds this query's contributions to dk, dv ([G, ld, D] float64, created
    zero if not given) and returns them too."""
    q, pq = _f32(q)
    k, pk = _f32(k)
    v, pv = _f32(v)
    dout, pdo = _f32(dout)
    sel = np.ascontiguousarray(np.asarray(sel, dtype=np.int32))
    dq = np.zeros((cfg.n_heads, cfg.head_dim), np.float64)
    if dk is None:
        dk = np.zeros(k.shape, np.float64)
    if dv is None:
        dv = np.zeros(v.shape, np.float64)
    assert dk.dtype == np.float64 and dk.flags.c_contiguous and dk.shape == k.shape
    assert dv.dtype == np.float64 and dv.flags.c_contiguous and dv.shape == v.shape
    _lib(acc).qsa_ref_attend_bwd(ctypes.byref(cfg), pq, pk, pv, k.shape[1], t, _p(sel, _I32), nsel, pdo,
                                 _p(dq, _D), _p(dk, _D), _p(dv, _D))
    return dq, dk, dv


def forward(cfg: RefConfig, q, q_idx, w, pos, k_idx, k, v, acc="f64",
            n_threads: int = 0):
    """The whole path for query tokens of ONE sequence.

    q [nq,H,D], q_idx [nq,Hi,dI], w [nq,Hi], pos [nq] (absolute positions),
    k_idx [n,dI], k/v [G,ld,D].  Returns dict(sel, nsel, o, lse).
    """
    q, pq = _f32(q)
    q_idx, pqi = _f32(q_idx)
    w, pw = _f32(w)
    k_idx, pki = _f32(k_idx)
    k, pk = _f32(k)
    v, pv = _f32(v)
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    nq = pos.size
    S = cfg.budget_tokens // cfg.r
    sel = np.zeros((nq, S), np.int32)
    nsel = np.zeros(nq, np.int32)
    o = np.zeros((nq, cfg.n_heads, cfg.head_dim), np.float64)
    lse = np.zeros((nq, cfg.n_heads), np.float64)
    _lib(acc).qsa_ref_forward(ctypes.byref(cfg), pq, pqi, pw, _p(pos, _I64), nq, pki, pk, pv,
                              k.shape[1], _p(sel, _I32), _p(nsel, _I32), _p(o, _D), _p(lse, _D),
                              int(n_threads))
    return {"sel": sel, "nsel": nsel, "o": o, "lse": lse}


def acc_bits(acc="f64") -> int:
    return _lib(acc).qsa_ref_acc_bits()
