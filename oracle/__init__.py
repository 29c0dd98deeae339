"""Plain CPU oracle for the TokenGate gated-prefill hot path (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use this package.  The product library never imports it and it
imports nothing from the product library.  The arithmetic lives in
``tg_oracle.c`` (fp64, plain loops, OpenMP over independent rows); this module
only builds it, marshals numpy arrays and returns numpy results.

Each function cites the passage it follows in the C source.  Method source:
TokenGate, "Adapting LLMs for Fast and Memory-Efficient Prefill with Learned
Token Pruning" (abstract page) and the news write-ups' "how it works" sections.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tg_oracle.c")
_LIB = os.path.join(_HERE, "libtg_oracle.so")
_lib = None

_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile tg_oracle.c into libtg_oracle.so (gcc -O2 -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        L.tgo_num_threads.restype = ctypes.c_int
        L.tgo_gate_score.argtypes = [_f32p, ctypes.c_int64, ctypes.c_int32, _f32p, _f32p,
                                     ctypes.c_int32, _f32p, ctypes.c_double, _i64p,
                                     ctypes.c_int64, _f64p]
        L.tgo_topk_select.argtypes = [_f32p, ctypes.c_int32, _i32p, _i32p, _i32p, _i32p,
                                      _i32p, _i32p]
        L.tgo_select_by_keys.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int32, _i32p,
                                         _i32p, _i32p, _i32p, _i32p, _i32p]
        L.tgo_gather_rows.argtypes = [_i32p, ctypes.c_int64, ctypes.c_int32, _i32p, _f32p,
                                      ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_double, _f64p]
        L.tgo_logsig.argtypes = [_i32p, ctypes.c_int64, ctypes.c_int32, _i32p, _i32p, _i32p,
                                 _f32p, _f64p]
        L.tgo_gated_attention.argtypes = [_f32p, _f32p, _f32p, ctypes.c_int32, _i32p,
                                          ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                          _f32p, _f32p, _f32p, _i64p, ctypes.c_int64, _f64p,
                                          _f64p]
        L.tgo_attention_loss.argtypes = [_f32p, _f32p, _f32p, ctypes.c_int32, _i32p, ctypes.c_int32,
                                         ctypes.c_int32, ctypes.c_int32, _f64p, _f64p, _f64p, _f32p,
                                         _f64p]
        L.tgo_gated_attention_backward.argtypes = [_f32p, _f32p, _f32p, ctypes.c_int32, _i32p,
                                                   ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                   _f64p, _f64p, _f64p, _f32p, _f64p, _f64p, _f64p]
        for name in ("tgo_gate_score", "tgo_topk_select", "tgo_select_by_keys",
                     "tgo_gather_rows", "tgo_logsig", "tgo_gated_attention", "tgo_attention_loss",
                     "tgo_gated_attention_backward"):
            getattr(L, name).restype = ctypes.c_int
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a, ctype):
    return None if a is None else a.ctypes.data_as(ctype)


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"oracle {name}: invalid arguments")


def num_threads() -> int:
    return int(_load().tgo_num_threads())


def gate_score(h, W1, b1, w2, b2, rows=None) -> np.ndarray:
    """z_j = w2 . GELU(W1 h_j + b1) + b2 in fp64 (exact-erf GELU).

    ``h`` [n, d] and ``W1`` [dg, d] hold the stored (bf16 or fp32) values as
    float32; ``rows`` optionally restricts scoring to a list of token rows.
    """
    L = _load()
    h = _c(h, np.float32)
    W1 = _c(W1, np.float32)
    b1 = _c(b1, np.float32)
    w2 = _c(w2, np.float32)
    n, d = h.shape
    dg = W1.shape[0]
    assert W1.shape[1] == d and b1.shape == (dg,) and w2.shape == (dg,)
    r = None if rows is None else _c(rows, np.int64)
    cnt = n if r is None else r.shape[0]
    out = np.empty(cnt, np.float64)
    _check(L.tgo_gate_score(_p(h, _f32p), n, d, _p(W1, _f32p), _p(b1, _f32p), dg,
                            _p(w2, _f32p), float(b2), _p(r, _i64p), cnt, _p(out, _f64p)),
           "gate_score")
    return out


def topk_select(z, cu_seqlens, doc_begin, doc_end, budget):
    """Per-prompt top-K of the document span, question protected.

    Returns (kept_idx [M] int32 global rows ascending per prompt, cu_kept [B+1]).
    """
    L = _load()
    z = _c(z, np.float32)
    cu = _c(cu_seqlens, np.int32)
    s = _c(doc_begin, np.int32)
    e = _c(doc_end, np.int32)
    k = _c(budget, np.int32)
    B = s.shape[0]
    kept = np.empty(max(int(cu[-1]), 1), np.int32)
    cu_kept = np.empty(B + 1, np.int32)
    _check(L.tgo_topk_select(_p(z, _f32p), B, _p(cu, _i32p), _p(s, _i32p), _p(e, _i32p),
                             _p(k, _i32p), _p(kept, _i32p), _p(cu_kept, _i32p)), "topk_select")
    return kept[: int(cu_kept[-1])].copy(), cu_kept


def select_by_keys(keys, cu_seqlens, doc_begin, doc_end, budget):
    """Random-K selection: per prompt, the K document tokens with the largest
    caller-drawn uint32 keys (lower index on ties), question protected.

    Returns (kept_idx [M] int32 global rows ascending per prompt, cu_kept [B+1]).
    """
    L = _load()
    keys = np.ascontiguousarray(keys, np.uint32)
    cu = _c(cu_seqlens, np.int32)
    s = _c(doc_begin, np.int32)
    e = _c(doc_end, np.int32)
    k = _c(budget, np.int32)
    B = s.shape[0]
    kept = np.empty(max(int(cu[-1]), 1), np.int32)
    cu_kept = np.empty(B + 1, np.int32)
    _check(L.tgo_select_by_keys(keys.ctypes.data_as(ctypes.POINTER(ctypes.c_uint32)), B,
                                _p(cu, _i32p), _p(s, _i32p), _p(e, _i32p), _p(k, _i32p),
                                _p(kept, _i32p), _p(cu_kept, _i32p)), "select_by_keys")
    return kept[: int(cu_kept[-1])].copy(), cu_kept


def gather_rows(kept_idx, cu_seqlens, src, rope_heads=0, head_dim=0, theta=1e6):
    """Compacted rows src[kept_idx] (fp64), optionally RoPE-rotated per head at
    each row's original in-prompt position."""
    L = _load()
    kept = _c(kept_idx, np.int32)
    cu = _c(cu_seqlens, np.int32)
    src2 = _c(src, np.float32).reshape(src.shape[0], -1)
    M = kept.shape[0]
    width = src2.shape[1]
    out = np.empty((M, width), np.float64)
    _check(L.tgo_gather_rows(_p(kept, _i32p), M, cu.shape[0] - 1, _p(cu, _i32p),
                             _p(src2, _f32p), width, rope_heads, head_dim, float(theta),
                             _p(out, _f64p)), "gather_rows")
    return out.reshape((M,) + tuple(src.shape[1:]))


def logsig(kept_idx, cu_seqlens, doc_begin, doc_end, z):
    """l_i = log sigmoid(z[kept_i]) for document tokens, 0 for question tokens."""
    L = _load()
    kept = _c(kept_idx, np.int32)
    cu = _c(cu_seqlens, np.int32)
    s = _c(doc_begin, np.int32)
    e = _c(doc_end, np.int32)
    z = _c(z, np.float32)
    out = np.empty(kept.shape[0], np.float64)
    _check(L.tgo_logsig(_p(kept, _i32p), kept.shape[0], s.shape[0], _p(cu, _i32p),
                        _p(s, _i32p), _p(e, _i32p), _p(z, _f32p), _p(out, _f64p)), "logsig")
    return out


def gated_attention(q, k, v, cu_kept, logsig=None, gain=None, temp=None, rows=None):
    """Token-gated causal GQA attention in fp64.

    q [M, Hq, dh], k/v [M, Hkv, dh] (stored values as float32), logsig [M] or
    None (no bias), gain/temp [Hq].  Returns (out [R, Hq, dh], lse [R, Hq]) for
    the listed query rows (all M when ``rows`` is None).
    """
    L = _load()
    q = _c(q, np.float32)
    k = _c(k, np.float32)
    v = _c(v, np.float32)
    cu = _c(cu_kept, np.int32)
    M, Hq, dh = q.shape
    Hkv = k.shape[1]
    gain = _c(np.zeros(Hq) if gain is None else gain, np.float32)
    temp = _c(np.ones(Hq) if temp is None else temp, np.float32)
    ls = None if logsig is None else _c(logsig, np.float32)
    r = None if rows is None else _c(rows, np.int64)
    cnt = M if r is None else r.shape[0]
    out = np.empty((cnt, Hq, dh), np.float64)
    lse = np.empty((cnt, Hq), np.float64)
    _check(L.tgo_gated_attention(_p(q, _f32p), _p(k, _f32p), _p(v, _f32p), cu.shape[0] - 1,
                                 _p(cu, _i32p), Hq, Hkv, dh, _p(ls, _f32p), _p(gain, _f32p),
                                 _p(temp, _f32p), _p(r, _i64p), cnt, _p(out, _f64p),
                                 _p(lse, _f64p)), "gated_attention")
    return out, lse


def _bwd_args(q, k, v, cu_kept, logsig, gain, temp, dout):
    q = _c(q, np.float32)
    k = _c(k, np.float32)
    v = _c(v, np.float32)
    dout = _c(dout, np.float32)
    cu = _c(cu_kept, np.int32)
    ls = _c(logsig, np.float64)
    g = _c(gain, np.float64)
    t = _c(temp, np.float64)
    M, Hq, dh = q.shape
    assert dout.shape == q.shape and ls.shape == (M,) and g.shape == (Hq,) and t.shape == (Hq,)
    return q, k, v, dout, cu, ls, g, t, Hq, k.shape[1], dh


def attention_loss(q, k, v, cu_kept, logsig, gain, temp, dout) -> float:
    """L = sum(dout * out) of the gated attention in fp64 (double log-gates, gains
    and temperatures), the scalar whose gradient gated_attention_backward gives."""
    L = _load()
    q, k, v, dout, cu, ls, g, t, Hq, Hkv, dh = _bwd_args(q, k, v, cu_kept, logsig, gain, temp, dout)
    out = np.zeros(1, np.float64)
    _check(L.tgo_attention_loss(_p(q, _f32p), _p(k, _f32p), _p(v, _f32p), cu.shape[0] - 1,
                                _p(cu, _i32p), Hq, Hkv, dh, _p(ls, _f64p), _p(g, _f64p),
                                _p(t, _f64p), _p(dout, _f32p), _p(out, _f64p)), "attention_loss")
    return float(out[0])


def gated_attention_backward(q, k, v, cu_kept, logsig, gain, temp, dout):
    """Exact fp64 gradient of sum(dout * out) with respect to the log-gates l
    [M], the gains g [Hq] and the temperatures tau [Hq]."""
    L = _load()
    q, k, v, dout, cu, ls, g, t, Hq, Hkv, dh = _bwd_args(q, k, v, cu_kept, logsig, gain, temp, dout)
    M = q.shape[0]
    d_l = np.zeros(max(M, 1), np.float64)
    d_g = np.zeros(Hq, np.float64)
    d_t = np.zeros(Hq, np.float64)
    _check(L.tgo_gated_attention_backward(_p(q, _f32p), _p(k, _f32p), _p(v, _f32p),
                                          cu.shape[0] - 1, _p(cu, _i32p), Hq, Hkv, dh,
                                          _p(ls, _f64p), _p(g, _f64p), _p(t, _f64p),
                                          _p(dout, _f32p), _p(d_l, _f64p), _p(d_g, _f64p),
                                          _p(d_t, _f64p)), "gated_attention_backward")
    return d_l[:M], d_g, d_t
