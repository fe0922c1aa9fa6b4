"""fp64 CPU oracle for exact softmax attention -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline leg (and
its ``--impl reference`` arm) may import this package.  The product path (the
CUDA library and its Python binding) never touches it, and the two share no
code: the only module both sides use is the seeded input generator, which holds
none of the method's arithmetic.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64); this module only
marshals arrays.  Sources of each definition (FlashAttention teaching pages):

* ``attention_rows`` -- the standard three-step computation, S = scale·QKᵀ,
  P = softmax(S), O = PV ("GPU 学习日报 Day 21", section 3.1), with the safe
  two-pass softmax of section 5.1, the causal mask of the section 6 table, and
  LSE = m + ln Σ e^{s-m} as the saved statistic (airsota "science-depth-m4-047",
  section 3 point (c)).
* ``attention_rows_online`` -- the one-pass recurrence of sections 5.2/5.3 of
  the same page, in fp64, used only as a pin against ``attention_rows``.
* ``softmax_two_pass`` / ``online_softmax`` -- the vector softmax of sections
  5.1/5.2 and practice exercise 2 (online vs two-pass).
* ``prob_row`` -- the probability row P_i of ``attention_rows``.
* ``attention_qk`` -- the same definition for Nq query rows against Nk keys
  (non-causal; the decode case Nq = 1 of "GPU 学习日报 Day 21", section 9 and FAQ Q5).
* ``attention_backward`` -- gradients of sum(dO * O) with respect to q, k, v:
  the chain rule through the three steps, every N x N matrix materialised
  (the gradients the backward pass recomputes from saved statistics,
  "science-depth-m4-047" section 3 point (c)).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        lib.oracle_softmax_two_pass.argtypes = [dp, i64, dp]
        lib.oracle_online_softmax.argtypes = [dp, i64, i64, dp, dp, dp, dp]
        lib.oracle_attention_rows.argtypes = [dp, dp, dp, i64, i64, i64, ctypes.c_int,
                                              ctypes.c_double, i64p, i64p, i64, dp, dp,
                                              ctypes.c_int]
        lib.oracle_attention_rows_online.argtypes = [dp, dp, dp, i64, i64, i64, ctypes.c_int,
                                                     ctypes.c_double, i64, i64p, i64p, i64,
                                                     dp, dp, ctypes.c_int]
        lib.oracle_attention_prob_row.argtypes = [dp, dp, dp, i64, i64, i64, ctypes.c_int,
                                                  ctypes.c_double, i64, i64, dp]
        lib.oracle_attention_rows_qk.argtypes = [dp, dp, dp, i64, i64, i64, i64, ctypes.c_double,
                                                 i64p, i64p, i64, dp, dp, ctypes.c_int]
        lib.oracle_attention_backward.argtypes = [dp, dp, dp, dp, i64, i64, ctypes.c_int,
                                                  ctypes.c_double, dp, dp, dp, ctypes.c_int]
        for fn in (lib.oracle_softmax_two_pass, lib.oracle_online_softmax,
                   lib.oracle_attention_rows, lib.oracle_attention_rows_online,
                   lib.oracle_attention_prob_row, lib.oracle_attention_rows_qk,
                   lib.oracle_attention_backward):
            fn.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def _dptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _iptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


def _f64(x) -> np.ndarray:
    """Widen to contiguous fp64 (exact for bf16/fp16/fp32 inputs)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def softmax_two_pass(x) -> np.ndarray:
    x = _f64(x).reshape(-1)
    p = np.empty_like(x)
    if _lib().oracle_softmax_two_pass(_dptr(x), x.size, _dptr(p)) != 0:
        raise ValueError("softmax_two_pass: bad arguments")
    return p


def online_softmax(x, block: int):
    """Returns (p, m, l, factors): probabilities, final max, final sum and the
    correction factor e^{m_old - m_new} of every block."""
    x = _f64(x).reshape(-1)
    p = np.empty_like(x)
    nb = (x.size + block - 1) // block
    factors = np.empty(max(nb, 1), dtype=np.float64)
    m = ctypes.c_double()
    l = ctypes.c_double()
    rc = _lib().oracle_online_softmax(_dptr(x), x.size, block, _dptr(p),
                                      ctypes.byref(m), ctypes.byref(l), _dptr(factors))
    if rc != 0:
        raise ValueError("online_softmax: bad arguments")
    return p, m.value, l.value, factors[:nb]


def _rows_for(N: int, rows):
    if rows is None:
        return np.arange(N, dtype=np.int64)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))


def attention_rows(q, k, v, causal: bool, scale: float, rows=None, heads=None,
                   nthreads: int | None = None, block: int = 0):
    """Oracle O and LSE for the given query rows of the given heads.

    q, k, v: [B, H, N, d] (torch or numpy, any float dtype; widened to fp64).
    heads: iterable of flat head indices b*H + h (default: all heads).
    rows: query-row indices used for every listed head (default: all rows).
    block: 0 for the three-step definition; > 0 for the online recurrence
    with that many keys per block.
    Returns (O [len(heads), len(rows), d] fp64, LSE [len(heads), len(rows)] fp64).
    """
    shape = tuple(q.shape)
    if len(shape) != 4 or tuple(k.shape) != shape or tuple(v.shape) != shape:
        raise ValueError("q, k, v must share one [B, H, N, d] shape")
    B, H, N, d = shape
    BH = B * H
    heads = list(range(BH)) if heads is None else [int(h) for h in heads]
    rows = _rows_for(N, rows)
    nthreads = default_threads() if nthreads is None else int(nthreads)
    qf = q.reshape(BH, N, d)
    kf = k.reshape(BH, N, d)
    vf = v.reshape(BH, N, d)
    O = np.empty((len(heads), rows.size, d), dtype=np.float64)
    L = np.empty((len(heads), rows.size), dtype=np.float64)
    lib = _lib()
    zeros = np.zeros(rows.size, dtype=np.int64)
    for n, bh in enumerate(heads):
        qh = _f64(qf[bh])
        kh = _f64(kf[bh])
        vh = _f64(vf[bh])
        o = np.empty((rows.size, d), dtype=np.float64)
        lse = np.empty(rows.size, dtype=np.float64)
        if block > 0:
            rc = lib.oracle_attention_rows_online(_dptr(qh), _dptr(kh), _dptr(vh), 1, N, d,
                                                  int(bool(causal)), float(scale), int(block),
                                                  _iptr(zeros), _iptr(rows), rows.size,
                                                  _dptr(o), _dptr(lse), nthreads)
        else:
            rc = lib.oracle_attention_rows(_dptr(qh), _dptr(kh), _dptr(vh), 1, N, d,
                                           int(bool(causal)), float(scale), _iptr(zeros),
                                           _iptr(rows), rows.size, _dptr(o), _dptr(lse),
                                           nthreads)
        if rc != 0:
            raise ValueError(f"oracle failed with status {rc}")
        O[n] = o
        L[n] = lse
    return O, L


def attention_rows_online(q, k, v, causal: bool, scale: float, block: int, rows=None,
                          heads=None, nthreads: int | None = None):
    if block < 1:
        raise ValueError("block must be >= 1")
    return attention_rows(q, k, v, causal, scale, rows=rows, heads=heads,
                          nthreads=nthreads, block=block)


def attention(q, k, v, causal: bool, scale: float, nthreads: int | None = None):
    """All rows of all heads: O [B, H, N, d] and LSE [B, H, N], fp64."""
    B, H, N, d = tuple(q.shape)
    O, L = attention_rows(q, k, v, causal, scale, nthreads=nthreads)
    return O.reshape(B, H, N, d), L.reshape(B, H, N)


def attention_qk(q, k, v, scale: float, heads=None, nthreads: int | None = None):
    """Non-causal attention of every query row of q [B, H, Nq, d] against the
    keys/values k, v [B, H, Nk, d] (decode: Nq = 1).  Returns
    (O [len(heads), Nq, d] fp64, LSE [len(heads), Nq] fp64)."""
    B, H, Nq, d = tuple(q.shape)
    if tuple(k.shape[:2]) != (B, H) or tuple(k.shape) != tuple(v.shape) or k.shape[3] != d:
        raise ValueError("q [B, H, Nq, d] and k, v [B, H, Nk, d] required")
    Nk = k.shape[2]
    BH = B * H
    heads = list(range(BH)) if heads is None else [int(h) for h in heads]
    nthreads = default_threads() if nthreads is None else int(nthreads)
    rows = np.arange(Nq, dtype=np.int64)
    zeros = np.zeros(Nq, dtype=np.int64)
    O = np.empty((len(heads), Nq, d), dtype=np.float64)
    L = np.empty((len(heads), Nq), dtype=np.float64)
    qf, kf, vf = q.reshape(BH, Nq, d), k.reshape(BH, Nk, d), v.reshape(BH, Nk, d)
    for n, bh in enumerate(heads):
        qh, kh, vh = _f64(qf[bh]), _f64(kf[bh]), _f64(vf[bh])
        o = np.empty((Nq, d), dtype=np.float64)
        lse = np.empty(Nq, dtype=np.float64)
        rc = _lib().oracle_attention_rows_qk(_dptr(qh), _dptr(kh), _dptr(vh), 1, Nq, Nk, d,
                                             float(scale), _iptr(zeros), _iptr(rows), Nq,
                                             _dptr(o), _dptr(lse), nthreads)
        if rc != 0:
            raise ValueError(f"oracle failed with status {rc}")
        O[n] = o
        L[n] = lse
    return O, L


def attention_backward(q, k, v, dout, causal: bool, scale: float, heads=None,
                       nthreads: int | None = None):
    """(dQ, dK, dV) fp64, each [len(heads), N, d], for the given heads of
    q, k, v, dout [B, H, N, d]."""
    shape = tuple(q.shape)
    if len(shape) != 4 or any(tuple(t.shape) != shape for t in (k, v, dout)):
        raise ValueError("q, k, v, dout must share one [B, H, N, d] shape")
    B, H, N, d = shape
    BH = B * H
    heads = list(range(BH)) if heads is None else [int(h) for h in heads]
    nthreads = default_threads() if nthreads is None else int(nthreads)
    out = [np.empty((len(heads), N, d), dtype=np.float64) for _ in range(3)]
    flat = [t.reshape(BH, N, d) for t in (q, k, v, dout)]
    for n, bh in enumerate(heads):
        qh, kh, vh, oh = (_f64(t[bh]) for t in flat)
        dq, dk, dv = (np.empty((N, d), dtype=np.float64) for _ in range(3))
        rc = _lib().oracle_attention_backward(_dptr(qh), _dptr(kh), _dptr(vh), _dptr(oh), N, d,
                                              int(bool(causal)), float(scale), _dptr(dq),
                                              _dptr(dk), _dptr(dv), nthreads)
        if rc != 0:
            raise ValueError(f"oracle failed with status {rc}")
        out[0][n], out[1][n], out[2][n] = dq, dk, dv
    return tuple(out)


def prob_row(q, k, v, causal: bool, scale: float, head: int, row: int) -> np.ndarray:
    """The probability row P_i (length N; zeros at masked keys) of one head."""
    B, H, N, d = tuple(q.shape)
    qh = _f64(q.reshape(B * H, N, d)[head])
    kh = _f64(k.reshape(B * H, N, d)[head])
    vh = _f64(v.reshape(B * H, N, d)[head])
    p = np.empty(N, dtype=np.float64)
    rc = _lib().oracle_attention_prob_row(_dptr(qh), _dptr(kh), _dptr(vh), 1, N, d,
                                          int(bool(causal)), float(scale), 0, int(row),
                                          _dptr(p))
    if rc != 0:
        raise ValueError(f"oracle failed with status {rc}")
    return p
