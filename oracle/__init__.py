"""CPU oracle for the deterministic-reduction kernels (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never does; the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, fp64 exact references and the
canonical fp32 reduction order).  This module compiles it with gcc on first
use (``-O2 -ffp-contract=off``, no fast-math) and wraps it for numpy arrays.
bf16 arrays are passed as ``uint16`` bit patterns.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, brute force, library routines or the worked example of
"The biggest Mystery of LLMs have just been solved" (Floating Point
Arithmetic Example, corrected), never against itself.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-Wall", "-Wextra"]

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (if stale or missing)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    L = ctypes.c_long
    I = ctypes.c_int
    F = ctypes.c_float
    D = ctypes.c_double
    sig = {
        "or_bf16_to_f32": (F, [ctypes.c_uint16]),
        "or_f32_to_bf16": (ctypes.c_uint16, [F]),
        "or_f32_to_bf16_array": (None, [P, L, P]),
        "or_tree_f32": (F, [P, L, L]),
        "or_tree_combine": (None, [P, L, L, P, I]),
        "or_canon_sum": (F, [P, L, I, I]),
        "or_exp": (F, [F]),
        "or_log": (F, [F]),
        "or_shrink_exact": (None, [P, P, P, L, L, L, L, P, P, I]),
        "or_expand_exact": (None, [P, P, P, L, L, L, L, P, P, P, I]),
        "or_gemm_exact": (None, [P, P, L, L, L, P, L, P, P, I]),
        "or_addmm_exact": (None, [P, P, P, L, L, L, P, L, P, P, I]),
        "or_segment": (None, [P, L, I, P, P]),
        "or_attn_decode_exact": (None, [P, P, P, P, L, L, L, L, L, D, P, I]),
        "or_attn_decode_canon": (None, [P, P, P, P, L, L, L, L, L, F, P, I]),
        "or_rmsnorm_exact": (None, [P, P, L, L, D, P, I]),
        "or_rmsnorm_canon": (None, [P, P, L, L, F, P, I]),
        "or_rmsnorm_inv_canon": (F, [P, L, F]),
        "or_log_softmax_exact": (None, [P, L, L, P, I]),
        "or_log_softmax_canon": (None, [P, L, L, P, I]),
        "or_mean_exact": (None, [P, L, L, P, I]),
        "or_mean_canon": (None, [P, L, L, P, I]),
        "or_max_threads": (I, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def max_threads() -> int:
    return int(_load().or_max_threads())


def _nt(nthreads):
    return int(nthreads) if nthreads else max_threads()


def _c(a, dtype):
    """C-contiguous array of the given dtype (copy only if needed)."""
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- scalars

def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp32 values."""
    b = _c(bits, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(values) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (oracle's own)."""
    v = _c(values, np.float32)
    out = np.empty(v.shape, np.uint16)
    _load().or_f32_to_bf16_array(_p(v), v.size, _p(out))
    return out


def exp_spec(x: float) -> np.float32:
    return np.float32(_load().or_exp(float(np.float32(x))))


def log_spec(x: float) -> np.float32:
    return np.float32(_load().or_log(float(np.float32(x))))


# ------------------------------------------------------------ reductions

def tree_sum(v) -> np.float32:
    """Canonical halving tree over a 1-D fp32 vector."""
    a = _c(v, np.float32)
    return np.float32(_load().or_tree_f32(_p(a), a.size, 1))


def tree_combine(parts, nthreads=None) -> np.ndarray:
    """parts [s, ...] fp32 -> canonical tree over axis 0."""
    a = _c(parts, np.float32)
    s = a.shape[0]
    count = a.size // s if s else 0
    out = np.empty(a.shape[1:], dtype=np.float32)
    _load().or_tree_combine(_p(a), s, count, _p(out), _nt(nthreads))
    return out


def canon_sum(v, T: int, V: int) -> np.float32:
    a = _c(v, np.float32)
    assert a.size % V == 0
    return np.float32(_load().or_canon_sum(_p(a), a.size, T, V))


# ------------------------------------------------------------------ LoRA

def shrink_exact(x, at, ids=None, nthreads=None):
    """x bf16 [M,K]; at bf16 [r,K] or [n_ad,r,K]; ids int32 [M] or None.
    Returns (y fp64 [M,r], bound fp64 [M,r])."""
    x = _c(x, np.uint16)
    at = _c(at, np.uint16)
    if at.ndim == 2:
        at = at[None]
    n_ad, r, K = at.shape
    M = x.shape[0]
    assert x.shape == (M, K)
    idp = None
    if ids is not None:
        ids = _c(ids, np.int32)
        assert ids.shape == (M,)
        idp = _p(ids)
    y = np.empty((M, r), np.float64)
    b = np.empty((M, r), np.float64)
    _load().or_shrink_exact(_p(x), _p(at), idp, n_ad, M, K, r, _p(y), _p(b), _nt(nthreads))
    return y, b


def expand_exact(y, bt, ids=None, prev=None, nthreads=None):
    """y fp32 [M,r]; bt bf16 [N,r] or [n_ad,N,r]; prev fp32 [M,N] or None.
    Returns (out fp64 [M,N], bound fp64 [M,N])."""
    y = _c(y, np.float32)
    bt = _c(bt, np.uint16)
    if bt.ndim == 2:
        bt = bt[None]
    n_ad, N, r = bt.shape
    M = y.shape[0]
    assert y.shape == (M, r)
    idp = None
    if ids is not None:
        ids = _c(ids, np.int32)
        idp = _p(ids)
    pp = None
    if prev is not None:
        prev = _c(prev, np.float32)
        assert prev.shape == (M, N)
        pp = _p(prev)
    out = np.empty((M, N), np.float64)
    b = np.empty((M, N), np.float64)
    _load().or_expand_exact(_p(y), _p(bt), idp, n_ad, M, r, N, pp, _p(out), _p(b), _nt(nthreads))
    return out, b


def segment(ids, n_adapters: int):
    """Stable counting sort by adapter id -> (perm int32 [n_valid], offsets int32 [n_ad+1])."""
    ids = _c(ids, np.int32)
    M = ids.size
    perm = np.full(M, -1, np.int32)
    offs = np.zeros(n_adapters + 1, np.int32)
    _load().or_segment(_p(ids), M, n_adapters, _p(perm), _p(offs))
    return perm[: offs[-1]], offs


# ------------------------------------------------------------------ GEMM

def gemm_exact(a, w, rows=None, nthreads=None):
    """a bf16 [M,K]; w bf16 [N,K]; C = a @ w.T in fp64.  rows: optional
    index list (only those rows are computed).  Returns (C, bound)."""
    a = _c(a, np.uint16)
    w = _c(w, np.uint16)
    M, K = a.shape
    N = w.shape[0]
    assert w.shape == (N, K)
    rp, nr = None, M
    if rows is not None:
        rows = _c(rows, np.int64)
        rp, nr = _p(rows), rows.size
    C = np.empty((nr, N), np.float64)
    b = np.empty((nr, N), np.float64)
    _load().or_gemm_exact(_p(a), _p(w), M, N, K, rp, nr if rows is not None else 0,
                          _p(C), _p(b), _nt(nthreads))
    return C, b


def addmm_exact(bias, a, w, rows=None, nthreads=None):
    """bias bf16 [N]; a bf16 [M,K]; w bf16 [N,K]; C = bias + a @ w.T in
    fp64 (torch.addmm).  rows: optional index list.  Returns (C, bound)
    with bound = |bias| + sum |a*w|."""
    bias = _c(bias, np.uint16)
    a = _c(a, np.uint16)
    w = _c(w, np.uint16)
    M, K = a.shape
    N = w.shape[0]
    assert w.shape == (N, K) and bias.shape == (N,)
    rp, nr = None, M
    if rows is not None:
        rows = _c(rows, np.int64)
        rp, nr = _p(rows), rows.size
    C = np.empty((nr, N), np.float64)
    b = np.empty((nr, N), np.float64)
    _load().or_addmm_exact(_p(bias), _p(a), _p(w), M, N, K, rp, nr if rows is not None else 0,
                           _p(C), _p(b), _nt(nthreads))
    return C, b


def _attn_args(q, k, v, lens):
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    lens = _c(lens, np.int32)
    B, Hq, D = q.shape
    B2, Hkv, Lmax, D2 = k.shape
    assert B2 == B and D2 == D and v.shape == k.shape and lens.shape == (B,) and Hq % Hkv == 0
    return q, k, v, lens, B, Hq, Hkv, D, Lmax


def attn_decode_exact(q, k, v, lens, scale, nthreads=None):
    """Decode attention in fp64: q bf16 [B,Hq,D]; k, v bf16 [B,Hkv,Lmax,D];
    lens int32 [B].  Returns out float64 [B,Hq,D]."""
    q, k, v, lens, B, Hq, Hkv, D, Lmax = _attn_args(q, k, v, lens)
    out = np.empty((B, Hq, D), np.float64)
    _load().or_attn_decode_exact(_p(q), _p(k), _p(v), _p(lens), B, Hq, Hkv, D, Lmax, float(scale), _p(out),
                                 _nt(nthreads))
    return out


def attn_decode_canon(q, k, v, lens, scale, nthreads=None):
    """Decode attention in the canonical fp32 order (256-key chunk frames,
    perfect trees, the written exp).  Returns out float32 [B,Hq,D]."""
    q, k, v, lens, B, Hq, Hkv, D, Lmax = _attn_args(q, k, v, lens)
    out = np.empty((B, Hq, D), np.float32)
    _load().or_attn_decode_canon(_p(q), _p(k), _p(v), _p(lens), B, Hq, Hkv, D, Lmax, float(np.float32(scale)),
                                 _p(out), _nt(nthreads))
    return out


# ------------------------------------------------------------- row ops

def rmsnorm_exact(x, w, eps=1e-6, nthreads=None):
    x = _c(x, np.uint16)
    w = _c(w, np.uint16)
    R, n = x.shape
    y = np.empty((R, n), np.float64)
    _load().or_rmsnorm_exact(_p(x), _p(w), R, n, float(eps), _p(y), _nt(nthreads))
    return y


def rmsnorm_canon(x, w, eps=1e-6, nthreads=None):
    x = _c(x, np.uint16)
    w = _c(w, np.uint16)
    R, n = x.shape
    assert n % 8 == 0
    y = np.empty((R, n), np.uint16)
    _load().or_rmsnorm_canon(_p(x), _p(w), R, n, float(np.float32(eps)), _p(y), _nt(nthreads))
    return y


def rmsnorm_inv_canon(xrow, eps=1e-6) -> np.float32:
    """The canonical fp32 scale 1/sqrt(mean(x^2) + eps) of one bf16 row."""
    x = _c(xrow, np.uint16)
    assert x.size % 8 == 0
    return np.float32(_load().or_rmsnorm_inv_canon(_p(x), x.size, float(np.float32(eps))))


def log_softmax_exact(x, nthreads=None):
    x = _c(x, np.float32)
    R, n = x.shape
    out = np.empty((R, n), np.float64)
    _load().or_log_softmax_exact(_p(x), R, n, _p(out), _nt(nthreads))
    return out


def log_softmax_canon(x, nthreads=None):
    x = _c(x, np.float32)
    R, n = x.shape
    assert n % 4 == 0
    out = np.empty((R, n), np.float32)
    _load().or_log_softmax_canon(_p(x), R, n, _p(out), _nt(nthreads))
    return out


def mean_exact(x, nthreads=None):
    x = _c(x, np.float32)
    R, n = x.shape
    out = np.empty(R, np.float64)
    _load().or_mean_exact(_p(x), R, n, _p(out), _nt(nthreads))
    return out


def mean_canon(x, nthreads=None):
    x = _c(x, np.float32)
    R, n = x.shape
    assert n % 4 == 0
    out = np.empty(R, np.float32)
    _load().or_mean_canon(_p(x), R, n, _p(out), _nt(nthreads))
    return out
