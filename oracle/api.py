"""ctypes wrapper around the plain-C oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU baseline).
Every function takes and returns numpy arrays; bf16 tensors travel as
uint16 bit patterns.  The library is compiled with gcc -O2 (no fast-math)
on first use if it is missing or older than its source.
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force=False):
    """Compile liboracle.so next to its source (gcc, -O2, strict IEEE)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB)
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def bf16_round_bits(x):
    """fp32 -> bf16 bits (RNE), element by element through the C routine."""
    lib = _load()
    lib.orc_bf16_round_bits.restype = ctypes.c_uint16
    lib.orc_bf16_round_bits.argtypes = [ctypes.c_float]
    x = np.asarray(x, np.float32).ravel()
    return np.array([lib.orc_bf16_round_bits(float(v)) for v in x], np.uint16)


def splitk(A, chunk=32):
    """Two-stage split-K reduction; returns (B [rows, nchunk], C [rows]) in fp64."""
    lib = _load()
    A = _c(A, np.float32)
    rows, cols = A.shape
    nchunk = (cols + chunk - 1) // chunk
    B = np.zeros((rows, nchunk), np.float64)
    C = np.zeros((rows,), np.float64)
    lib.orc_splitk(_p(A), ctypes.c_int(rows), ctypes.c_int(cols), ctypes.c_int(chunk), _p(B), _p(C))
    return B, C


def rmsnorm(X, gamma, eps=1e-5):
    lib = _load()
    X = _c(X, np.uint16)
    gamma = _c(gamma, np.uint16)
    rows, hidden = X.shape
    xn = np.zeros_like(X)
    lib.orc_rmsnorm(_p(X), _p(gamma), ctypes.c_int(rows), ctypes.c_int(hidden), ctypes.c_double(eps), _p(xn))
    return xn


def mlp(X, gamma, Wgu, Wd, eps=1e-5, want_intermediates=False):
    """Decode MLP y = down(silu(gate(xn)) * up(xn)), xn = rmsnorm(x); bf16 bits out."""
    lib = _load()
    X = _c(X, np.uint16)
    B, hidden = X.shape
    inter = Wgu.shape[0] // 2
    assert Wgu.shape == (2 * inter, hidden) and Wd.shape == (hidden, inter)
    Y = np.zeros((B, hidden), np.uint16)
    xn = np.zeros((B, hidden), np.uint16)
    h = np.zeros((B, inter), np.uint16)
    lib.orc_mlp(_p(X), _p(_c(gamma, np.uint16)), _p(_c(Wgu, np.uint16)), _p(_c(Wd, np.uint16)),
                ctypes.c_int(B), ctypes.c_int(hidden), ctypes.c_int(inter), ctypes.c_double(eps),
                _p(Y), _p(xn), _p(h))
    if want_intermediates:
        return Y, xn, h
    return Y


def mlp_rows(X, gamma, Wgu, Wd, rows, eps=1e-5):
    """Decode MLP for the listed rows of X only."""
    lib = _load()
    X = _c(X, np.uint16)
    hidden = X.shape[1]
    inter = Wgu.shape[0] // 2
    rows = _c(rows, np.int32)
    Y = np.zeros((len(rows), hidden), np.uint16)
    lib.orc_mlp_rows(_p(X), _p(_c(gamma, np.uint16)), _p(_c(Wgu, np.uint16)), _p(_c(Wd, np.uint16)),
                     _p(rows), ctypes.c_int(len(rows)), ctypes.c_int(hidden), ctypes.c_int(inter),
                     ctypes.c_double(eps), _p(Y))
    return Y


def router_logits(X, Wr, bias):
    lib = _load()
    X = _c(X, np.uint16)
    Wr = _c(Wr, np.uint16)
    T, hidden = X.shape
    E = Wr.shape[0]
    out = np.zeros((T, E), np.float32)
    lib.orc_router_logits(_p(X), _p(Wr), _p(_c(bias, np.float32)), ctypes.c_int(T),
                          ctypes.c_int(hidden), ctypes.c_int(E), _p(out))
    return out


def topk_softmax(logits, k):
    lib = _load()
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    lib.orc_topk_softmax(_p(logits), ctypes.c_int(T), ctypes.c_int(E), ctypes.c_int(k), _p(idx), _p(w))
    return idx, w


def group(topk, E, bm):
    """Returns dict(counts, indptr, perm, task_indptr, pos)."""
    lib = _load()
    topk = _c(topk, np.int32)
    T, k = topk.shape
    counts = np.zeros(E, np.int32)
    indptr = np.zeros(E + 1, np.int32)
    perm = np.zeros(T * k, np.int32)
    task_indptr = np.zeros(E + 1, np.int32)
    pos = np.zeros(T * k, np.int32)
    lib.orc_group(_p(topk), ctypes.c_int(T), ctypes.c_int(k), ctypes.c_int(E), ctypes.c_int(bm),
                  _p(counts), _p(indptr), _p(perm), _p(task_indptr), _p(pos))
    return dict(counts=counts, indptr=indptr, perm=perm, task_indptr=task_indptr, pos=pos)


def moe_grouped(X, W1, W2, topk, w, indptr, perm, want_h=False):
    lib = _load()
    X = _c(X, np.uint16)
    T, hidden = X.shape
    E, two_inter, _ = W1.shape
    inter = two_inter // 2
    k = topk.shape[1]
    Y = np.zeros((T, hidden), np.uint16)
    h = np.zeros((T * k, inter), np.uint16) if want_h else None
    lib.orc_moe_grouped(_p(X), _p(_c(W1, np.uint16)), _p(_c(W2, np.uint16)), _p(_c(topk, np.int32)),
                        _p(_c(w, np.float32)), _p(_c(indptr, np.int32)), _p(_c(perm, np.int32)),
                        ctypes.c_int(T), ctypes.c_int(hidden), ctypes.c_int(inter), ctypes.c_int(E),
                        ctypes.c_int(k), _p(Y), _p(h))
    return (Y, h) if want_h else Y


def moe_per_token(X, Wr, bias, W1, W2, tokens, k):
    """Per-token MoE evaluation of the listed tokens; returns (Y_rows, topk_rows, w_rows)."""
    lib = _load()
    X = _c(X, np.uint16)
    hidden = X.shape[1]
    E, two_inter, _ = W1.shape
    inter = two_inter // 2
    tokens = _c(tokens, np.int32)
    n = len(tokens)
    Y = np.zeros((n, hidden), np.uint16)
    tk = np.zeros((n, k), np.int32)
    w = np.zeros((n, k), np.float32)
    lib.orc_moe_per_token(_p(X), _p(_c(Wr, np.uint16)), _p(_c(bias, np.float32)), _p(_c(W1, np.uint16)),
                          _p(_c(W2, np.uint16)), _p(tokens), ctypes.c_int(n), ctypes.c_int(hidden),
                          ctypes.c_int(inter), ctypes.c_int(E), ctypes.c_int(k), _p(Y), _p(tk), _p(w))
    return Y, tk, w


def moe_rows_given_routing(X, W1, W2, tokens, topk_rows, w_rows):
    lib = _load()
    X = _c(X, np.uint16)
    hidden = X.shape[1]
    E, two_inter, _ = W1.shape
    inter = two_inter // 2
    tokens = _c(tokens, np.int32)
    n = len(tokens)
    k = topk_rows.shape[1]
    Y = np.zeros((n, hidden), np.uint16)
    lib.orc_moe_rows_given_routing(_p(X), _p(_c(W1, np.uint16)), _p(_c(W2, np.uint16)), _p(tokens),
                                   _p(_c(topk_rows, np.int32)), _p(_c(w_rows, np.float32)),
                                   ctypes.c_int(n), ctypes.c_int(hidden), ctypes.c_int(inter),
                                   ctypes.c_int(k), _p(Y))
    return Y


def moe(X, Wr, bias, W1, W2, k, bm=128):
    """Whole MoE layer through the grouped path; returns a dict of every
    intermediate the method defines (logits, topk, w, grouping, h, y)."""
    logits = router_logits(X, Wr, bias)
    tk, w = topk_softmax(logits, k)
    g = group(tk, W1.shape[0], bm)
    Y, h = moe_grouped(X, W1, W2, tk, w, g["indptr"], g["perm"], want_h=True)
    out = dict(logits=logits, topk=tk, w=w, y=Y, h=h)
    out.update(g)
    return out


__all__ = ["build", "bf16_round_bits", "splitk", "rmsnorm", "mlp", "mlp_rows", "router_logits",
           "topk_softmax", "group", "moe_grouped", "moe_per_token", "moe_rows_given_routing", "moe"]
