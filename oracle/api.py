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
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fopenmp",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB)
        _lib.orc_moe_grouped.restype = ctypes.c_int
        for f in ("orc_get_threads", "orc_max_threads"):
            getattr(_lib, f).restype = ctypes.c_int
        _lib.orc_set_threads(ctypes.c_int(int(os.environ.get("ORACLE_THREADS", "1"))))
    return _lib


def set_threads(n):
    """OpenMP threads for the oracle's parallel loops (tokens, rows, pairs);
    results are bit-identical for every thread count."""
    _load().orc_set_threads(ctypes.c_int(int(n)))


def get_threads():
    return _load().orc_get_threads()


def max_threads():
    """Processors available to this process."""
    return _load().orc_max_threads()


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
    indptr = _c(indptr, np.int32)
    perm = _c(perm, np.int32)
    if indptr.shape != (E + 1,) or perm.shape != (T * k,):
        raise ValueError("malformed grouping: indptr must have E+1 entries and perm T*k")
    rc = lib.orc_moe_grouped(_p(X), _p(_c(W1, np.uint16)), _p(_c(W2, np.uint16)), _p(_c(topk, np.int32)),
                             _p(_c(w, np.float32)), _p(indptr), _p(perm),
                             ctypes.c_int(T), ctypes.c_int(hidden), ctypes.c_int(inter), ctypes.c_int(E),
                             ctypes.c_int(k), _p(Y), _p(h))
    if rc != 0:
        raise ValueError("malformed grouping: indptr/perm do not group the pairs of topk by expert")
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


def rope(x, pos, base=500000.0):
    """Rotary embedding of one bf16 head vector at position pos (bf16 out)."""
    lib = _load()
    x = _c(x, np.uint16)
    out = np.zeros_like(x)
    lib.orc_rope_bf16(_p(x), ctypes.c_int(x.shape[0]), ctypes.c_int(int(pos)), ctypes.c_double(base), _p(out))
    return out


def decode_layer(X, pos, w, Kc, Vc, n_q, n_kv, eps=1e-5, rope_base=500000.0):
    """One decode step of the layer for B requests (see orc_decode_layer).
    w: dict(g1, Wqkv, gq, gk, Wo, g2, Wgu, Wd) of bf16 bits.  Kc, Vc:
    [B, n_kv, max_ctx, hd] caches; copies are updated and returned.
    Returns dict(y, q, k, a, h1, Kc, Vc)."""
    lib = _load()
    X = _c(X, np.uint16)
    pos = _c(pos, np.int32)
    B, hidden = X.shape
    Kc = np.array(Kc, dtype=np.uint16, copy=True)
    Vc = np.array(Vc, dtype=np.uint16, copy=True)
    _, nkv2, max_ctx, hd = Kc.shape
    assert nkv2 == n_kv and Vc.shape == Kc.shape and Kc.shape[0] == B
    inter = w["Wgu"].shape[0] // 2
    Y = np.zeros((B, hidden), np.uint16)
    q = np.zeros((B, n_q * hd), np.uint16)
    k = np.zeros((B, n_kv * hd), np.uint16)
    a = np.zeros((B, n_q * hd), np.uint16)
    h1 = np.zeros((B, hidden), np.uint16)
    rc = lib.orc_decode_layer(_p(X), _p(pos), ctypes.c_int(B), ctypes.c_int(hidden), ctypes.c_int(n_q),
                              ctypes.c_int(n_kv), ctypes.c_int(hd), ctypes.c_int(inter),
                              _p(_c(w["g1"], np.uint16)), _p(_c(w["Wqkv"], np.uint16)), _p(_c(w["gq"], np.uint16)),
                              _p(_c(w["gk"], np.uint16)), _p(_c(w["Wo"], np.uint16)), _p(_c(w["g2"], np.uint16)),
                              _p(_c(w["Wgu"], np.uint16)), _p(_c(w["Wd"], np.uint16)), _p(Kc), _p(Vc),
                              ctypes.c_int(max_ctx), ctypes.c_double(eps), ctypes.c_double(rope_base),
                              _p(Y), _p(q), _p(k), _p(a), _p(h1))
    if rc != 0:
        raise ValueError("decode layer: a position lies outside the cache")
    return dict(y=Y, q=q, k=k, a=a, h1=h1, Kc=Kc, Vc=Vc)


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


__all__ = ["build", "set_threads", "get_threads", "max_threads", "bf16_round_bits", "splitk", "rmsnorm", "mlp", "mlp_rows", "router_logits",
           "topk_softmax", "group", "moe_grouped", "moe_per_token", "moe_rows_given_routing", "moe", "rope", "decode_layer"]
