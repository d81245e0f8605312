"""Seeded synthetic inputs for the three workloads (split-K, decode MLP, MoE).

This module holds the input recipe only: random draws, the conversion of
the draws to the stored dtype (bf16 bit patterns, round-to-nearest-even)
and the expert-bias recipe.  It holds none of the method's arithmetic.  It
is shared by the tests, the benchmark and the smoke check, which hand the
same arrays to the CPU oracle and to the device library.

Recipe (numpy PCG64 ``default_rng(seed)``):
  split-K  A fp32 [rows, 128] ~ U[-1, 1]                          seed 1
  MLP      X [B, hidden] ~ N(0,1); gamma ~ N(1, 0.1);
           Wgu [2*inter, hidden], Wd [hidden, inter] ~ N(0, 0.02)  seeds 10+B, 11, 12, 13
  MoE      X [T, hidden] ~ N(0,1); Wr [E, hidden] ~ N(0, 0.02);
           W1 [E, 2*inter, hidden], W2 [E, hidden, inter] ~ N(0, 0.02);
           bias[e] = -s * ln(1 + pi(e)), pi a seeded permutation of
           0..E-1 (a Zipf(s) popularity prior on the experts; s = 0 gives
           zero bias)                                              seeds 100+log2(T) (1000+T when T is
           not a power of two), 20, 21, 22, 23
  MoE->MLP the MoE inputs above, then a dense MLP on the layer's output:
           gamma ~ N(1, 0.1), Wgu [2*mlp_inter, hidden], Wd [hidden,
           mlp_inter] ~ N(0, 0.02)                                  seeds 50, 51, 52
  decode   X [B, hidden] ~ N(0,1); context lengths ~ U{512..4096} (the
           new token's position); K and V caches [B, n_kv, max_ctx, hd]
           ~ N(0,1) at the cached positions, zero beyond;
           g1, gq, gk, g2 ~ N(1, 0.1); Wqkv [(n_q+2n_kv)*hd, hidden],
           Wo [hidden, n_q*hd] ~ N(0, 0.02); Wgu, Wd as for the MLP   seeds 40+B, 41, 42, 43, 44..49, 12, 13
"""
import math

import numpy as np


def f32_to_bf16_bits(x):
    """fp32 array -> bf16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    r = (u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b):
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(rng, shape, mean, std, chunk=1 << 26):
    """N(mean, std) draws in fp32, stored as bf16 bits; drawn in chunks so a
    1 GB weight never holds a float64 copy."""
    n = int(np.prod(shape))
    out = np.empty(n, np.uint16)
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        v = rng.standard_normal(m, dtype=np.float32)
        v *= np.float32(std)
        v += np.float32(mean)
        out[i:i + m] = f32_to_bf16_bits(v)
    return out.reshape(shape)


def splitk_inputs(rows, cols=128, seed=1):
    rng = np.random.default_rng(seed)
    return rng.uniform(-1.0, 1.0, size=(rows, cols)).astype(np.float32)


def mlp_inputs(B, hidden=4096, inter=14336, weights=True):
    """dict(X, gamma, Wgu, Wd); bf16 tensors as uint16 bit patterns."""
    d = dict(
        X=_normal_bf16(np.random.default_rng(10 + B), (B, hidden), 0.0, 1.0),
        gamma=_normal_bf16(np.random.default_rng(11), (hidden,), 1.0, 0.1),
    )
    if weights:
        d["Wgu"] = _normal_bf16(np.random.default_rng(12), (2 * inter, hidden), 0.0, 0.02)
        d["Wd"] = _normal_bf16(np.random.default_rng(13), (hidden, inter), 0.0, 0.02)
    return d


def expert_bias(E, s, seed=23):
    """Zipf(s) popularity prior: the expert of rank r (1 = hottest) gets
    logit bias -s*ln(r); ranks are a seeded permutation of the experts."""
    rank = np.random.default_rng(seed).permutation(E)
    return (-float(s) * np.log1p(rank.astype(np.float64))).astype(np.float32)


def moe_inputs(T, hidden=2048, inter=768, E=128, zipf_s=1.2, weights=True):
    """dict(X, Wr, bias, W1, W2); bf16 tensors as uint16 bit patterns."""
    if T > 0 and (T & (T - 1)) == 0:
        xseed = 100 + int(math.log2(T))
    else:
        xseed = 1000 + T
    d = dict(
        X=_normal_bf16(np.random.default_rng(xseed), (T, hidden), 0.0, 1.0),
        Wr=_normal_bf16(np.random.default_rng(20), (E, hidden), 0.0, 0.02),
        bias=expert_bias(E, zipf_s),
    )
    if weights:
        d["W1"] = _normal_bf16(np.random.default_rng(21), (E, 2 * inter, hidden), 0.0, 0.02)
        d["W2"] = _normal_bf16(np.random.default_rng(22), (E, hidden, inter), 0.0, 0.02)
    return d


def decode_inputs(B, hidden=4096, n_q=32, n_kv=8, hd=128, inter=14336, ctx_lo=512, ctx_hi=4096, max_ctx=None,
                  weights=True):
    """dict(X, pos, Kc, Vc[, g1, Wqkv, gq, gk, Wo, g2, Wgu, Wd]) for one decode
    step of B requests; pos[b] = tokens already cached for request b.  Both
    caches are [B, n_kv, max_ctx, hd] here; the device takes V transposed
    (v_cache_device)."""
    if max_ctx is None:
        max_ctx = (ctx_hi + 1 + 7) // 8 * 8  # the device reads cache rows as 16-byte multiples
    pos = np.random.default_rng(41).integers(ctx_lo, ctx_hi + 1, size=64 if B <= 64 else B)[:B].astype(np.int32)
    Kc = np.zeros((B, n_kv, max_ctx, hd), np.uint16)
    Vc = np.zeros((B, n_kv, max_ctx, hd), np.uint16)
    rk, rv = np.random.default_rng(42), np.random.default_rng(43)
    for b in range(B):
        n = int(pos[b])
        Kc[b, :, :n] = _normal_bf16(rk, (n_kv, n, hd), 0.0, 1.0)
        Vc[b, :, :n] = _normal_bf16(rv, (n_kv, n, hd), 0.0, 1.0)
    d = dict(X=_normal_bf16(np.random.default_rng(40 + B), (B, hidden), 0.0, 1.0), pos=pos, Kc=Kc, Vc=Vc)
    if weights:
        d["g1"] = _normal_bf16(np.random.default_rng(44), (hidden,), 1.0, 0.1)
        d["Wqkv"] = _normal_bf16(np.random.default_rng(45), ((n_q + 2 * n_kv) * hd, hidden), 0.0, 0.02)
        d["gq"] = _normal_bf16(np.random.default_rng(46), (hd,), 1.0, 0.1)
        d["gk"] = _normal_bf16(np.random.default_rng(47), (hd,), 1.0, 0.1)
        d["Wo"] = _normal_bf16(np.random.default_rng(48), (hidden, n_q * hd), 0.0, 0.02)
        d["g2"] = _normal_bf16(np.random.default_rng(49), (hidden,), 1.0, 0.1)
        d["Wgu"] = _normal_bf16(np.random.default_rng(12), (2 * inter, hidden), 0.0, 0.02)
        d["Wd"] = _normal_bf16(np.random.default_rng(13), (hidden, inter), 0.0, 0.02)
    return d


def dense_mlp_weights(hidden=2048, inter=6144):
    """dict(gamma, Wgu, Wd) of the dense MLP after the MoE layer."""
    return dict(gamma=_normal_bf16(np.random.default_rng(50), (hidden,), 1.0, 0.1),
                Wgu=_normal_bf16(np.random.default_rng(51), (2 * inter, hidden), 0.0, 0.02),
                Wd=_normal_bf16(np.random.default_rng(52), (hidden, inter), 0.0, 0.02))


def v_cache_device(Vc):
    """The device's V cache layout, [B, n_kv, hd, max_ctx] (keys contiguous),
    from [B, n_kv, max_ctx, hd]; the same function maps it back."""
    return np.ascontiguousarray(np.swapaxes(Vc, 2, 3))
