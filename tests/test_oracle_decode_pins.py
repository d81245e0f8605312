"""Pins of the decode-layer oracle ("Event Tensor：用“事件张量”编译动态
Megakernel", §端到端低 batch serving: the decoding pipeline of Attention,
RoPE, KV-cache, Norm and MLP; the Q branch runs Norm + RoPE, the K branch
Norm + RoPE + cache append) against library routines and invariants:
torch's scaled-dot-product attention and RMSNorm, rotary embedding as a
complex rotation, single-key attention, the cache write, a zero output
projection."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads as W

DIMS = dict(hidden=64, n_q=4, n_kv=2, hd=16, inter=32)


def f32(b):
    return W.bf16_bits_to_f32(b)


def bf16(t):
    """torch fp64 -> bf16 bits by the same two-step rounding (fp32, then RNE)."""
    return W.f32_to_bf16_bits(t.to(torch.float32).numpy())


def small(B=3, ctx_lo=2, ctx_hi=9, max_ctx=12):
    d = W.decode_inputs(B, ctx_lo=ctx_lo, ctx_hi=ctx_hi, max_ctx=max_ctx, **DIMS)
    return d, {k: d[k] for k in ("g1", "Wqkv", "gq", "gk", "Wo", "g2", "Wgu", "Wd")}


def test_rope_is_a_complex_rotation():
    x = W.f32_to_bf16_bits(np.random.default_rng(0).standard_normal(128).astype(np.float32))
    for pos in (0, 1, 17, 4000):
        got = f32(oracle.rope(x, pos))
        v = torch.from_numpy(f32(x).astype(np.float64))
        z = torch.complex(v[:64], v[64:])
        theta = 500000.0 ** (-torch.arange(64, dtype=torch.float64) * 2 / 128)
        r = z * torch.polar(torch.ones(64, dtype=torch.float64), pos * theta)
        ref = bf16(torch.cat([r.real, r.imag]))
        # the same rotation up to the last rounding: at most one bf16 ulp of the vector's scale
        assert np.max(np.abs(got - f32(ref))) <= 2.0 ** -7 * np.abs(f32(x)).max()
    assert np.array_equal(oracle.rope(x, 0), x)   # position 0: identity


def test_rope_scores_depend_on_relative_position():
    rng = np.random.default_rng(1)
    q = W.f32_to_bf16_bits(rng.standard_normal(128).astype(np.float32))
    k = W.f32_to_bf16_bits(rng.standard_normal(128).astype(np.float32))
    s1 = float(np.dot(f32(oracle.rope(q, 40)).astype(np.float64), f32(oracle.rope(k, 10))))
    s2 = float(np.dot(f32(oracle.rope(q, 1040)).astype(np.float64), f32(oracle.rope(k, 1010))))
    assert abs(s1 - s2) <= 0.05 * (abs(s1) + 1.0)   # equal up to the bf16 rounding of the rotated vectors


def test_single_key_attention_returns_the_value():
    """At position 0 the only key is the new token's: softmax of one score
    is 1 and the attention output is its value vector."""
    d, w = small(B=2, ctx_lo=0, ctx_hi=0)
    out = oracle.decode_layer(d["X"], np.zeros(2, np.int32), w, d["Kc"], d["Vc"], 4, 2)
    hd, nq, nkv = 16, 4, 2
    for b in range(2):
        for h in range(nq):
            g = h // (nq // nkv)
            v_new = out["Vc"][b, g, 0]
            assert np.array_equal(out["a"][b, h * hd:(h + 1) * hd], v_new)


def test_cache_append_writes_only_the_new_position():
    d, w = small()
    out = oracle.decode_layer(d["X"], d["pos"], w, d["Kc"], d["Vc"], 4, 2)
    for b, p in enumerate(d["pos"]):
        for g in range(2):
            assert np.array_equal(out["Kc"][b, g, p], out["k"][b, g * 16:(g + 1) * 16])
        keep = np.ones(12, bool)
        keep[p] = False
        assert np.array_equal(out["Kc"][b][:, keep], d["Kc"][b][:, keep])
        assert np.array_equal(out["Vc"][b][:, keep], d["Vc"][b][:, keep])


def test_zero_output_projection_keeps_the_residual():
    d, w = small()
    w = dict(w, Wo=np.zeros_like(w["Wo"]))
    out = oracle.decode_layer(d["X"], d["pos"], w, d["Kc"], d["Vc"], 4, 2)
    assert np.array_equal(out["h1"], d["X"])


def test_layer_matches_torch_library_routines():
    """The whole step composed from torch fp64 library routines (rms_norm,
    scaled_dot_product_attention with grouped KV heads, silu, matmul) and a
    complex-number rotary embedding, rounded to bf16 where the layer hands
    bf16 tensors on."""
    d, w = small(B=3)
    out = oracle.decode_layer(d["X"], d["pos"], w, d["Kc"], d["Vc"], 4, 2)
    T = lambda a: torch.from_numpy(f32(a).astype(np.float64))  # noqa: E731
    B, H, nq, nkv, hd, I = 3, 64, 4, 2, 16, 32
    x = T(d["X"])
    xn = T(bf16(F.rms_norm(x, (H,), T(w["g1"]), eps=1e-5)))
    qkv = T(bf16(xn @ T(w["Wqkv"]).T))
    theta = 500000.0 ** (-torch.arange(hd // 2, dtype=torch.float64) * 2 / hd)

    def rot(v, p):
        z = torch.complex(v[..., :hd // 2], v[..., hd // 2:]) * torch.polar(torch.ones_like(theta), p * theta)
        return torch.cat([z.real, z.imag], -1)

    Kc, Vc = T(out["Kc"]), T(out["Vc"])   # the oracle's own caches after the append (checked above)
    y_ref = np.zeros((B, H), np.uint16)
    for b in range(B):
        p = int(d["pos"][b])
        q = qkv[b, :nq * hd].reshape(nq, hd)
        k = qkv[b, nq * hd:(nq + nkv) * hd].reshape(nkv, hd)
        q = T(bf16(rot(F.rms_norm(q, (hd,), T(w["gq"]), eps=1e-5), p)))
        k = T(bf16(rot(F.rms_norm(k, (hd,), T(w["gk"]), eps=1e-5), p)))
        assert np.array_equal(bf16(q.reshape(-1)), out["q"][b])
        assert np.array_equal(bf16(k.reshape(-1)), out["k"][b])
        keys, vals = Kc[b, :, :p + 1], Vc[b, :, :p + 1]          # [nkv, p+1, hd]
        o = F.scaled_dot_product_attention(q[:, None], keys.repeat_interleave(nq // nkv, 0),
                                           vals.repeat_interleave(nq // nkv, 0))[:, 0]
        a = T(bf16(o.reshape(-1)))
        assert np.max(np.abs(f32(out["a"][b]) - a.numpy())) <= 1e-2 * np.abs(a.numpy()).max()
        h1 = T(bf16(x[b] + T(out["a"][b]) @ T(w["Wo"]).T))
        assert np.array_equal(bf16(h1), out["h1"][b])
        xn2 = T(bf16(F.rms_norm(h1, (H,), T(w["g2"]), eps=1e-5)))
        gu = xn2 @ T(w["Wgu"]).T
        hm = T(bf16(F.silu(gu[:I]) * gu[I:]))
        y_ref[b] = bf16(h1 + hm @ T(w["Wd"]).T)
    err = np.abs(f32(out["y"]).astype(np.float64) - f32(y_ref)).max() / np.abs(f32(y_ref)).max()
    assert err <= 1e-2


def test_position_outside_the_cache_is_rejected():
    d, w = small(B=1)
    with pytest.raises(ValueError):
        oracle.decode_layer(d["X"], np.array([12], np.int32), w, d["Kc"], d["Vc"], 4, 2)
