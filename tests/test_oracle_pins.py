"""Pins of the CPU oracle against things other than itself: closed forms,
invariants, brute force, library routines, and the pages' worked examples.

Sources: "Event Tensor：用“事件张量”编译动态 Megakernel" (reading notes on the
MLSys 2026 paper), sections cited per test.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W


def f32(b):
    return W.bf16_bits_to_f32(b)


# ------------------------------------------------------------------ bf16 --

def test_bf16_rounding_known_values():
    # 1.0 exact; 1 + 2^-8 is a tie between 1.0 and 1 + 2^-7 -> even (1.0);
    # 1 + 3*2^-8 is a tie -> even (1 + 2^-6 ... mantissa 0x02)
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0], np.float32)
    got = oracle.bf16_round_bits(vals)
    assert list(got) == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x0000]


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(4096).astype(np.float32) * 7
    mine = oracle.bf16_round_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)


# --------------------------------------------------------------- split-K --
# §Split-K reduction 示例: B[i,j] = sum of 32 columns, C[i] = sum_j B[i,j].

def test_splitk_closed_form_row_sum():
    A = W.splitk_inputs(64 * 32)
    B, C = oracle.splitk(A, 32)
    assert B.shape == (2048, 4)
    row = np.array([math.fsum(map(float, r)) for r in A])
    assert np.max(np.abs(C - row)) <= 1e-12 * np.max(np.abs(A).sum(1))


def test_splitk_partials_are_column_blocks():
    A = np.arange(6 * 128, dtype=np.float32).reshape(6, 128) % 7 - 3  # small integers: exact sums
    B, C = oracle.splitk(A, 32)
    for j in range(4):
        assert np.array_equal(B[:, j], A[:, 32 * j:32 * j + 32].astype(np.float64).sum(1))
    assert np.array_equal(C, A.astype(np.float64).sum(1))


def test_splitk_ones_and_ragged():
    B, C = oracle.splitk(np.ones((3, 128), np.float32), 32)
    assert np.all(B == 32.0) and np.all(C == 128.0)
    B, C = oracle.splitk(np.ones((2, 100), np.float32), 32)  # ragged last chunk: 4 columns
    assert list(B[0]) == [32.0, 32.0, 32.0, 4.0] and np.all(C == 100.0)


# --------------------------------------------------------------- RMSNorm --

def test_rmsnorm_unit_gamma_gives_unit_rms():
    d = W.mlp_inputs(1, hidden=4096, weights=False)
    g1 = np.full(4096, 0x3F80, np.uint16)  # gamma = 1
    xn = f32(oracle.rmsnorm(d["X"], g1))
    assert abs(float((xn.astype(np.float64) ** 2).sum()) - 4096.0) < 4096 * 2 ** -7


def test_rmsnorm_matches_torch_fp64():
    d = W.mlp_inputs(4, hidden=256, weights=False)
    x = torch.from_numpy(f32(d["X"])).double()
    g = torch.from_numpy(f32(d["gamma"])).double()
    ref = torch.nn.functional.rms_norm(x, (256,), g, eps=1e-5).float()
    ref_b = ref.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.rmsnorm(d["X"], d["gamma"], 1e-5), ref_b)


def test_rmsnorm_scale_invariant():
    d = W.mlp_inputs(2, hidden=512, weights=False)
    x2 = W.f32_to_bf16_bits(f32(d["X"]) * 4.0)  # power of two: exact in bf16
    assert np.array_equal(oracle.rmsnorm(d["X"], d["gamma"], 0.0), oracle.rmsnorm(x2, d["gamma"], 0.0))


# ------------------------------------------------------------------- MLP --

def _torch_bits(t):
    return t.float().to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _torch_swiglu(x, Wgu, inter):
    g = x @ Wgu[:inter].T
    u = x @ Wgu[inter:].T
    return torch.nn.functional.silu(g) * u


def test_mlp_matches_torch_fp64_small():
    d = W.mlp_inputs(3, hidden=128, inter=96)
    Y, xn, h = oracle.mlp(d["X"], d["gamma"], d["Wgu"], d["Wd"], want_intermediates=True)
    t = lambda b: torch.from_numpy(f32(b)).double()
    xn_ref = torch.nn.functional.rms_norm(t(d["X"]), (128,), t(d["gamma"]), eps=1e-5)
    assert np.array_equal(xn, _torch_bits(xn_ref))
    h_ref = _torch_swiglu(t(xn), t(d["Wgu"]), 96)
    assert np.array_equal(h, _torch_bits(h_ref))
    y_ref = t(h) @ t(d["Wd"]).T
    assert np.array_equal(Y, _torch_bits(y_ref))


def test_mlp_identity_down_reproduces_h():
    d = W.mlp_inputs(2, hidden=64, inter=64)
    eye = W.f32_to_bf16_bits(np.eye(64, dtype=np.float32))
    Y, _, h = oracle.mlp(d["X"], d["gamma"], d["Wgu"], eye, want_intermediates=True)
    assert np.array_equal(Y, h)


def test_mlp_zero_up_gives_zero():
    d = W.mlp_inputs(2, hidden=64, inter=32)
    Wgu = d["Wgu"].copy()
    Wgu[32:] = 0
    Y = oracle.mlp(d["X"], d["gamma"], Wgu, d["Wd"])
    assert np.all(f32(Y) == 0.0)


def test_mlp_rows_equals_full():
    d = W.mlp_inputs(5, hidden=64, inter=48)
    Y = oracle.mlp(d["X"], d["gamma"], d["Wgu"], d["Wd"])
    Yr = oracle.mlp_rows(d["X"], d["gamma"], d["Wgu"], d["Wd"], [4, 0, 2])
    assert np.array_equal(Yr, Y[[4, 0, 2]])


# ------------------------------------------------------------------- MoE --

def test_router_logits_match_numpy():
    d = W.moe_inputs(5, hidden=256, inter=64, E=16, weights=False)
    got = oracle.router_logits(d["X"], d["Wr"], d["bias"])
    ref = (f32(d["X"]).astype(np.float64) @ f32(d["Wr"]).astype(np.float64).T + d["bias"]).astype(np.float32)
    assert np.max(np.abs(got - ref)) <= 1e-6 * np.max(np.abs(ref))


def test_topk_matches_full_sort_with_ties():
    rng = np.random.default_rng(3)
    l = rng.integers(-4, 5, size=(50, 32)).astype(np.float32)  # many ties
    idx, w = oracle.topk_softmax(l, 8)
    for t in range(50):
        order = np.lexsort((np.arange(32), -l[t]))  # value desc, then index asc
        assert list(idx[t]) == list(order[:8])
        sel = l[t, order[:8]].astype(np.float64)
        e = np.exp(sel - sel.max())
        assert np.allclose(w[t], e / e.sum(), rtol=1e-6, atol=0)
    assert np.allclose(w.sum(1), 1.0, atol=1e-6)


def test_group_matches_stable_sort():
    rng = np.random.default_rng(4)
    T, k, E, bm = 37, 4, 9, 5
    topk = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    g = oracle.group(topk, E, bm)
    flat = topk.ravel()
    perm_ref = np.argsort(flat, kind="stable")
    assert np.array_equal(g["perm"], perm_ref)
    assert np.array_equal(g["counts"], np.bincount(flat, minlength=E))
    assert np.array_equal(g["indptr"], np.concatenate([[0], np.cumsum(g["counts"])]))
    assert np.array_equal(g["task_indptr"], np.concatenate([[0], np.cumsum((g["counts"] + bm - 1) // bm)]))
    assert np.array_equal(g["pos"][g["perm"]], np.arange(T * k))


def test_moe_grouped_equals_per_token():
    d = W.moe_inputs(6, hidden=128, inter=32, E=8, zipf_s=0.8)
    out = oracle.moe(d["X"], d["Wr"], d["bias"], d["W1"], d["W2"], k=3, bm=2)
    Yp, tk, w = oracle.moe_per_token(d["X"], d["Wr"], d["bias"], d["W1"], d["W2"], np.arange(6), 3)
    assert np.array_equal(out["topk"], tk)
    assert np.array_equal(out["w"], w)
    assert np.array_equal(out["y"], Yp)


def test_moe_one_expert_top1_is_plain_swiglu():
    d = W.moe_inputs(4, hidden=64, inter=32, E=1, zipf_s=0.0)
    out = oracle.moe(d["X"], d["Wr"], d["bias"], d["W1"], d["W2"], k=1)
    assert np.all(out["w"] == 1.0)
    t = lambda b: torch.from_numpy(f32(b)).double()
    h = _torch_bits(_torch_swiglu(t(d["X"]), t(d["W1"][0]), 32))
    y = _torch_bits(t(h) @ t(d["W2"][0]).T)
    assert np.array_equal(out["y"], y)


def test_moe_two_experts_one_token_by_hand():
    # one token, top-2 of 2 experts: y = w0*o0 + w1*o1 with o_e = plain SwiGLU of expert e
    d = W.moe_inputs(1, hidden=32, inter=16, E=2, zipf_s=0.0)
    out = oracle.moe(d["X"], d["Wr"], d["bias"], d["W1"], d["W2"], k=2)
    t = lambda b: torch.from_numpy(f32(b)).double()
    l = (t(d["X"]) @ t(d["Wr"]).T).float().double()[0]
    e0, e1 = (0, 1) if l[0] >= l[1] else (1, 0)
    a = math.exp(float(l[e1] - l[e0]))
    w0, w1 = 1.0 / (1.0 + a), a / (1.0 + a)
    o = []
    for e in (e0, e1):
        h = t(_torch_bits(_torch_swiglu(t(d["X"]), t(d["W1"][e]), 16)))
        o.append(h @ t(d["W2"][e]).T)
    y = _torch_bits(float(np.float32(w0)) * o[0] + float(np.float32(w1)) * o[1])
    assert list(out["topk"][0]) == [e0, e1]
    assert np.array_equal(out["y"], y)


def test_zipf_bias_recipe():
    b0 = W.expert_bias(128, 0.0)
    assert np.all(b0 == 0)
    b = W.expert_bias(128, 1.2)
    assert np.allclose(np.sort(-b.astype(np.float64) / 1.2), np.log(np.arange(1, 129)), rtol=1e-6, atol=1e-6)


# -------------------------------------------------------- failure / threads --

def test_moe_grouped_rejects_malformed_grouping():
    """A grouping that does not list every pair of topk under its own expert
    is an error, not an all-zero output."""
    d = W.moe_inputs(6, hidden=64, inter=32, E=4, zipf_s=0.0)
    tk, w = oracle.topk_softmax(oracle.router_logits(d["X"], d["Wr"], d["bias"]), 2)
    g = oracle.group(tk, 4, 128)
    oracle.moe_grouped(d["X"], d["W1"], d["W2"], tk, w, g["indptr"], g["perm"])  # well formed: fine
    cases = [
        (g["indptr"], np.r_[g["perm"][1:], g["perm"][:1]]),        # pairs listed under the wrong expert
        (g["indptr"], np.r_[g["perm"][:1], g["perm"][:-1]]),       # a pair listed twice, one missing
        (np.r_[g["indptr"][:-1], g["indptr"][-1] - 1], g["perm"]),  # indptr does not cover every pair
    ]
    for ip, pm in cases:
        with pytest.raises(ValueError):
            oracle.moe_grouped(d["X"], d["W1"], d["W2"], tk, w, ip, pm)


def test_results_do_not_depend_on_thread_count():
    d = W.moe_inputs(9, hidden=128, inter=64, E=8, zipf_s=0.8)
    before = oracle.get_threads()
    outs = []
    try:
        for n in (1, 3):
            oracle.set_threads(n)
            lg = oracle.router_logits(d["X"], d["Wr"], d["bias"])
            tk, w = oracle.topk_softmax(lg, 3)
            g = oracle.group(tk, 8, 128)
            y = oracle.moe_grouped(d["X"], d["W1"], d["W2"], tk, w, g["indptr"], g["perm"])
            yt, _, _ = oracle.moe_per_token(d["X"], d["Wr"], d["bias"], d["W1"], d["W2"], list(range(9)), 3)
            outs.append((lg, y, yt))
    finally:
        oracle.set_threads(before)
    for a, b in zip(outs[0], outs[1]):
        assert np.array_equal(a, b)
