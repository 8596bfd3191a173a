"""Pins of the oracle's gradients to facts that do not come from the oracle.

The backward is the derivative of the forward by the chain rule (the pages
report their speedup for training the NR-MMDiT: Mage-Flow video overview,
00:05:08; paper summary, "Training Infrastructure"). Central finite
differences of the forward are the independent check of every gradient;
closed forms and invariants pin the rest: constant values kill the q/k
gradients, the value gradients of a sample sum to the sum of its output
gradients, RMSNorm's scale invariance makes each input gradient orthogonal to
its input, a one-token sample passes the gradient straight to v, and packing
changes nothing.
"""
import numpy as np
import pytest

import oracle
from packed_attention_b200 import synth
from packed_attention_b200.workloads import WORKLOADS, make_inputs, random_pack

NAMES = ("g_q_text", "g_q_img", "g_k_text", "g_k_img")


def rand_problem(seed, samples, H, d):
    rng = np.random.default_rng(seed)
    T = oracle.total_tokens(samples)
    q, k, v, G = (rng.standard_normal((T, H, d)) for _ in range(4))
    gam = {n: 1.0 + 0.1 * rng.standard_normal(d) for n in NAMES}
    return q, k, v, G, gam


def loss(q, k, v, gam, samples, G, **kw):
    return float(np.sum(oracle.attn_grad(q, k, v, gam, samples, **kw)["out"] * G))


@pytest.mark.parametrize("d,F,eps", [(16, 0, 1e-6), (16, 4, 1e-6), (8, 4, 0.3), (12, 0, 0.0)])
def test_gradients_match_central_differences(d, F, eps):
    samples = [(2, 2, 3, 1), (0, 1, 2, 2), (3, 1, 1, 1)]
    H = 2
    q, k, v, G, gam = rand_problem(10 + d + F, samples, H, d)
    kw = dict(eps=eps, frame_dims=F)
    g = oracle.attn_grad(q, k, v, gam, samples, dout=G, **kw)
    rng = np.random.default_rng(d * 100 + F)
    h = 1e-6
    for name, grad in (("q", g["dq"]), ("k", g["dk"]), ("v", g["dv"])):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in q.shape)
            args = {"q": q, "k": k, "v": v}
            plus, minus = args[name].copy(), args[name].copy()
            plus[idx] += h
            minus[idx] -= h
            fd = (loss(**{**args, name: plus}, gam=gam, samples=samples, G=G, **kw) -
                  loss(**{**args, name: minus}, gam=gam, samples=samples, G=G, **kw)) / (2 * h)
            assert grad[idx] == pytest.approx(fd, rel=1e-6, abs=1e-8), (name, idx)
    for nm in NAMES:
        for m in rng.choice(d, size=4, replace=False):
            plus = {**gam, nm: gam[nm].copy()}
            minus = {**gam, nm: gam[nm].copy()}
            plus[nm][m] += h
            minus[nm][m] -= h
            fd = (loss(q, k, v, plus, samples, G, **kw) - loss(q, k, v, minus, samples, G, **kw)) / (2 * h)
            assert g["dgamma"][nm][m] == pytest.approx(fd, rel=1e-6, abs=1e-8), (nm, m)


def test_forward_equals_the_bf16_oracle():
    w = WORKLOADS[0]
    inp = make_inputs(w)
    q, k, v = (synth.bf16_bits_to_f64(inp[n]) for n in ("q", "k", "v"))
    out = oracle.attn_grad(q, k, v, {n: inp[n] for n in NAMES}, w.samples)["out"]
    ref = oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)


def test_constant_values_give_zero_query_and_key_gradients():
    samples = [(3, 2, 4, 1), (1, 3, 3, 2)]
    H, d = 2, 16
    q, k, v, G, gam = rand_problem(3, samples, H, d)
    start = 0
    for (nt, gh, gw, f) in samples:
        L = nt + f * gh * gw
        v[start:start + L] = v[start]  # one value vector per (sample, head)
        start += L
    g = oracle.attn_grad(q, k, v, gam, samples, dout=G, frame_dims=4)
    assert np.max(np.abs(g["dq"])) < 1e-12 and np.max(np.abs(g["dk"])) < 1e-12
    for nm in NAMES:
        assert np.max(np.abs(g["dgamma"][nm])) < 1e-12


def test_value_gradients_sum_to_output_gradients():
    samples = [(2, 3, 3, 1), (0, 2, 5, 1), (4, 1, 1, 1)]
    H, d = 3, 16
    q, k, v, G, gam = rand_problem(4, samples, H, d)
    g = oracle.attn_grad(q, k, v, gam, samples, dout=G)
    start = 0
    for (nt, gh, gw, f) in samples:
        L = nt + f * gh * gw
        np.testing.assert_allclose(g["dv"][start:start + L].sum(0), G[start:start + L].sum(0),
                                   rtol=0, atol=1e-12)
        start += L


def test_input_gradients_orthogonal_to_inputs_without_eps():
    samples = [(2, 3, 4, 1), (1, 2, 2, 2)]
    H, d = 2, 16
    q, k, v, G, gam = rand_problem(5, samples, H, d)
    g = oracle.attn_grad(q, k, v, gam, samples, dout=G, eps=0.0, frame_dims=8)
    # RMSNorm makes the forward invariant to scaling a (token, head) row of q or k
    np.testing.assert_allclose(np.sum(g["dq"] * q, axis=-1), 0.0, atol=1e-12)
    np.testing.assert_allclose(np.sum(g["dk"] * k, axis=-1), 0.0, atol=1e-12)
    assert np.max(np.abs(g["dq"])) > 1e-3  # and the gradients themselves are not zero


def test_one_token_sample_passes_the_gradient_to_v():
    samples = [(0, 1, 1, 1), (1, 2, 2, 1)]
    H, d = 2, 8
    q, k, v, G, gam = rand_problem(6, samples, H, d)
    g = oracle.attn_grad(q, k, v, gam, samples, dout=G)
    np.testing.assert_allclose(g["dv"][0], G[0], rtol=0, atol=1e-15)
    assert np.all(g["dq"][0] == 0.0) and np.all(g["dk"][0] == 0.0)


def test_packed_gradients_equal_each_sample_alone():
    rng = np.random.default_rng(8)
    samples = random_pack(rng, 3, 5, 4, 2)
    H, d = 2, 16
    q, k, v, G, gam = rand_problem(7, samples, H, d)
    g = oracle.attn_grad(q, k, v, gam, samples, dout=G, frame_dims=4)
    start = 0
    dg_sum = {nm: np.zeros(d) for nm in NAMES}
    for smp in samples:
        L = smp[0] + smp[3] * smp[1] * smp[2]
        sl = slice(start, start + L)
        gi = oracle.attn_grad(q[sl], k[sl], v[sl], gam, [smp], dout=G[sl], frame_dims=4)
        for key in ("out", "dq", "dk", "dv"):
            np.testing.assert_allclose(g[key][sl], gi[key], rtol=0, atol=1e-13)
        for nm in NAMES:
            dg_sum[nm] += gi["dgamma"][nm]
        start += L
    for nm in NAMES:
        np.testing.assert_allclose(g["dgamma"][nm], dg_sum[nm], rtol=0, atol=1e-12)


def test_grad_rejects_bad_arguments():
    samples = [(1, 2, 2, 1)]
    q, k, v, G, gam = rand_problem(9, samples, 1, 16)
    with pytest.raises(ValueError):
        oracle.attn_grad(q, k, v, gam, samples, dout=G, frame_dims=6)
    with pytest.raises(ValueError):
        oracle.attn_grad(q, k, v, gam, [(1, 2, 2, 0)], dout=G)
    with pytest.raises(ValueError):
        oracle.attn_grad(q, k[:, :, :8], v, gam, samples, dout=G)


def test_lse_is_the_log_normaliser_of_the_scores():
    # log sum_u exp(s_tu) over the sample, from the prologue's q_hat, k_hat
    samples = [(2, 2, 3, 1), (1, 1, 1, 1), (0, 1, 1, 1)]
    H, d = 2, 16
    q, k, v, G, gam = rand_problem(12, samples, H, d)
    qb, kb = synth.f64_to_bf16_bits(q), synth.f64_to_bf16_bits(k)
    qv, kv, vv = (synth.bf16_bits_to_f64(x) for x in (qb, kb, synth.f64_to_bf16_bits(v)))
    g32 = {n: gam[n].astype(np.float32).astype(np.float64) for n in NAMES}
    lse = oracle.attn_grad(qv, kv, vv, g32, samples)["lse"]
    qh = oracle.qk_prologue(qb, samples, g32["g_q_text"], g32["g_q_img"])
    kh = oracle.qk_prologue(kb, samples, g32["g_k_text"], g32["g_k_img"])
    start = 0
    for (nt, gh, gw, f) in samples:
        L = nt + f * gh * gw
        for h in range(H):
            s = qh[start:start + L, h] @ kh[start:start + L, h].T / np.sqrt(d)
            mx = s.max(axis=1, keepdims=True)
            ref = (mx + np.log(np.exp(s - mx).sum(axis=1, keepdims=True)))[:, 0]
            np.testing.assert_allclose(lse[start:start + L, h], ref, rtol=0, atol=1e-12)
        start += L
    # a one-token sample: lse = its own score
    t = start - 1
    for h in range(H):
        assert lse[t, h] == pytest.approx(qh[t, h] @ kh[t, h] / np.sqrt(d), abs=1e-12)
