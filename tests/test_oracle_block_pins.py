"""Pins of the sub-layer oracle (``oracle.block``) to closed forms and
invariants that do not come from the oracle itself.

The sub-layer: adaLN modulation, per-modality QKV projection, the packed
joint attention (pinned in test_oracle_pins.py), per-modality output
projection and the gated residual (Mage-Flow paper summary,
"Native-Resolution MMDiT (NR-MMDiT)" and "Training Infrastructure").
"""
import numpy as np
import pytest

import oracle
from oracle import block
from packed_attention_b200 import synth
from packed_attention_b200.workloads import Workload, make_block_inputs

SAMPLES = [(3, 2, 3, 1), (0, 2, 2, 2), (5, 1, 1, 1)]
H, D = 2, 8
C = H * D


def params(seed=1, samples=SAMPLES):
    w = Workload("pin", tuple(samples), H, D, seed)
    inp = make_block_inputs(w)
    p = {k: (synth.bf16_bits_to_f64(v) if v.dtype == np.uint16 else v.astype(np.float64))
         for k, v in inp.items() if k != "h"}
    return synth.bf16_bits_to_f64(inp["h"]), p


def test_layer_norm_closed_form():
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    # mean 2.5, variance 1.25: (x - 2.5) / sqrt(1.25)
    np.testing.assert_allclose(block.layer_norm(x, 0.0),
                               [[-1.5, -0.5, 0.5, 1.5]] / np.sqrt(1.25), rtol=0, atol=1e-15)
    # eps inside the root: variance 1.25 + 0.75 = 2
    np.testing.assert_allclose(block.layer_norm(x, 0.75), [[-1.5, -0.5, 0.5, 1.5]] / np.sqrt(2.0),
                               rtol=0, atol=1e-15)
    rng = np.random.default_rng(0)
    y = block.layer_norm(rng.standard_normal((5, 64)) * 3 + 7, 0.0)
    np.testing.assert_allclose(y.mean(axis=1), 0.0, atol=1e-13)
    np.testing.assert_allclose((y ** 2).mean(axis=1), 1.0, atol=1e-12)


def test_token_routing():
    sid, mod = block.token_sample_modality(SAMPLES)
    # sample 0: 3 text + 6 image; sample 1: 8 image; sample 2: 5 text + 1 image
    assert sid.tolist() == [0] * 9 + [1] * 8 + [2] * 6
    assert mod.tolist() == [0] * 3 + [1] * 6 + [1] * 8 + [0] * 5 + [1]


def test_adaln_modulation_per_sample_and_modality():
    h, p = params()
    x = block.adaln(h, p["shift"], p["scale"], SAMPLES, 1e-6)
    # scale = -1 leaves only the shift
    x0 = block.adaln(h, p["shift"], -np.ones_like(p["scale"]), SAMPLES, 1e-6)
    sid, mod = block.token_sample_modality(SAMPLES)
    np.testing.assert_array_equal(x0, p["shift"][sid, mod])
    # changing the shift of (sample 1, image) moves only those tokens, by that much
    s2 = p["shift"].copy()
    s2[1, 1] += 0.5
    x2 = block.adaln(h, s2, p["scale"], SAMPLES, 1e-6)
    moved = (sid == 1) & (mod == 1)
    np.testing.assert_allclose(x2[moved] - x[moved], 0.5, atol=1e-14)
    np.testing.assert_array_equal(x2[~moved], x[~moved])


def test_linear_uses_the_tokens_modality():
    h, p = params()
    x = block.adaln(h, p["shift"], p["scale"], SAMPLES, 1e-6)
    out = block.linear_by_modality(x, p["w_qkv"], p["b_qkv"], SAMPLES)
    _, mod = block.token_sample_modality(SAMPLES)
    for t in (0, 4, 12, 20, 22):
        m = mod[t]
        ref = [sum(p["w_qkv"][m, n, c] * x[t, c] for c in range(C)) + p["b_qkv"][m, n]
               for n in range(3 * C)]
        np.testing.assert_allclose(out[t], ref, rtol=0, atol=1e-12)


def test_zero_gate_is_the_identity_and_zero_projection_adds_the_bias():
    h, p = params()
    p0 = dict(p, gate=np.zeros_like(p["gate"]))
    np.testing.assert_array_equal(block.block_fwd(h, p0, SAMPLES, H, D)["h_out"], h)
    p1 = dict(p, w_o=np.zeros_like(p["w_o"]))
    sid, mod = block.token_sample_modality(SAMPLES)
    ref = h + p["gate"][sid, mod] * p["b_o"][mod]
    np.testing.assert_allclose(block.block_fwd(h, p1, SAMPLES, H, D)["h_out"], ref, rtol=0,
                               atol=1e-14)


def test_qkv_thirds_feed_q_k_v():
    # q and k projections zero: q_hat = k_hat = 0, uniform attention, so o is
    # the per-sample mean of v; with the v third = identity and no bias, v = x.
    h, p = params()
    w = np.zeros_like(p["w_qkv"])
    w[:, 2 * C:, :] = np.eye(C)
    pz = dict(p, w_qkv=w, b_qkv=np.zeros_like(p["b_qkv"]))
    r = block.block_fwd(h, pz, SAMPLES, H, D)
    x = block.adaln(h, p["shift"], p["scale"], SAMPLES, 1e-6)
    np.testing.assert_allclose(r["v"].reshape(-1, C), x, rtol=0, atol=1e-14)
    start = 0
    for (nt, gh, gw, f) in SAMPLES:
        L = nt + f * gh * gw
        mean = x[start:start + L].mean(axis=0)
        np.testing.assert_allclose(r["o"][start:start + L].reshape(L, C), np.tile(mean, (L, 1)),
                                   rtol=0, atol=1e-13)
        start += L


def test_block_on_a_pack_equals_each_sample_alone():
    h, p = params()
    full = block.block_fwd(h, p, SAMPLES, H, D, frame_dims=4)["h_out"]
    start = 0
    for i, smp in enumerate(SAMPLES):
        L = smp[0] + smp[3] * smp[1] * smp[2]
        pi = dict(p, shift=p["shift"][i:i + 1], scale=p["scale"][i:i + 1], gate=p["gate"][i:i + 1])
        alone = block.block_fwd(h[start:start + L], pi, [smp], H, D, frame_dims=4)["h_out"]
        np.testing.assert_allclose(full[start:start + L], alone, rtol=0, atol=1e-13)
        start += L


def test_attention_stage_is_the_pinned_attention():
    # the sub-layer's attention is the same function the path's oracle computes
    h, p = params()
    r = block.block_fwd(h, p, SAMPLES, H, D)
    ref = oracle.attn_grad(r["q"], r["k"], r["v"], {g: p[g] for g in block.GAMMAS}, SAMPLES)["out"]
    np.testing.assert_array_equal(r["o"], ref)
