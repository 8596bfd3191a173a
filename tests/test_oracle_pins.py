"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test checks a closed form, an invariant the mathematics fixes, a special
case that reduces to a textbook form, or an independent dense brute-force
formulation. A plausible mistake in the oracle (a dropped eps, a wrong RoPE
axis or pairing, a sign error in the rotation, a swapped gamma, attention that
leaks across samples, a transposed operand) fails at least one of them.

Passages followed: Mage-Flow paper summary, "Native-Resolution MMDiT
(NR-MMDiT)" (modality-specific normalization; packing with per-sample
cumulative offsets); video overview 00:03:16 (per-sample 2D rotary embeddings);
capabilities page, "Key Capabilities" (per-sample 2D RoPE).
"""
import math

import numpy as np
import pytest

import oracle
from packed_attention_b200 import synth
from packed_attention_b200.workloads import WORKLOADS, make_inputs, random_pack

ONE_BF16 = 0x3F80  # 1.0


def bits(x):
    return synth.f64_to_bf16_bits(np.asarray(x, dtype=np.float64))


def rand_bits(seed, shape, scale=1.0):
    z = synth.normals(seed, 99, int(np.prod(shape))).reshape(shape) * scale
    return bits(z)


def ones_gammas(d):
    g = np.ones(d, dtype=np.float32)
    return {"g_q_text": g, "g_q_img": g, "g_k_text": g, "g_k_img": g}


def rand_gammas(seed, d):
    return {name: synth.bf16_bits_to_f64(bits(1 + 0.1 * synth.normals(seed, 50 + i, d))).astype(np.float32)
            for i, name in enumerate(("g_q_text", "g_q_img", "g_k_text", "g_k_img"))}


def vals(b):
    return synth.bf16_bits_to_f64(b)


# ---------------------------------------------------------------- RMSNorm ---

@pytest.mark.parametrize("d", [64, 128])
def test_rmsnorm_unit_vector_closed_form(d):
    # One nonzero entry a at dim m: mean square a^2/d, so x_hat_m = a / sqrt(a^2/d + eps).
    samples = [(1, 1, 1, 1)]  # token 0 text, token 1 image at (0, 0)
    for m, a, eps in [(0, 1.0, 0.0), (d - 1, -2.5, 0.0), (7, 0.75, 1e-2)]:
        x = np.zeros((2, 1, d), dtype=np.uint16)
        x[:, 0, m] = bits(a)
        g = np.ones(d, dtype=np.float32)
        y = oracle.qk_prologue(x, samples, g, g, eps=eps)
        expect = a / math.sqrt(a * a / d + eps)
        for t in range(2):
            assert y[t, 0, m] == pytest.approx(expect, rel=1e-14)
            others = np.delete(y[t, 0], m)
            assert np.all(others == 0.0)


def test_rmsnorm_scale_invariance_and_eps_placement():
    d = 128
    x = rand_bits(3, (1, 1, d))
    x8 = bits(vals(x) * 8.0)  # exact in bf16
    g = np.ones(d, dtype=np.float32)
    ms = float(np.mean(vals(x) ** 2))
    for eps in (0.0, 1e-6, 0.5):
        y1 = oracle.qk_prologue(np.concatenate([x, x]), [(1, 1, 1, 1)], g, g, eps=eps)[0, 0]
        y8 = oracle.qk_prologue(np.concatenate([x8, x8]), [(1, 1, 1, 1)], g, g, eps=eps)[0, 0]
        # y(8x)/y(x) = sqrt(ms + eps) / sqrt(ms + eps/64): eps sits inside the root, once.
        ratio = math.sqrt(ms + eps) / math.sqrt(ms + eps / 64.0)
        np.testing.assert_allclose(y8, y1 * ratio, rtol=1e-13, atol=0)
    # With eps = 0 the normalised row has mean square exactly 1.
    y = oracle.qk_prologue(np.concatenate([x, x]), [(1, 1, 1, 1)], g, g, eps=0.0)[0, 0]
    assert np.mean(y ** 2) == pytest.approx(1.0, rel=1e-13)


def test_rmsnorm_zero_row_is_zero():
    d = 64
    x = np.zeros((3, 2, d), dtype=np.uint16)
    g = np.full(d, 1.7, dtype=np.float32)
    y = oracle.qk_prologue(x, [(1, 1, 2, 1)], g, g, eps=1e-6)
    assert np.all(y == 0.0)


def test_gamma_selected_by_modality():
    d = 64
    samples = [(2, 1, 1, 1)]  # tokens 0, 1 text; token 2 image at (0, 0) (no rotation)
    row = rand_bits(5, (1, 1, d))
    x = np.repeat(row, 3, axis=0)
    one = np.ones(d, dtype=np.float32)
    n = oracle.qk_prologue(x, samples, one, one, eps=1e-6)
    g_text = rand_gammas(1, d)["g_q_text"]
    g_img = rand_gammas(2, d)["g_q_img"]
    y = oracle.qk_prologue(x, samples, g_text, g_img, eps=1e-6)
    np.testing.assert_allclose(y[0, 0], n[0, 0] * g_text, rtol=1e-14)
    np.testing.assert_allclose(y[1, 0], n[1, 0] * g_text, rtol=1e-14)
    np.testing.assert_allclose(y[2, 0], n[2, 0] * g_img, rtol=1e-14)


# ------------------------------------------------------------------- RoPE ---

def test_rope_identity_at_grid_origin():
    d = 128
    samples = [(1, 3, 3, 1)]  # token 0 text, token 1 image at (0, 0)
    row = rand_bits(7, (1, 2, d))
    x = np.repeat(row, 10, axis=0)
    g = rand_gammas(3, d)["g_k_img"]
    y = oracle.qk_prologue(x, samples, g, g)
    np.testing.assert_array_equal(y[1], y[0])
    assert not np.allclose(y[2], y[0])  # (0, 1) does rotate


@pytest.mark.parametrize("d", [64, 128])
def test_rope_unit_vector_angles(d):
    """e_m at grid cell (r, c) turns by r*theta_j (first half) or c*theta_j (second half)."""
    half = d // 2
    H_lat, W_lat = 5, 7
    samples = [(0, H_lat, W_lat, 1)]
    T = H_lat * W_lat
    g = np.ones(d, dtype=np.float32)
    root_d = math.sqrt(d)
    cases = [(0, 3, 2), (1, 3, 2), (half // 2 - 1, 4, 6), (2, 1, 5)]
    for j, r, c in cases:
        theta = 10000.0 ** (-2.0 * j / half)
        for axis, pos in ((0, r), (1, c)):
            for odd in (0, 1):
                m = axis * half + 2 * j + odd
                x = np.zeros((T, 1, d), dtype=np.uint16)
                x[:, 0, m] = ONE_BF16
                y = oracle.qk_prologue(x, samples, g, g, eps=0.0)[r * W_lat + c, 0]
                phi = pos * theta
                i0 = axis * half + 2 * j
                if odd == 0:   # (1, 0) -> (cos, sin)
                    want = (math.cos(phi), math.sin(phi))
                else:          # (0, 1) -> (-sin, cos)
                    want = (-math.sin(phi), math.cos(phi))
                assert y[i0] == pytest.approx(root_d * want[0], abs=1e-12)
                assert y[i0 + 1] == pytest.approx(root_d * want[1], abs=1e-12)
                mask = np.ones(d, bool)
                mask[[i0, i0 + 1]] = False
                assert np.all(y[mask] == 0.0)


def test_rope_theta_literal_values():
    # d = 64: theta_1 = 10000^(-2/32) = 10^(-1/4); d = 128: theta_1 = 10000^(-2/64) = 10^(-1/8).
    for d, theta1 in ((64, 0.5623413251903491), (128, 0.7498942093324559)):
        x = np.zeros((2, 1, d), dtype=np.uint16)
        x[:, 0, 2] = ONE_BF16  # pair j = 1, first (row) half
        g = np.ones(d, dtype=np.float32)
        y = oracle.qk_prologue(x, [(0, 2, 1, 1)], g, g, eps=0.0)[1, 0]  # token 1: (r=1, c=0)
        assert math.atan2(y[3], y[2]) == pytest.approx(theta1, abs=1e-13)


def test_rope_preserves_norm():
    d = 128
    H_lat, W_lat = 9, 11
    samples = [(1, H_lat, W_lat, 1)]
    row = rand_bits(11, (1, 3, d))
    x = np.repeat(row, 1 + H_lat * W_lat, axis=0)
    g = rand_gammas(4, d)["g_q_img"]
    y = oracle.qk_prologue(x, samples, g, g)
    ref = np.linalg.norm(y[0], axis=-1)
    for t in range(1, y.shape[0]):
        np.testing.assert_allclose(np.linalg.norm(y[t], axis=-1), ref, rtol=1e-13)


@pytest.mark.parametrize("d", [64, 128])
def test_rope_scores_depend_only_on_offset(d):
    H_lat = W_lat = 16
    samples = [(0, H_lat, W_lat, 1)]
    T = H_lat * W_lat
    qrow, krow = rand_bits(13, (1, 1, d)), rand_bits(14, (1, 1, d))
    g = np.ones(d, dtype=np.float32)
    qh = oracle.qk_prologue(np.repeat(qrow, T, 0), samples, g, g)[:, 0]
    kh = oracle.qk_prologue(np.repeat(krow, T, 0), samples, g, g)[:, 0]

    def tok(r, c):
        return r * W_lat + c

    rng = np.random.default_rng(0)
    for _ in range(40):
        r1, c1, r2, c2 = rng.integers(0, 8, size=4)
        a, b = rng.integers(0, 8, size=2)
        s0 = qh[tok(r1, c1)] @ kh[tok(r2, c2)]
        s1 = qh[tok(r1 + a, c1 + b)] @ kh[tok(r2 + a, c2 + b)]
        assert s1 == pytest.approx(s0, abs=1e-10 * d)


# ---------------------------------------------------- 3D RoPE (frame axis) ---
# Reading under test: with frame_dims = F, dims [0, F) turn by the frame index
# f, [F, F + S) by the grid row r and [F + S, d) by the column c, S = (d - F)/2;
# pair j of a part of width w turns by pos * 10000^(-2j/w).

@pytest.mark.parametrize("d,F", [(64, 8), (128, 16), (128, 32), (64, 60)])
def test_rope3d_unit_vector_angles(d, F):
    S = (d - F) // 2
    H_lat, W_lat, frames = 3, 4, 3
    samples = [(0, H_lat, W_lat, frames)]
    T = frames * H_lat * W_lat
    g = np.ones(d, dtype=np.float32)
    root_d = math.sqrt(d)
    parts = ((0, F), (F, S), (F + S, S))  # (first dim, width): frame, row, column
    for f, r, c in ((2, 1, 3), (1, 2, 0), (0, 2, 3)):
        t = f * H_lat * W_lat + r * W_lat + c
        for (first, width), pos in zip(parts, (f, r, c)):
            for j in sorted({0, min(1, width // 2 - 1), width // 2 - 1}):
                for odd in (0, 1):
                    m = first + 2 * j + odd
                    x = np.zeros((T, 1, d), dtype=np.uint16)
                    x[:, 0, m] = ONE_BF16
                    y = oracle.qk_prologue(x, samples, g, g, eps=0.0, frame_dims=F)[t, 0]
                    phi = pos * 10000.0 ** (-2.0 * j / width)
                    want = (math.cos(phi), math.sin(phi)) if odd == 0 else (-math.sin(phi), math.cos(phi))
                    i0 = first + 2 * j
                    assert y[i0] == pytest.approx(root_d * want[0], abs=1e-12)
                    assert y[i0 + 1] == pytest.approx(root_d * want[1], abs=1e-12)
                    mask = np.ones(d, bool)
                    mask[[i0, i0 + 1]] = False
                    assert np.all(y[mask] == 0.0)


def test_rope3d_theta_literal_values():
    # Widths chosen so that the frequencies are powers of ten:
    # F = 16: pair 1 turns by 10000^(-2/16) = 10^(-1/2) per frame, pair 4 by 10^-2;
    # S = 56 (d = 128): pair 7 turns by 10000^(-14/56) = 10^-1 per row;
    # d = 64, F = 8: frame pair 1 by 10^-1, S = 28: row pair 7 by 10^-2.
    cases = [(128, 16, 2, 0.31622776601683794, "f"), (128, 16, 8, 0.01, "f"),
             (128, 16, 16 + 14, 0.1, "r"), (128, 16, 16 + 56 + 14, 0.1, "c"),
             (64, 8, 2, 0.1, "f"), (64, 8, 8 + 14, 0.01, "r")]
    for d, F, m, theta, axis in cases:
        samples = [(0, 2, 2, 2)]  # token 4 + (r*2 + c): frame 1
        x = np.zeros((8, 1, d), dtype=np.uint16)
        x[:, 0, m] = ONE_BF16
        g = np.ones(d, dtype=np.float32)
        y = oracle.qk_prologue(x, samples, g, g, eps=0.0, frame_dims=F)
        # one step along the axis: frame 1 at (0, 0), frame 0 at (1, 0), frame 0 at (0, 1)
        t = {"f": 4, "r": 2, "c": 1}[axis]
        assert math.atan2(y[t, 0, m + 1], y[t, 0, m]) == pytest.approx(theta, abs=1e-13)


@pytest.mark.parametrize("d,F", [(64, 8), (128, 16)])
def test_rope3d_scores_depend_only_on_offset(d, F):
    H_lat, W_lat, frames = 6, 6, 4
    samples = [(0, H_lat, W_lat, frames)]
    T = frames * H_lat * W_lat
    qrow, krow = rand_bits(15, (1, 1, d)), rand_bits(16, (1, 1, d))
    g = np.ones(d, dtype=np.float32)
    qh = oracle.qk_prologue(np.repeat(qrow, T, 0), samples, g, g, frame_dims=F)[:, 0]
    kh = oracle.qk_prologue(np.repeat(krow, T, 0), samples, g, g, frame_dims=F)[:, 0]

    def tok(f, r, c):
        return (f * H_lat + r) * W_lat + c

    rng = np.random.default_rng(1)
    seen_frame_effect = False
    for _ in range(40):
        f1, f2 = rng.integers(0, 2, size=2)
        r1, c1, r2, c2 = rng.integers(0, 3, size=4)
        a = int(rng.integers(0, 2))
        b, c = rng.integers(0, 3, size=2)
        s0 = qh[tok(f1, r1, c1)] @ kh[tok(f2, r2, c2)]
        s1 = qh[tok(f1 + a, r1 + b, c1 + c)] @ kh[tok(f2 + a, r2 + b, c2 + c)]
        assert s1 == pytest.approx(s0, abs=1e-10 * d)
        if f1 != f2:
            s_same = qh[tok(f1, r1, c1)] @ kh[tok(f1, r2, c2)]
            seen_frame_effect |= abs(s_same - s0) > 1e-6
    assert seen_frame_effect  # the frame offset does change the score


def test_rope3d_frames_differ_only_in_frame_dims():
    # Identical raw tokens in the target (f = 0) and source (f = 1) frames:
    # row/column dims agree exactly, the target's frame dims are unrotated and
    # the source's frame dims are the target's turned by theta_j.
    d, F = 128, 16
    samples = [(3, 4, 5, 2)]
    x = rand_bits(96, (43, 2, d))
    x[23:43] = x[3:23]
    g = rand_gammas(9, d)
    y = oracle.qk_prologue(x, samples, g["g_k_text"], g["g_k_img"], frame_dims=F)
    y2d = oracle.qk_prologue(x, samples, g["g_k_text"], g["g_k_img"])
    np.testing.assert_array_equal(y[23:43, :, F:], y[3:23, :, F:])
    # the normalised values alone: every token read as text, with the image gamma
    nrm = oracle.qk_prologue(x, [(42, 1, 1, 1)], g["g_k_img"], g["g_k_img"])
    # target frame dims: the normalised values themselves (f = 0 is the identity)
    np.testing.assert_allclose(y[3:23, :, :F], nrm[3:23, :, :F], rtol=0, atol=1e-15)
    for j in range(F // 2):
        th = 10000.0 ** (-2.0 * j / F)
        a, b = y[3:23, :, 2 * j], y[3:23, :, 2 * j + 1]
        np.testing.assert_allclose(y[23:43, :, 2 * j], a * math.cos(th) - b * math.sin(th), atol=1e-13)
        np.testing.assert_allclose(y[23:43, :, 2 * j + 1], a * math.sin(th) + b * math.cos(th), atol=1e-13)
    # text tokens are never rotated, so they agree with the 2D prologue
    np.testing.assert_array_equal(y[:3], y2d[:3])


def test_rope3d_preserves_norm_and_rejects_bad_splits():
    d = 128
    samples = [(1, 3, 4, 3)]
    T = 1 + 36
    row = rand_bits(17, (1, 2, d))
    x = np.repeat(row, T, axis=0)
    g = rand_gammas(4, d)["g_q_img"]
    for F in (4, 16, 124):
        y = oracle.qk_prologue(x, samples, g, g, frame_dims=F)
        ref = np.linalg.norm(y[0], axis=-1)
        for t in range(1, T):
            np.testing.assert_allclose(np.linalg.norm(y[t], axis=-1), ref, rtol=1e-13)
    for F in (-4, 2, 6, 126, 128):
        with pytest.raises(ValueError):
            oracle.qk_prologue(x, samples, g, g, frame_dims=F)


@pytest.mark.parametrize("trial", range(4))
def test_rope3d_dense_brute_force(trial):
    rng = np.random.default_rng(700 + trial)
    samples = random_pack(rng, int(rng.integers(1, 4)), 8, 4, 3)
    d = (64, 128)[trial % 2]
    F = (8, 16, 32, 4)[trial]
    H = int(rng.integers(1, 3))
    q, k, v, g = _pack_inputs(samples, H, d, 300 + trial)
    a = oracle.joint_attn(q, k, v, g, samples, frame_dims=F)
    b = oracle.dense_attn(q, k, v, g, samples, frame_dims=F)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    if any(f > 1 for (_, _, _, f) in samples):
        assert not np.allclose(a, oracle.joint_attn(q, k, v, g, samples), atol=1e-6)


# -------------------------------------------------------------- attention ---

def _pack_inputs(samples, H, d, seed):
    T = oracle.total_tokens(samples)
    return (rand_bits(seed, (T, H, d)), rand_bits(seed + 1, (T, H, d)), rand_bits(seed + 2, (T, H, d)),
            rand_gammas(seed, d))


def _seg_bounds(samples):
    lens = [nt + f * h * w for nt, h, w, f in samples]
    starts = np.concatenate([[0], np.cumsum(lens)])
    return starts


def test_constant_v_returns_v():
    samples = [(3, 4, 5, 1), (0, 2, 3, 2), (7, 1, 1, 1)]
    H, d = 3, 64
    q, k, _, g = _pack_inputs(samples, H, d, 20)
    T = q.shape[0]
    starts = _seg_bounds(samples)
    v = np.zeros((T, H, d), dtype=np.uint16)
    const = rand_bits(21, (len(samples), H, d))
    for i in range(len(samples)):
        v[starts[i]:starts[i + 1]] = const[i]
    o = oracle.joint_attn(q, k, v, g, samples)
    for i in range(len(samples)):
        np.testing.assert_allclose(o[starts[i]:starts[i + 1]],
                                   np.broadcast_to(vals(const[i]), o[starts[i]:starts[i + 1]].shape),
                                   rtol=1e-12, atol=1e-14)


def test_zero_q_returns_segment_mean_of_v():
    samples = [(5, 3, 3, 1), (2, 6, 2, 1)]
    H, d = 2, 128
    _, k, v, g = _pack_inputs(samples, H, d, 30)
    q = np.zeros_like(k)
    o = oracle.joint_attn(q, k, v, g, samples)
    starts = _seg_bounds(samples)
    for i in range(len(samples)):
        mean = vals(v[starts[i]:starts[i + 1]]).mean(axis=0)
        np.testing.assert_allclose(o[starts[i]:starts[i + 1]],
                                   np.broadcast_to(mean, o[starts[i]:starts[i + 1]].shape),
                                   rtol=1e-12, atol=1e-14)


def test_zero_scale_is_uniform_attention():
    samples = [(4, 2, 3, 1), (1, 1, 2, 1)]
    q, k, v, g = _pack_inputs(samples, 2, 64, 35)
    o = oracle.joint_attn(q, k, v, g, samples, scale=0.0)
    starts = _seg_bounds(samples)
    for i in range(len(samples)):
        mean = vals(v[starts[i]:starts[i + 1]]).mean(axis=0)
        np.testing.assert_allclose(o[starts[i]:starts[i + 1]],
                                   np.broadcast_to(mean, o[starts[i]:starts[i + 1]].shape), rtol=1e-12)


def test_single_token_sample_returns_its_v():
    samples = [(0, 1, 1, 1), (3, 2, 2, 1), (1, 0 + 1, 1, 1)]
    q, k, v, g = _pack_inputs(samples, 2, 64, 40)
    o = oracle.joint_attn(q, k, v, g, samples)
    np.testing.assert_array_equal(o[0], vals(v[0]))


def test_two_token_sample_is_a_logistic_mix():
    # Softmax over two keys is the logistic function of the score difference.
    samples = [(1, 1, 1, 1)]  # text token 0, image token 1 at (0, 0)
    H, d = 2, 128
    q, k, v, g = _pack_inputs(samples, H, d, 45)
    o = oracle.joint_attn(q, k, v, g, samples)
    qh = np.empty((2, H, d))
    kh = np.empty((2, H, d))
    qh[0] = oracle.qk_prologue(q, samples, g["g_q_text"], g["g_q_text"])[0]
    qh[1] = oracle.qk_prologue(q, samples, g["g_q_img"], g["g_q_img"])[1]
    kh[0] = oracle.qk_prologue(k, samples, g["g_k_text"], g["g_k_text"])[0]
    kh[1] = oracle.qk_prologue(k, samples, g["g_k_img"], g["g_k_img"])[1]
    scale = 1 / math.sqrt(d)
    for t in range(2):
        for h in range(H):
            s0 = qh[t, h] @ kh[0, h] * scale
            s1 = qh[t, h] @ kh[1, h] * scale
            w0 = 1.0 / (1.0 + math.exp(s1 - s0))
            want = w0 * vals(v[0, h]) + (1 - w0) * vals(v[1, h])
            np.testing.assert_allclose(o[t, h], want, rtol=1e-12, atol=1e-14)


def test_gamma_routing_by_role_and_modality():
    samples = [(6, 3, 4, 1), (0, 2, 5, 1)]
    H, d = 2, 64
    q, k, v, g = _pack_inputs(samples, H, d, 50)
    base = oracle.joint_attn(q, k, v, g, samples)
    starts = _seg_bounds(samples)
    text_rows = np.zeros(q.shape[0], bool)
    text_rows[0:6] = True
    # A zero query gamma for text makes exactly the text queries uniform.
    g2 = dict(g, g_q_text=np.zeros(d, np.float32))
    o = oracle.joint_attn(q, k, v, g2, samples)
    mean0 = vals(v[starts[0]:starts[1]]).mean(axis=0)
    np.testing.assert_allclose(o[text_rows], np.broadcast_to(mean0, o[text_rows].shape), rtol=1e-12)
    np.testing.assert_array_equal(o[~text_rows], base[~text_rows])
    # A zero query gamma for images makes exactly the image queries uniform.
    g3 = dict(g, g_q_img=np.zeros(d, np.float32))
    o = oracle.joint_attn(q, k, v, g3, samples)
    np.testing.assert_array_equal(o[text_rows], base[text_rows])
    for i in range(2):
        sel = np.zeros_like(text_rows)
        sel[starts[i]:starts[i + 1]] = True
        sel &= ~text_rows
        mean = vals(v[starts[i]:starts[i + 1]]).mean(axis=0)
        np.testing.assert_allclose(o[sel], np.broadcast_to(mean, o[sel].shape), rtol=1e-12)
    # The text key gamma cannot reach a sample that has no text.
    g4 = dict(g, g_k_text=g["g_k_text"] * 2)
    o = oracle.joint_attn(q, k, v, g4, samples)
    np.testing.assert_array_equal(o[starts[1]:], base[starts[1]:])
    assert not np.allclose(o[:starts[1]], base[:starts[1]])


def test_packed_equals_each_sample_alone():
    rng = np.random.default_rng(1)
    samples = random_pack(rng, 4, 12, 6, 2)
    H, d = 3, 128
    q, k, v, g = _pack_inputs(samples, H, d, 60)
    packed = oracle.joint_attn(q, k, v, g, samples)
    starts = _seg_bounds(samples)
    for i, s in enumerate(samples):
        sl = slice(starts[i], starts[i + 1])
        alone = oracle.joint_attn(q[sl], k[sl], v[sl], g, [s])
        np.testing.assert_allclose(packed[sl], alone, rtol=0, atol=1e-13)


def test_sample_order_permutes_outputs():
    rng = np.random.default_rng(2)
    samples = random_pack(rng, 3, 10, 5, 1)
    H, d = 2, 64
    q, k, v, g = _pack_inputs(samples, H, d, 70)
    out = oracle.joint_attn(q, k, v, g, samples)
    starts = _seg_bounds(samples)
    order = [2, 0, 1]
    idx = np.concatenate([np.arange(starts[i], starts[i + 1]) for i in order])
    out_p = oracle.joint_attn(q[idx], k[idx], v[idx], g, [samples[i] for i in order])
    np.testing.assert_allclose(out_p, out[idx], rtol=0, atol=1e-13)


def test_dense_brute_force_on_tiny_pack():
    w = WORKLOADS[0]
    inp = make_inputs(w)
    a = oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples)
    b = oracle.dense_attn(inp["q"], inp["k"], inp["v"], inp, w.samples)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


@pytest.mark.parametrize("trial", range(6))
def test_dense_brute_force_on_random_packs(trial):
    rng = np.random.default_rng(100 + trial)
    n = int(rng.integers(1, 5))
    samples = random_pack(rng, n, 10, 5, 2)
    d = 64 if trial % 2 == 0 else 128
    H = int(rng.integers(1, 4))
    q, k, v, g = _pack_inputs(samples, H, d, 200 + trial)
    a = oracle.joint_attn(q, k, v, g, samples)
    b = oracle.dense_attn(q, k, v, g, samples)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_row_subset_matches_full_output():
    rng = np.random.default_rng(3)
    samples = random_pack(rng, 3, 8, 6, 2)
    H, d = 3, 64
    q, k, v, g = _pack_inputs(samples, H, d, 80)
    full = oracle.joint_attn(q, k, v, g, samples)
    T = q.shape[0]
    rows = rng.choice(T * H, size=min(50, T * H), replace=False)
    sub = oracle.joint_attn(q, k, v, g, samples, rows=rows, n_threads=3)
    np.testing.assert_array_equal(sub, full.reshape(T * H, d)[rows])


def test_key_outliers_cancel_in_the_norm():
    # Scaling whole raw K rows by 8 only moves the eps term: with eps = 0 nothing changes.
    samples = [(4, 4, 4, 1), (2, 3, 5, 1)]
    H, d = 2, 128
    q, k, v, g = _pack_inputs(samples, H, d, 90)
    rows = synth.choose_rows(4, synth.STREAM_OUTLIER_ROWS, k.shape[0], 5)
    k8 = k.copy()
    k8[rows] = bits(vals(k[rows]) * 8.0)
    a = oracle.joint_attn(q, k, v, g, samples, eps=0.0)
    b = oracle.joint_attn(q, k8, v, g, samples, eps=0.0)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_editing_frames_share_grid_positions():
    # Two frames with identical raw tokens give identical normalised, rotated rows.
    d = 128
    samples = [(3, 4, 5, 2)]
    T = 3 + 2 * 20
    x = rand_bits(95, (T, 2, d))
    x[23:43] = x[3:23]
    g = rand_gammas(9, d)
    y = oracle.qk_prologue(x, samples, g["g_k_text"], g["g_k_img"])
    np.testing.assert_array_equal(y[23:43], y[3:23])


def test_invalid_samples_rejected():
    assert oracle.total_tokens([(1, 0, 3, 1)]) == -1
    assert oracle.total_tokens([(-1, 2, 3, 1)]) == -1
    assert oracle.total_tokens([(1, 2, 3, 0)]) == -1
    assert oracle.total_tokens([(1, 2, 3, 1), (0, 1, 1, 2)]) == 9


def test_golden_closed_forms():
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")
    with open(path) as f:
        gold = json.load(f)
    for d in (64, 128):
        x = np.zeros((2, 1, d), dtype=np.uint16)
        x[:, 0, 2] = ONE_BF16
        g = np.ones(d, dtype=np.float32)
        y = oracle.qk_prologue(x, [(0, 2, 1, 1)], g, g, eps=0.0)[1, 0]
        assert math.atan2(y[3], y[2]) == pytest.approx(gold["rope_theta1"][str(d)], abs=1e-13)
    for c in gold["rmsnorm_one_hot"]["cases"]:
        d = c["d"]
        x = np.zeros((2, 1, d), dtype=np.uint16)
        x[:, 0, c["m"]] = bits(c["a"])
        g = np.ones(d, dtype=np.float32)
        y = oracle.qk_prologue(x, [(1, 1, 1, 1)], g, g, eps=c["eps"])
        assert y[0, 0, c["m"]] == pytest.approx(c["x_hat_m"], rel=1e-14)
