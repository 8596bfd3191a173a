"""The seeded input generator and the workload table (host only)."""
import numpy as np
import pytest
import torch

from packed_attention_b200 import synth
from packed_attention_b200.workloads import CFG_PACKS, WORKLOADS, make_inputs


def test_splitmix64_known_answers():
    # Published outputs of SplitMix64 started from state 0 (Vigna's splitmix64.c):
    # the n-th output is the finaliser applied to n * 0x9E3779B97F4A7C15.
    idx = np.arange(1, 4, dtype=np.uint64)
    with np.errstate(over="ignore"):
        got = synth._mix64(idx * synth._GOLDEN)
    assert [int(x) for x in got] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_streams_are_deterministic_and_distinct():
    a = synth.splitmix64(1, 0, 1000)
    b = synth.splitmix64(1, 0, 1000)
    c = synth.splitmix64(1, 1, 1000)
    d = synth.splitmix64(2, 0, 1000)
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, c) and not np.array_equal(a, d)
    # Counter-based: any window of the stream can be produced on its own.
    np.testing.assert_array_equal(synth.splitmix64(1, 0, 100, offset=900), a[900:])


def test_normals_moments():
    z = synth.normals(7, 3, 400_000)
    assert abs(z.mean()) < 0.01
    assert abs(z.std() - 1.0) < 0.01
    assert abs(np.mean(z ** 4) - 3.0) < 0.05


def test_bf16_rounding_matches_torch_on_fp32_values():
    x32 = (synth.normals(0, 0, 100_000) * 3).astype(np.float32)
    ours = synth.f64_to_bf16_bits(x32.astype(np.float64))
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def test_bf16_rounding_ties_to_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties to the even mantissa (1.0).
    assert synth.f64_to_bf16_bits(np.array([1 + 2.0 ** -8]))[0] == 0x3F80
    assert synth.f64_to_bf16_bits(np.array([1 + 3 * 2.0 ** -8]))[0] == 0x3F82
    assert synth.f64_to_bf16_bits(np.array([-(1 + 2.0 ** -8 + 2.0 ** -30)]))[0] == 0xBF81
    with pytest.raises(ValueError):
        synth.f64_to_bf16_bits(np.array([np.inf]))


def test_choose_rows_distinct_sorted():
    r = synth.choose_rows(4, synth.STREAM_OUTLIER_ROWS, 21248, 212)
    assert len(np.unique(r)) == 212 and np.all(np.diff(r) > 0) and r.max() < 21248


@pytest.mark.parametrize("cfg,T,sum_l2,n_seg", [
    (0, 152, 11_584, 2),
    (1, 4608, 5_308_416, 4),
    (2, 14_688, 45_116_786, 6),
    (3, 8704, 75_759_616, 1),
    (4, 21_248, 304_414_720, 2),
])
def test_workload_sizes(cfg, T, sum_l2, n_seg):
    w = WORKLOADS[cfg]
    assert w.total_tokens == T
    assert w.sum_L2 == sum_l2
    assert len(w.samples) == n_seg
    assert w.flops == 4 * w.heads * w.head_dim * sum_l2


def test_tiny_inputs_shapes_and_distributions():
    w = WORKLOADS[0]
    inp = make_inputs(w)
    assert inp["q"].shape == (152, 2, 64) and inp["q"].dtype == np.uint16
    g = inp["g_q_text"]
    assert g.shape == (64,) and g.dtype == np.float32
    # gammas are bf16-representable and close to 1 + 0.1 N(0, 1)
    np.testing.assert_array_equal(synth.bf16_bits_to_f64(synth.f64_to_bf16_bits(g.astype(np.float64))), g)
    assert 0.5 < g.min() and g.max() < 1.5


def test_edit_reference_tokens_have_half_sigma():
    w = WORKLOADS[3].with_heads(2)
    inp = make_inputs(w)
    v = synth.bf16_bits_to_f64(inp["v"])
    assert abs(v[:4608].std() - 1.0) < 0.02
    assert abs(v[4608:].std() - 0.5) < 0.01


@pytest.mark.parametrize("name", sorted(CFG_PACKS))
def test_cfg_pack_layout(name):
    cp = CFG_PACKS[name]
    w = cp.packed()
    # request by request: cond (prompt + grid), then uncond (empty prompt + same grid)
    assert len(w.samples) == 2 * len(cp.requests)
    for r, (nt, h, wd) in enumerate(cp.requests):
        assert w.samples[2 * r] == (nt, h, wd, 1)
        assert w.samples[2 * r + 1] == (cp.n_text_uncond, h, wd, 1)
    cond, uncond = cp.branch_tokens("cond"), cp.branch_tokens("uncond")
    # the two branches partition the pack's tokens, each in increasing order
    both = np.sort(np.concatenate([cond, uncond]))
    np.testing.assert_array_equal(both, np.arange(w.total_tokens))
    assert np.all(np.diff(cond) > 0) and np.all(np.diff(uncond) > 0)
    assert len(cond) == cp.branch("cond").total_tokens
    assert len(uncond) == cp.branch("uncond").total_tokens
    # the first token of each branch segment is where the pack places it
    starts = np.concatenate([[0], np.cumsum(w.seg_lens)[:-1]])
    assert cond[0] == starts[0] and uncond[0] == starts[1]
