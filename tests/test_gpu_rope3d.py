"""3D RoPE (frame, row, column) on the GPU against the oracle.

Editing samples concatenate the source latents with the target latents and
tell them apart with a frame dimension of the rotary embedding (Mage-Flow
paper summary, "Native-Resolution MMDiT (NR-MMDiT)", Conditioning). The
library's reading: dims [0, F) turn by the frame index, then two parts of
(d - F) / 2 dims by the grid row and column (``mf_qk_prologue_3d``,
``mf_joint_attn_fwd_3d``).
"""
import numpy as np
import pytest
import torch

import oracle
import packed_attention_b200 as pa
from packed_attention_b200.workloads import EXTRA_WORKLOADS, Workload, make_inputs, random_pack
from test_gpu_parity import (MAX_ABS, REL_RMS, bf16_to_f64, errors, sample_rows, to_dev)

pytestmark = pytest.mark.gpu

EDIT3D = EXTRA_WORKLOADS["edit_1024sq_rope3d"]


def run3d(w: Workload, inp, dev):
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, w.token_budget, device=dev)
    t = to_dev(inp, dev)
    out = pa.joint_attention(t["q"], t["k"], t["v"], t, plan, eps=w.eps,
                             frame_dims=w.rope_frame_dims)
    assert pa.device_error() == 0
    return plan, t, out


@pytest.mark.parametrize("w", [EDIT3D.with_heads(1),
                               Workload("frames_d64", ((7, 6, 9, 3), (0, 5, 5, 2), (30, 4, 16, 1)),
                                        heads=3, head_dim=64, seed=41, rope_frame_dims=8),
                               Workload("frames_d128_f4", ((3, 7, 5, 4),), heads=2, head_dim=128,
                                        seed=42, rope_frame_dims=4)],
                         ids=lambda w: w.name)
def test_prologue_3d_matches_oracle(cuda_device, w):
    inp = make_inputs(w)
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, w.token_budget, device=cuda_device)
    t = to_dev(inp, cuda_device)
    ws = plan.new_workspace()
    pa.qk_prologue(t["q"], t["k"], t, plan, ws, eps=w.eps, frame_dims=w.rope_frame_dims)
    qh, kh = pa.workspace_views(ws, plan)
    for got, x, gt, gi in ((qh, "q", "g_q_text", "g_q_img"), (kh, "k", "g_k_text", "g_k_img")):
        ref = oracle.qk_prologue(inp[x], w.samples, inp[gt], inp[gi], eps=w.eps,
                                 frame_dims=w.rope_frame_dims)
        g = bf16_to_f64(got)
        # one bf16 rounding of fp32 arithmetic (see the 2D prologue test)
        slack = 1e-5 * np.max(np.abs(ref), axis=-1, keepdims=True)
        bad = np.abs(g - ref) > 2.0 ** -7 * np.abs(ref) + slack
        assert not bad.any(), f"{bad.sum()} of {bad.size} {x}_hat elements off by more than 1 ulp"


def test_frame_dims_zero_is_the_2d_path(cuda_device):
    w = EDIT3D.with_heads(2)
    inp = make_inputs(w)
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, device=cuda_device)
    t = to_dev(inp, cuda_device)
    a = pa.joint_attention(t["q"], t["k"], t["v"], t, plan)             # mf_joint_attn_fwd
    ws = plan.new_workspace()
    from packed_attention_b200._native import check, lib
    import ctypes
    out = torch.empty_like(t["q"])
    P = ctypes.c_void_p
    check("mf_joint_attn_fwd_3d", lib().mf_joint_attn_fwd_3d(
        P(t["q"].data_ptr()), P(t["k"].data_ptr()), P(t["v"].data_ptr()),
        *[P(t[n].data_ptr()) for n in pa.GAMMA_NAMES], P(plan.cu_seqlens.data_ptr()),
        P(plan.segs.data_ptr()), plan.n_samples, P(plan.work.data_ptr()), plan.n_work,
        plan.total_tokens, plan.heads, plan.head_dim, 1e-6, 0, 0.0, P(out.data_ptr()),
        P(ws.data_ptr()), ws.numel(), P(torch.cuda.current_stream().cuda_stream)))
    assert pa.device_error() == 0
    assert torch.equal(a.view(torch.int16), out.view(torch.int16))


def test_edit_pack_3d_sampled_rows(cuda_device):
    w = EDIT3D
    inp = make_inputs(w)
    _, _, out = run3d(w, inp, cuda_device)
    got_all = bf16_to_f64(out)
    assert np.all(np.isfinite(got_all))
    rows = sample_rows(w, np.random.default_rng(33))
    ref = oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps, rows=rows,
                            frame_dims=w.rope_frame_dims)
    max_abs, rel_rms = errors(got_all.reshape(-1, w.head_dim)[rows], ref)
    assert max_abs <= MAX_ABS and rel_rms <= REL_RMS, (max_abs, rel_rms)
    # the frame axis matters: the 2D forward of the same inputs differs
    ref2d = oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps, rows=rows)
    assert np.sqrt(np.mean((ref - ref2d) ** 2)) > 10 * REL_RMS * np.sqrt(np.mean(ref ** 2))


def test_edit_pack_3d_every_element(cuda_device):
    """The 1024^2 edit pack with the frame axis: every element of the output
    against the oracle."""
    from test_gpu_parity import compare_every_element
    w = EDIT3D
    inp = make_inputs(w)
    _, _, out = run3d(w, inp, cuda_device)
    compare_every_element(w, inp, out, w.name)


@pytest.mark.parametrize("trial", range(4))
def test_random_packs_3d_full_compare(cuda_device, trial):
    rng = np.random.default_rng(800 + trial)
    samples = random_pack(rng, int(rng.integers(1, 5)), 200, 20, 3)
    d = (64, 128)[trial % 2]
    F = int(rng.integers(1, d // 4)) * 4  # a multiple of 4 in [4, d - 4]
    w = Workload(f"random3d_{trial}", samples, heads=int(rng.integers(1, 4)), head_dim=d,
                 seed=850 + trial, rope_frame_dims=F)
    inp = make_inputs(w)
    _, _, out = run3d(w, inp, cuda_device)
    ref = oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps,
                            frame_dims=F)
    max_abs, rel_rms = errors(bf16_to_f64(out), ref)
    assert max_abs <= MAX_ABS and rel_rms <= REL_RMS, (F, max_abs, rel_rms)
