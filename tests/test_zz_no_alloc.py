"""The allocation-free entry point, mf_joint_attn_fwd_static_scratch.

It serves callers that cannot allocate device memory: a plugin that is given
a stream but no allocator, code running inside a global-mode stream capture
(where cudaMalloc is not allowed), or a latency-critical loop that cannot
afford cudaMalloc's implicit device synchronisation. Its scratch is an array
inside the library instead of a caller workspace.

These tests call it through the C ABI and compare it with the regular
workspace entry point, mf_joint_attn_fwd, on two calls in a row (the array
keeps the previous call's contents, which must not leak into the next
result). This file sorts last so that a run stopping at the first failure has
already run every other test; it also passes when run alone.
"""
import ctypes

import numpy as np
import pytest
import torch

import packed_attention_b200 as pa
from packed_attention_b200 import _native
from packed_attention_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_RMS = 5e-3


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _static_call(t, plan, out, eps, stream):
    return _native.lib().mf_joint_attn_fwd_static_scratch(
        _p(t["q"]), _p(t["k"]), _p(t["v"]), _p(t["g_q_text"]), _p(t["g_q_img"]),
        _p(t["g_k_text"]), _p(t["g_k_img"]), _p(plan.cu_seqlens), _p(plan.segs),
        plan.n_samples, _p(plan.work), plan.n_work, plan.total_tokens, plan.heads, plan.head_dim,
        float(eps), 0.0, _p(out), ctypes.c_void_p(stream.cuda_stream))


def _inputs(w, dev):
    inp = make_inputs(w)
    t = {n: torch.from_numpy(inp[n].view(np.int16)).view(torch.bfloat16).to(dev)
         for n in ("q", "k", "v")}
    t.update({n: torch.from_numpy(inp[n]).to(dev) for n in pa.GAMMA_NAMES})
    return t


def _errors(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    d = a - b
    return float(np.abs(d).max()), float(np.sqrt((d ** 2).mean() / (b ** 2).mean()))


# The 512^2 batch (4 x 1152 tokens, 24 heads) needs 56.6 MB of scratch: it fits.
PACKS = [WORKLOADS[1],
         Workload("ragged", ((77, 12, 20, 1), (0, 9, 15, 1), (5, 1, 1, 1)), heads=3,
                  head_dim=64, seed=31)]


@pytest.mark.parametrize("w", PACKS, ids=[w.name for w in PACKS])
def test_static_scratch_matches_workspace_entry(cuda_device, w):
    assert pa.workspace_bytes(w.total_tokens, w.heads, w.head_dim) <= \
        _native.MF_STATIC_SCRATCH_BYTES
    t = _inputs(w, cuda_device)
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, w.token_budget, device=cuda_device)
    stream = torch.cuda.current_stream()
    ref = pa.joint_attention(t["q"], t["k"], t["v"], t, plan, eps=w.eps)
    for _ in range(2):  # two calls in a row over the same shared scratch
        out = torch.full_like(ref, float("nan"))
        assert _static_call(t, plan, out, w.eps, stream) == 0
        assert pa.device_error(stream) == 0
        max_abs, rel_rms = _errors(out, ref)
        assert max_abs <= MAX_ABS and rel_rms <= REL_RMS, (max_abs, rel_rms)
        # Same kernels on the same inputs: in practice bit-identical.
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_static_scratch_rejects_packs_that_do_not_fit(cuda_device):
    w = WORKLOADS[3]  # 8704 tokens x 24 heads: 107 MB of scratch, more than the array
    assert pa.workspace_bytes(w.total_tokens, w.heads, w.head_dim) > \
        _native.MF_STATIC_SCRATCH_BYTES
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, device=cuda_device)
    small = torch.zeros(16, dtype=torch.bfloat16, device=cuda_device)
    g = torch.ones(w.head_dim, dtype=torch.float32, device=cuda_device)
    t = {"q": small, "k": small, "v": small, "g_q_text": g, "g_q_img": g, "g_k_text": g,
         "g_k_img": g}
    out = torch.zeros(16, dtype=torch.bfloat16, device=cuda_device)
    # Refused on size before anything is launched (the small buffers are never read).
    assert _static_call(t, plan, out, w.eps, torch.cuda.current_stream()) == -4
    assert pa.device_error() == 0
