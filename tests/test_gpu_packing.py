"""Packing on the GPU: a sample's output depends on its own tokens only.

Native-resolution packing puts samples of different sizes, and the two
branches of classifier-free guidance, into one forward (Mage-Flow paper
summary, "Native-Resolution MMDiT (NR-MMDiT)": native-resolution packing and
packed CFG inference). Attention is confined to each sample, so the packed
forward must give each sample exactly what a forward of that sample alone
gives. The kernels reach that bit for bit: every tile is laid out from the
sample's own start, keys past its end are masked to zero weight, and rows
past its end are neither stored nor allowed to steer the shared rescale
decision of their warp.
"""
import numpy as np
import pytest
import torch

import oracle
import packed_attention_b200 as pa
from packed_attention_b200.workloads import CFG_PACKS, Workload, make_inputs, random_pack
from test_gpu_parity import (MAX_ABS, REL_RMS, bf16_to_f64, compare_every_element, errors,
                             run_gpu, sample_rows)

pytestmark = pytest.mark.gpu


def gather_inputs(inp, tokens):
    out = {n: np.ascontiguousarray(inp[n][tokens]) for n in ("q", "k", "v")}
    out.update({n: inp[n] for n in pa.GAMMA_NAMES})
    return out


def bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy()


@pytest.mark.parametrize("name", sorted(CFG_PACKS))
def test_cfg_pack_equals_separate_branches(cuda_device, name):
    cp = CFG_PACKS[name]
    w = cp.packed()
    inp = make_inputs(w)
    _, _, out = run_gpu(w, inp, cuda_device)
    packed = bits(out)
    for branch in ("cond", "uncond"):
        tok = cp.branch_tokens(branch)
        wb = cp.branch(branch)
        assert wb.total_tokens == len(tok)
        _, _, ob = run_gpu(wb, gather_inputs(inp, tok), cuda_device)
        assert np.array_equal(packed[tok], bits(ob)), branch


@pytest.mark.parametrize("name", sorted(CFG_PACKS))
def test_cfg_pack_matches_oracle(cuda_device, name):
    """The packed CFG forward against the oracle on every element."""
    w = CFG_PACKS[name].packed()
    inp = make_inputs(w)
    _, _, out = run_gpu(w, inp, cuda_device)
    compare_every_element(w, inp, out, name)


@pytest.mark.parametrize("trial", range(6))
def test_each_sample_alone_is_bitwise_equal(cuda_device, trial):
    rng = np.random.default_rng(900 + trial)
    samples = random_pack(rng, int(rng.integers(2, 7)), 300, 40, 2)
    w = Workload(f"pack_{trial}", samples, heads=int(rng.integers(1, 4)),
                 head_dim=(64, 128)[trial % 2], seed=950 + trial)
    inp = make_inputs(w)
    _, _, out = run_gpu(w, inp, cuda_device)
    packed = bits(out)
    start = 0
    for i, L in enumerate(w.seg_lens):
        tok = np.arange(start, start + L)
        wi = Workload(f"pack_{trial}_s{i}", (samples[i],), w.heads, w.head_dim, w.seed)
        _, _, oi = run_gpu(wi, gather_inputs(inp, tok), cuda_device)
        assert np.array_equal(packed[tok], bits(oi)), i
        start += L


def test_schedule_does_not_change_results(cuda_device):
    """The work list's schedule (mf_schedule_work over any number of CTAs,
    with its padding entries, or none) only moves whole items between CTAs:
    forward, log-normaliser and backward are bit-identical."""
    w = Workload("sched", ((77, 12, 20, 1), (0, 9, 15, 1), (5, 1, 1, 1), (200, 8, 8, 2),
                           (31, 1, 1, 1)), heads=3, head_dim=128, seed=18)
    inp = make_inputs(w)
    t = {n: torch.from_numpy(inp[n].view(np.int16)).view(torch.bfloat16).to(cuda_device)
         for n in ("q", "k", "v")}
    t.update({n: torch.from_numpy(inp[n]).to(cuda_device) for n in pa.GAMMA_NAMES})
    dout = torch.from_numpy(
        np.random.default_rng(3).standard_normal(t["q"].shape).astype(np.float32)).to(
        cuda_device).to(torch.bfloat16)
    results = []
    for ctas in (0, None, 1, 5, 37, 1000):
        plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, device=cuda_device, ctas=ctas)
        if ctas == 5:
            assert (plan.work[:, 2] < 0).any()  # the padded layout is exercised
        out, lse = pa.joint_attention_fwd_lse(t["q"], t["k"], t["v"], t, plan, eps=w.eps)
        g = pa.joint_attention_bwd(t["q"], t["k"], t["v"], t, plan, out, lse, dout, eps=w.eps)
        assert pa.device_error() == 0
        results.append((bits(out), lse.cpu().numpy(), bits(g["dq"]), bits(g["dk"]),
                        bits(g["dv"]), [g[n].cpu().numpy() for n in pa.GAMMA_NAMES]))
    ref = results[0]
    for r in results[1:]:
        for a, b in zip(ref[:5], r[:5]):
            assert np.array_equal(a, b)
        for a, b in zip(ref[5], r[5]):
            assert np.array_equal(a, b)
