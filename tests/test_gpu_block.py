"""The joint-attention sub-layer around the path on the GPU against its fp64
oracle (``oracle.block``): adaLN, per-modality QKV projection with the
QK-RMSNorm and rotation fused into the GEMM epilogue, the packed attention,
per-modality output projection with bias, gate and residual fused into the
GEMM epilogue (Mage-Flow paper summary, "Native-Resolution MMDiT (NR-MMDiT)",
"Training Infrastructure").

Tolerances: x, v are one bf16 rounding of fp32 arithmetic on bf16 inputs
(2^-8 relative, with slack for the fp32 reduction over C); o carries the
attention's error (rel-RMS 5e-3, the forward's bound); h' = h + gate * y is
rounded to bf16 once, so its error is within one ulp of h' (half an ulp,
doubled where the rounding crosses a power of two) plus the error of gate * y
(0.1 of the update's RMS; a CPU model of these roundings and of the
attention's error reproduces the measured figures exactly).
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import block as oblock
import packed_attention_b200 as pa
from packed_attention_b200 import synth
from packed_attention_b200.workloads import WORKLOADS, Workload, make_block_inputs
from test_gpu_parity import bf16_to_f64

pytestmark = pytest.mark.gpu


def to_dev(inp, dev):
    t = {}
    for k, v in inp.items():
        if v.dtype == np.uint16:
            t[k] = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).to(dev)
        else:
            t[k] = torch.from_numpy(np.ascontiguousarray(v)).to(dev)
    return t


def oracle_params(inp):
    return {k: (synth.bf16_bits_to_f64(v) if v.dtype == np.uint16 else v.astype(np.float64))
            for k, v in inp.items() if k != "h"}


def run_block(w: Workload, dev, frame_dims=0):
    inp = make_block_inputs(w)
    t = to_dev(inp, dev)
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, w.token_budget, device=dev)
    ws = torch.empty(pa.block_workspace_bytes(plan), dtype=torch.uint8, device=dev)
    out = pa.attn_block_fwd(t["h"], t, t, plan, frame_dims=frame_dims, workspace=ws)
    assert pa.device_error() == 0
    return inp, plan, ws, out


def rel(got, ref):
    d = got - ref
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return float(np.sqrt(np.mean(d ** 2))) / rms, float(np.max(np.abs(d))) / rms


def report(name, errs):
    path = os.environ.get("MF_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"block": name, **errs}) + "\n")


BLOCKS = [
    Workload("block_tiny_d64", ((16, 8, 8, 1), (8, 4, 16, 1)), heads=2, head_dim=64, seed=30),
    Workload("block_ragged_d128", ((77, 12, 20, 1), (0, 9, 15, 1), (5, 1, 1, 1), (200, 8, 8, 2)),
             heads=2, head_dim=128, seed=31),
    Workload("block_mixed_h4", ((40, 16, 16, 1), (130, 4, 64, 1), (3, 1, 1, 1)), heads=4,
             head_dim=128, seed=32),
]


@pytest.mark.parametrize("w", BLOCKS, ids=lambda w: w.name)
@pytest.mark.parametrize("frame_dims", [0, 16])
def test_block_matches_oracle(cuda_device, w, frame_dims):
    fd = frame_dims if w.head_dim == 128 else frame_dims // 2
    inp, plan, ws, out = run_block(w, cuda_device, fd)
    h = synth.bf16_bits_to_f64(inp["h"])
    ref = oblock.block_fwd(h, oracle_params(inp), w.samples, w.heads, w.head_dim, frame_dims=fd)
    views = pa.block_workspace_views(ws, plan)
    errs = {}
    C = w.heads * w.head_dim
    for key in ("x", "v", "o"):
        r = ref[key].reshape(-1, C)
        errs[key] = rel(bf16_to_f64(views[key]), r)
    got = bf16_to_f64(out)
    upd = ref["h_out"] - h
    d = got - ref["h_out"]
    errs["h_out_vs_update_rms"] = (float(np.sqrt(np.mean(d ** 2)) / np.sqrt(np.mean(upd ** 2))),
                                   float(np.max(np.abs(d))))
    report(f"{w.name}_F{fd}", errs)
    assert errs["x"][0] < 4e-3 and errs["v"][0] < 6e-3, errs
    assert errs["o"][0] < 1e-2, errs
    # h' is rounded once to bf16: within one ulp of the larger of the two
    # values (half an ulp, doubled where the rounding crosses a power of two)
    # plus the error of gate * y: |gate| reaches 4 of its sigmas and y carries
    # the attention's error (rel-RMS ~3.5e-3, tails to ~5 sigma), which puts
    # |gate * dy| near 0.04 of the update's RMS; allowed: 0.1
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.maximum(np.abs(ref["h_out"]), np.abs(got)),
                                              1e-30))) - 7)
    bad = np.abs(d) > ulp + 0.1 * np.sqrt(np.mean(upd ** 2)) + 1e-6
    assert not bad.any(), (int(bad.sum()), errs, ref["h_out"][bad][:4], got[bad][:4])


def test_block_gate_zero_returns_h(cuda_device):
    w = BLOCKS[1]
    inp = make_block_inputs(w)
    inp["gate"] = np.zeros_like(inp["gate"])
    t = to_dev(inp, cuda_device)
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, device=cuda_device)
    out = pa.attn_block_fwd(t["h"], t, t, plan)
    assert pa.device_error() == 0
    assert torch.equal(out.view(torch.int16), t["h"].view(torch.int16))


def test_block_full_size_sampled(cuda_device):
    """The 1024^2 edit pack with the 24 x 128 hidden size: every stage at full
    size, on sampled rows. The attention is tested on its own elsewhere; here
    the output projection is checked from the GPU's own attention output."""
    import oracle
    w = WORKLOADS[3]
    inp, plan, ws, out = run_block(w, cuda_device)
    C, H, D = w.heads * w.head_dim, w.heads, w.head_dim
    h = synth.bf16_bits_to_f64(inp["h"])
    p = oracle_params(inp)
    views = pa.block_workspace_views(ws, plan)
    x = oblock.adaln(h, p["shift"], p["scale"], w.samples, 1e-6)
    assert rel(bf16_to_f64(views["x"]), x)[0] < 4e-3
    rows = np.sort(np.random.default_rng(5).choice(w.total_tokens, 256, replace=False))
    sid, mod = oblock.token_sample_modality(w.samples)
    xr = bf16_to_f64(views["x"])[rows]  # the GEMM's own input
    qkv = np.stack([xr[i] @ p["w_qkv"][mod[t]].T + p["b_qkv"][mod[t]] for i, t in enumerate(rows)])
    # v: one rounding of the fp32 product
    assert rel(bf16_to_f64(views["v"])[rows], qkv[:, 2 * C:])[0] < 4e-3
    # q_hat: RMSNorm and rotation of the full pack's q, evaluated on these rows
    q_full = np.zeros((w.total_tokens, H, D))
    q_full[rows] = qkv[:, :C].reshape(-1, H, D)
    q_bits = synth.f64_to_bf16_bits(q_full)
    qh_ref = oracle.qk_prologue(q_bits, w.samples, p["g_q_text"], p["g_q_img"])[rows]
    qh = bf16_to_f64(views["q_hat"])[rows]
    assert rel(qh, qh_ref)[0] < 6e-3
    # h' from the GPU's attention output o
    o = bf16_to_f64(views["o"])[rows]
    y = np.stack([o[i] @ p["w_o"][mod[t]].T + p["b_o"][mod[t]] for i, t in enumerate(rows)])
    ref = h[rows] + p["gate"][sid[rows], mod[rows]] * y
    d = bf16_to_f64(out)[rows] - ref
    got = bf16_to_f64(out)[rows]
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.maximum(np.abs(ref), np.abs(got)), 1e-30))) - 7)
    assert np.all(np.abs(d) <= ulp + 1e-3), float(np.max(np.abs(d)))
