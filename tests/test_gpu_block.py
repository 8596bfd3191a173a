"""The joint-attention sub-layer around the path on the GPU against its fp64
oracle (``oracle.block``): adaLN, per-modality QKV projection with the
QK-RMSNorm and rotation fused into the GEMM epilogue, the packed attention,
per-modality output projection with bias, gate and residual fused into the
GEMM epilogue (Mage-Flow paper summary, "Native-Resolution MMDiT (NR-MMDiT)",
"Training Infrastructure").

Error model, fixed before measuring (the bounds below follow from it):
* x and v are one bf16 rounding of fp32 arithmetic on bf16 inputs (2^-9
  relative RMS each, v also inherits x's); bounds 4e-3 and 6e-3 rel-RMS;
* o is the packed attention on the sub-layer's own q_hat, k_hat, v: held to
  the forward's own bar, rel-RMS <= 5e-3;
* the output GEMM accumulates C exact bf16 products and the bias in fp32:
  whatever the order, |y32 - y| <= A = (C + 1) 2^-23 (sum_j |W_ij o_j| + |b_i|);
* h' = bf16(h + gate * y32), one rounding of at most 2^-8 of the value, so
  |h' - h'_ref| <= 2^-8 (|h'_ref| + E) + E, where E bounds the error of the
  unrounded value: |gate| (A + 8 eps_o rho_o ||W_i||_2) + 2^-23 |h'_ref|.
  The middle term carries o's error through the output projection: W_i . do
  is a sum of C terms of random sign, Gaussian with RMS eps_o rho_o ||W_i||_2
  (eps_o = 5e-3 the forward's bar, rho_o the RMS of the token's o row), taken
  at 8 sigma. Nothing in a bound depends on the value under test.
* With h = 0 and gate = 1 the output is bf16(y) alone, compared with W_o o + b_o
  computed in fp64 from the GPU's own o: the GEMM and its bias are checked
  on their own, to within one rounding plus A.
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


def gemm_acc_bound(o, w_o, b_o, mod):
    """A per element: the worst-case fp32 accumulation error of W_o o + b_o
    over C products and the bias, o [T, C], w_o [2, C, C], b_o [2, C]."""
    C = o.shape[1]
    s = np.empty_like(o)
    for m in (0, 1):
        rows = mod == m
        if rows.any():
            s[rows] = np.abs(o[rows]) @ np.abs(w_o[m]).T + np.abs(b_o[m])
    return (C + 1) * 2.0 ** -23 * s


def h_out_bound(h_ref, gate_t, acc, o_ref, w_o, mod, eps_o=5e-3, k_sigma=8.0):
    """Per element of h': one rounding of a value within E of h'_ref."""
    rho_o = np.sqrt(np.mean(o_ref ** 2, axis=1, keepdims=True))
    wnorm = np.sqrt(np.sum(w_o.astype(np.float64) ** 2, axis=2))  # [2, C]: ||W_i||_2 per output
    e = np.abs(gate_t) * (acc + k_sigma * eps_o * rho_o * wnorm[mod]) + 2.0 ** -23 * np.abs(h_ref)
    return np.ldexp(np.abs(h_ref) + e, -8) + e


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
    p = oracle_params(inp)
    sid, mod = oblock.token_sample_modality(w.samples)
    o_ref = ref["o"].reshape(-1, C)
    acc = gemm_acc_bound(o_ref, p["w_o"], p["b_o"], mod)
    bound = h_out_bound(ref["h_out"], p["gate"][sid, mod], acc, o_ref, p["w_o"], mod)
    d = np.abs(got - ref["h_out"])
    errs["h_out_bound_used"] = float(np.max(d / bound))
    report(f"{w.name}_F{fd}", errs)
    assert errs["x"][0] < 4e-3 and errs["v"][0] < 6e-3, errs
    assert errs["o"][0] <= 5e-3, errs
    assert errs["h_out_bound_used"] <= 1.0, errs


@pytest.mark.parametrize("w", BLOCKS, ids=lambda w: w.name)
def test_block_output_projection_alone(cuda_device, w):
    """h = 0 and gate = 1: the output is bf16(W_o o + b_o), compared element
    by element with the product computed in fp64 from the GPU's own o. The
    bias is drawn 10x larger than in the other tests so that an error of a
    few percent in it could not hide under the rounding."""
    inp = make_block_inputs(w)
    inp["h"] = np.zeros_like(inp["h"])
    inp["gate"] = np.ones_like(inp["gate"])
    inp["b_o"] = (inp["b_o"] * 10.0).astype(np.float32)
    t = to_dev(inp, cuda_device)
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, w.token_budget, device=cuda_device)
    ws = torch.empty(pa.block_workspace_bytes(plan), dtype=torch.uint8, device=cuda_device)
    out = pa.attn_block_fwd(t["h"], t, t, plan, workspace=ws)
    assert pa.device_error() == 0
    C = w.heads * w.head_dim
    p = oracle_params(inp)
    _, mod = oblock.token_sample_modality(w.samples)
    o = bf16_to_f64(pa.block_workspace_views(ws, plan)["o"]).reshape(-1, C)
    y_ref = oblock.linear_by_modality(o, p["w_o"], p["b_o"], w.samples)
    acc = gemm_acc_bound(o, p["w_o"], p["b_o"], mod)
    bound = np.ldexp(np.abs(y_ref) + acc, -8) + acc
    d = np.abs(bf16_to_f64(out) - y_ref)
    used = float(np.max(d / bound))
    report(f"{w.name}_y", {"y_bound_used": used,
                           "y_rel_rms": float(np.sqrt(np.mean(d ** 2) / np.mean(y_ref ** 2)))})
    assert used <= 1.0, used


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
    # h' from the GPU's attention output o: one rounding of h + gate * y32,
    # y32 within the fp32 accumulation bound of y
    o = bf16_to_f64(views["o"])[rows]
    y = np.stack([o[i] @ p["w_o"][mod[t]].T + p["b_o"][mod[t]] for i, t in enumerate(rows)])
    ref = h[rows] + p["gate"][sid[rows], mod[rows]] * y
    acc = gemm_acc_bound(o, p["w_o"], p["b_o"], mod[rows])
    e = np.abs(p["gate"][sid[rows], mod[rows]]) * acc + 2.0 ** -23 * np.abs(ref)
    bound = np.ldexp(np.abs(ref) + e, -8) + e
    d = np.abs(bf16_to_f64(out)[rows] - ref)
    assert np.all(d <= bound), float(np.max(d / bound))
