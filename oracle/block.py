"""fp64 oracle of the attention sub-layer around the packed path (numpy).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: the tests, the smoke
check and the benchmark's CPU legs may use it; the product path never does.

What it computes, in the order of the NR-MMDiT's joint-attention sub-layer
[Mage-Flow paper summary, "Native-Resolution MMDiT (NR-MMDiT)": an MMDiT
with modality-specific normalization and joint self-attention; "Training
Infrastructure": adaptive normalization / RoPE / gating fused into kernels].
Readings adopted where the pages give no formula (adaLN-Zero as in DiT, the
text and image streams of an MMDiT with their own parameters):

  for token t of sample s with modality m (text or image):
  1. x_t   = LN(h_t) * (1 + scale[s, m]) + shift[s, m]
             LN over the C channels, no affine, (h - mean) / sqrt(var + eps_ln)
  2. qkv_t = W_qkv[m] x_t + b_qkv[m]          (W_qkv[m]: [3C, C]; q, k, v = thirds)
  3. o     = the packed joint attention of q, k, v ([T, H, d] views), with
             its QK-RMSNorm and RoPE (oracle.attn_grad, fp64)
  4. y_t   = W_o[m] o_t + b_o[m]               (W_o[m]: [C, C])
  5. h'_t  = h_t + gate[s, m] * y_t
All arithmetic fp64; matrix products by numpy.
"""
from __future__ import annotations

import numpy as np

from . import attn_grad

GAMMAS = ("g_q_text", "g_q_img", "g_k_text", "g_k_img")


def token_sample_modality(samples):
    """Per token of the pack: its sample index and modality (0 text, 1 image)."""
    sid, mod = [], []
    for i, (nt, gh, gw, f) in enumerate(samples):
        n_img = f * gh * gw
        sid += [i] * (nt + n_img)
        mod += [0] * nt + [1] * n_img
    return np.asarray(sid, dtype=np.int64), np.asarray(mod, dtype=np.int64)


def layer_norm(x, eps):
    """Row-wise (h - mean) / sqrt(var + eps) over the last axis, no affine."""
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    return (x - mean) / np.sqrt(var + eps)


def adaln(h, shift, scale, samples, eps_ln):
    """Step 1: x = LN(h) * (1 + scale[s, m]) + shift[s, m], [T, C]."""
    sid, mod = token_sample_modality(samples)
    return layer_norm(h, eps_ln) * (1.0 + scale[sid, mod]) + shift[sid, mod]


def linear_by_modality(x, w, b, samples):
    """x_t W[m]^T + b[m] with m the token's modality; w: [2, N, K], b: [2, N]."""
    _, mod = token_sample_modality(samples)
    out = np.empty((x.shape[0], w.shape[1]), dtype=np.float64)
    for m in (0, 1):
        rows = mod == m
        if rows.any():
            out[rows] = x[rows] @ w[m].T + b[m]
    return out


def block_fwd(h, p, samples, heads, head_dim, eps_ln=1e-6, eps=1e-6, frame_dims=0,
              scale=None):
    """The whole sub-layer. ``p`` holds shift, scale, gate ([n, 2, C]), w_qkv
    ([2, 3C, C]), b_qkv ([2, 3C]), w_o ([2, C, C]), b_o ([2, C]) and the four
    QK-norm gammas, all as float64-convertible arrays. Returns a dict of every
    intermediate (x, q, k, v, o, y) and the output ``h_out``."""
    h = np.asarray(h, dtype=np.float64)
    T, C = h.shape
    if C != heads * head_dim:
        raise ValueError("hidden size must be heads * head_dim")
    f = {k: np.asarray(v, dtype=np.float64) for k, v in p.items()}
    x = adaln(h, f["shift"], f["scale"], samples, eps_ln)
    qkv = linear_by_modality(x, f["w_qkv"], f["b_qkv"], samples)
    q, k, v = (qkv[:, i * C:(i + 1) * C].reshape(T, heads, head_dim) for i in range(3))
    o = attn_grad(q, k, v, {g: f[g] for g in GAMMAS}, samples, eps=eps, scale=scale,
                  frame_dims=frame_dims)["out"]
    y = linear_by_modality(o.reshape(T, C), f["w_o"], f["b_o"], samples)
    sid, mod = token_sample_modality(samples)
    h_out = h + f["gate"][sid, mod] * y
    return {"x": x, "q": q, "k": k, "v": v, "o": o, "y": y, "h_out": h_out}
