"""The five synthetic packs the path is tested and measured on, and their inputs.

Each sample is ``(n_text, H_lat, W_lat, frames)``: ``n_text`` text tokens, then
``frames`` latent grids of ``H_lat`` rows x ``W_lat`` columns, flattened row
major. Grid sizes follow the 16x latent downsampling of the tokenizer
(Mage-Flow paper summary, "Mage-VAE": 1024^2 -> 64x64); the resolutions and
aspect ratios (512^2 to 2048^2, 4:1) follow its "Native-Resolution MMDiT"
section and the 512-2048 / 4:1 range it quotes. No dataset stands behind these
inputs: every value is drawn by :mod:`packed_attention_b200.synth`.

Only shapes and value distributions live here; nothing in this module computes
any part of the attention.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

from . import synth


@dataclass(frozen=True)
class Workload:
    name: str
    samples: tuple  # of (n_text, H_lat, W_lat, frames)
    heads: int
    head_dim: int
    seed: int
    token_budget: int = 0
    # (first_token, last_token_exclusive, sigma): tokens drawn N(0, sigma) instead of N(0, 1)
    sigma_ranges: tuple = ()
    # fraction of raw K token rows (all heads) multiplied by outlier_scale
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    eps: float = 1e-6
    notes: str = field(default="", compare=False)
    # 3D RoPE: dims of head_dim that rotate by the frame index (0: 2D RoPE)
    rope_frame_dims: int = 0

    @property
    def seg_lens(self):
        return [nt + f * h * w for (nt, h, w, f) in self.samples]

    @property
    def total_tokens(self) -> int:
        return sum(self.seg_lens)

    @property
    def sum_L2(self) -> int:
        return sum(L * L for L in self.seg_lens)

    @property
    def flops(self) -> int:
        """Algorithmic FLOPs of the attention: 4 * H * d * sum_i L_i^2."""
        return 4 * self.heads * self.head_dim * self.sum_L2

    def with_heads(self, heads: int) -> "Workload":
        return Workload(self.name + f"_h{heads}", self.samples, heads, self.head_dim, self.seed,
                        self.token_budget, self.sigma_ranges, self.outlier_frac, self.outlier_scale,
                        self.eps, self.notes, self.rope_frame_dims)


WORKLOADS = {
    0: Workload("tiny_pack", ((16, 8, 8, 1), (8, 4, 16, 1)), heads=2, head_dim=64, seed=0,
                notes="two samples: 16 text + 8x8 grid, 8 text + 4x16 grid"),
    1: Workload("uniform_512sq", ((128, 32, 32, 1),) * 4, heads=24, head_dim=128, seed=1,
                notes="4 x (128 text + 32x32 grid) = 4608 tokens"),
    2: Workload("mixed_native_res",
                ((77, 32, 32, 1), (200, 48, 64, 1), (256, 64, 64, 1),
                 (40, 16, 64, 1), (128, 64, 48, 1), (99, 40, 40, 1)),
                heads=24, head_dim=128, seed=2, token_budget=15400,
                notes="six native-resolution samples, 14,688 tokens under a 15,400-token budget"),
    3: Workload("edit_1024sq", ((512, 64, 64, 2),), heads=24, head_dim=128, seed=3,
                sigma_ranges=((512 + 4096, 512 + 2 * 4096, 0.5),),
                notes="512 text + 64x64 target + 64x64 reference grid (same positions), 8704 tokens"),
    4: Workload("hires_2048sq_4to1", ((512, 128, 128, 1), (256, 32, 128, 1)), heads=24,
                head_dim=128, seed=4, outlier_frac=0.01, outlier_scale=8.0,
                notes="2048^2 sample (16,896 tokens) + 4:1 sample (4,352 tokens); 1% of K rows x8"),
}

# Editing with the frame axis of the RoPE: the 1024^2 edit pack, its source
# (reference) grid told apart from the target grid by a 3D rotation (Mage-Flow
# paper summary, "Native-Resolution MMDiT (NR-MMDiT)", Conditioning). The
# pages give no split of head_dim; F = d/8 = 16 dims for the frame leaves 56
# for each grid axis.
EXTRA_WORKLOADS = {
    "edit_1024sq_rope3d": Workload(
        "edit_1024sq_rope3d", ((512, 64, 64, 2),), heads=24, head_dim=128, seed=3,
        sigma_ranges=((512 + 4096, 512 + 2 * 4096, 0.5),), rope_frame_dims=16,
        notes="the 1024^2 edit pack under 3D RoPE: 16 frame dims, 56 per grid axis"),
}


def make_inputs(w: Workload):
    """bf16 bit patterns (uint16) for q, k, v ``[T, H, d]`` and the four gammas.

    Gammas are returned as fp32 arrays holding bf16-representable values
    ``bf16(1 + 0.1 z)``. Returns a dict of numpy arrays.
    """
    T, H, d = w.total_tokens, w.heads, w.head_dim
    n = T * H * d
    sig = np.ones(T, dtype=np.float64)
    for lo, hi, s in w.sigma_ranges:
        sig[lo:hi] = s
    out = {}
    for name, stream in (("q", synth.STREAM_Q), ("k", synth.STREAM_K), ("v", synth.STREAM_V)):
        z = synth.normals(w.seed, stream, n).reshape(T, H, d)
        if w.sigma_ranges:
            z *= sig[:, None, None]
        bits = np.empty(z.shape, dtype=np.uint16)
        rows = max(1, (1 << 22) // (H * d))
        with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
            def conv(lo):
                bits[lo:lo + rows] = synth.f64_to_bf16_bits(z[lo:lo + rows])
            list(ex.map(conv, range(0, T, rows)))
        out[name] = bits
    if w.outlier_frac > 0:
        n_rows = int(round(w.outlier_frac * T))
        rows = synth.choose_rows(w.seed, synth.STREAM_OUTLIER_ROWS, T, n_rows)
        kv = synth.bf16_bits_to_f64(out["k"][rows]) * w.outlier_scale
        out["k"][rows] = synth.f64_to_bf16_bits(kv)
        out["outlier_rows"] = rows
    for name, stream in (("g_q_text", synth.STREAM_GQ_TEXT), ("g_q_img", synth.STREAM_GQ_IMG),
                         ("g_k_text", synth.STREAM_GK_TEXT), ("g_k_img", synth.STREAM_GK_IMG)):
        g = 1.0 + 0.1 * synth.normals(w.seed, stream, d)
        out[name] = synth.bf16_bits_to_f64(synth.f64_to_bf16_bits(g)).astype(np.float32)
    return out


def random_pack(rng: np.random.Generator, n_samples: int, max_text: int, max_side: int,
                max_frames: int = 1):
    """A random list of samples for small parity and edge-case packs."""
    out = []
    for _ in range(n_samples):
        out.append((int(rng.integers(0, max_text + 1)), int(rng.integers(1, max_side + 1)),
                    int(rng.integers(1, max_side + 1)), int(rng.integers(1, max_frames + 1))))
    return tuple(out)


@dataclass(frozen=True)
class CfgPack:
    """Classifier-free guidance evaluated as one pack.

    Each request contributes two samples that share its latent grid: the
    conditional branch (its prompt's text tokens, then the grid) and the
    unconditional branch (the empty prompt, then the same grid). Both go into
    one pack and one forward instead of two (Mage-Flow paper summary,
    "Native-Resolution MMDiT (NR-MMDiT)": packed CFG inference; video
    overview, 00:04:03). The pages give no text length for the unconditional
    branch; the empty prompt is read as ``n_text_uncond`` = 0 text tokens.
    Samples are packed request by request: cond_0, uncond_0, cond_1, ...
    """
    name: str
    requests: tuple  # of (n_text_cond, H_lat, W_lat)
    heads: int
    head_dim: int
    seed: int
    n_text_uncond: int = 0
    notes: str = field(default="", compare=False)

    def samples(self, branch=None):
        """Samples of the whole pack (branch None), or of one branch ('cond' / 'uncond')."""
        out = []
        for (nt, h, w) in self.requests:
            if branch in (None, "cond"):
                out.append((nt, h, w, 1))
            if branch in (None, "uncond"):
                out.append((self.n_text_uncond, h, w, 1))
        return tuple(out)

    def packed(self) -> Workload:
        return Workload(self.name, self.samples(), self.heads, self.head_dim, self.seed,
                        notes=self.notes)

    def branch(self, branch: str) -> Workload:
        return Workload(f"{self.name}_{branch}", self.samples(branch), self.heads, self.head_dim,
                        self.seed, notes=f"{branch} branch of {self.name}")

    def branch_tokens(self, branch: str) -> np.ndarray:
        """Token indices, in the packed layout, of the given branch's samples in order."""
        idx, start = [], 0
        for i, L in enumerate(self.packed().seg_lens):
            if (i % 2 == 0) == (branch == "cond"):
                idx.append(np.arange(start, start + L))
            start += L
        return np.concatenate(idx)


CFG_PACKS = {
    "cfg_1024sq": CfgPack("cfg_1024sq", ((512, 64, 64),), heads=24, head_dim=128, seed=5,
                          notes="one 1024^2 request: cond 512 text + 64x64, uncond 64x64"),
    "cfg_mixed_native_res": CfgPack(
        "cfg_mixed_native_res", ((128, 32, 32), (256, 64, 64), (40, 16, 64), (200, 48, 64)),
        heads=24, head_dim=128, seed=6,
        notes="four requests (512^2, 1024^2, 4:1, 768x1024), each cond + uncond"),
}


# ------------------------------------------------ the sub-layer around it ---

STREAM_H, STREAM_WQKV, STREAM_BQKV, STREAM_WO, STREAM_BO = 8, 9, 10, 11, 12
STREAM_SHIFT, STREAM_SCALE, STREAM_GATE = 13, 14, 15


def make_block_inputs(w: Workload):
    """Seeded inputs of the joint-attention sub-layer around the path, for a
    pack ``w`` with hidden size C = heads * head_dim.

    h: bf16 bits [T, C], N(0, 1). Per modality (0 text, 1 image): w_qkv bf16
    bits [2, 3C, C] and w_o [2, C, C], N(0, 1/C) so that the products stay
    O(1); biases b_qkv [2, 3C], b_o [2, C] fp32, 0.02 N(0, 1). Per sample and
    modality: shift, scale, gate fp32 [n, 2, C], 0.1 N(0, 1). The four
    QK-norm gammas as in :func:`make_inputs`.
    """
    T, C, n = w.total_tokens, w.heads * w.head_dim, len(w.samples)

    def bf16(stream, shape, std):
        z = synth.normals(w.seed, stream, int(np.prod(shape))).reshape(shape) * std
        return synth.f64_to_bf16_bits(z)

    def f32(stream, shape, std):
        z = synth.normals(w.seed, stream, int(np.prod(shape))).reshape(shape) * std
        return z.astype(np.float32)

    out = {
        "h": bf16(STREAM_H, (T, C), 1.0),
        "w_qkv": bf16(STREAM_WQKV, (2, 3 * C, C), 1.0 / np.sqrt(C)),
        "b_qkv": f32(STREAM_BQKV, (2, 3 * C), 0.02),
        "w_o": bf16(STREAM_WO, (2, C, C), 1.0 / np.sqrt(C)),
        "b_o": f32(STREAM_BO, (2, C), 0.02),
        "shift": f32(STREAM_SHIFT, (n, 2, C), 0.1),
        "scale": f32(STREAM_SCALE, (n, 2, C), 0.1),
        "gate": f32(STREAM_GATE, (n, 2, C), 0.1),
    }
    g = make_inputs(Workload(w.name, ((0, 1, 1, 1),), w.heads, w.head_dim, w.seed))
    out.update({k: g[k] for k in ("g_q_text", "g_q_img", "g_k_text", "g_k_img")})
    return out
