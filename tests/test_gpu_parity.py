"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Bar: max-abs error <= 2e-2 and relative RMS error <= 5e-3 over the compared
elements (bf16 output, fp32 accumulation); the prologue's q_hat / k_hat
within one bf16 rounding of the oracle. Small packs are compared element by
element in full. The five full-size packs run in the same launch
configuration the benchmark times and are compared on every element of the
output (the oracle's full output is cached on disk per workload) and, as a
fast smoke, on sampled rows (every segment's first and last rows, tile
boundaries, ragged tails and random rows).
"""
import hashlib
import json
import os
import time

import numpy as np
import pytest
import torch

import oracle
import packed_attention_b200 as pa
from packed_attention_b200 import synth
from packed_attention_b200.workloads import WORKLOADS, Workload, make_inputs, random_pack

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_RMS = 5e-3


def to_dev(inp, dev):
    t = {}
    for name in ("q", "k", "v"):
        t[name] = torch.from_numpy(inp[name].view(np.int16)).view(torch.bfloat16).to(dev)
    for name in pa.GAMMA_NAMES:
        t[name] = torch.from_numpy(inp[name]).to(dev)
    return t


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def errors(got, ref):
    diff = got - ref
    max_abs = float(np.max(np.abs(diff)))
    rel_rms = float(np.sqrt(np.mean(diff ** 2)) / np.sqrt(np.mean(ref ** 2)))
    return max_abs, rel_rms


def run_gpu(w: Workload, inp, dev, out=None):
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, w.token_budget, device=dev)
    t = to_dev(inp, dev)
    out = pa.joint_attention(t["q"], t["k"], t["v"], t, plan, eps=w.eps, out=out)
    assert pa.device_error() == 0
    return plan, t, out


def sample_rows(w: Workload, rng, n_random=256):
    """Flat row indices token * H + head: segment edges, tile edges, tails, random."""
    T, H = w.total_tokens, w.heads
    toks = set()
    start = 0
    for L in w.seg_lens:
        end = start + L
        for t in (start, start + 1, end - 2, end - 1):
            if start <= t < end:
                toks.add(t)
        for b in range(start + 127, end, 128):
            toks.update({b, min(b + 1, end - 1)})
        last = start + (L - 1) // 128 * 128  # first row of the ragged tail tile
        toks.update(range(last, min(last + 3, end)))
        start = end
    toks = np.array(sorted(toks), dtype=np.int64)
    heads_e = rng.integers(0, H, size=len(toks))
    rows = set((toks * H + heads_e).tolist())
    rows.update(rng.integers(0, T * H, size=n_random).tolist())
    return np.array(sorted(rows), dtype=np.int64)


# ------------------------------------------------------------- prologue ---

@pytest.mark.parametrize("cfg,heads", [(0, None), (2, 2), (3, 1)])
def test_prologue_matches_oracle(cuda_device, cfg, heads):
    w = WORKLOADS[cfg] if heads is None else WORKLOADS[cfg].with_heads(heads)
    check_prologue(w, cuda_device)


@pytest.mark.parametrize("d", (64, 128))
@pytest.mark.parametrize("heads", (5, 11, 13, 22, 24))
def test_prologue_head_groups(cuda_device, heads, d):
    """A warp of the prologue covers 32 / (d/8) heads per instruction (2 at
    d = 128, 4 at d = 64) and keeps five such groups in flight: head counts
    whose last group is partial, with and without groups refilled beyond the
    first five, on 74 tokens (a partial last block of 8 tokens)."""
    w = Workload(f"heads{heads}_d{d}", ((13, 5, 7, 1), (0, 3, 4, 2), (1, 1, 1, 1)),
                 heads=heads, head_dim=d, seed=90 + heads)
    assert w.total_tokens == 74
    check_prologue(w, cuda_device)


def check_prologue(w: Workload, cuda_device):
    inp = make_inputs(w)
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, w.token_budget, device=cuda_device)
    t = to_dev(inp, cuda_device)
    ws = plan.new_workspace()
    pa.qk_prologue(t["q"], t["k"], t, plan, ws, eps=w.eps)
    qh, kh = pa.workspace_views(ws, plan)
    for got, x, gt, gi in ((qh, "q", "g_q_text", "g_q_img"), (kh, "k", "g_k_text", "g_k_img")):
        ref = oracle.qk_prologue(inp[x], w.samples, inp[gt], inp[gi], eps=w.eps)
        g = bf16_to_f64(got)
        # fp32 arithmetic rounded once to bf16: within one bf16 ulp (2^-7
        # relative) plus the fp32 error of the norm and rotation, which is
        # relative to the row's magnitude, not to an element that cancels.
        slack = 1e-5 * np.max(np.abs(ref), axis=-1, keepdims=True)
        bad = np.abs(g - ref) > 2.0 ** -7 * np.abs(ref) + slack
        assert not bad.any(), f"{bad.sum()} of {bad.size} {x}_hat elements off by more than 1 ulp"
        # and within half an ulp (2^-8 relative bounds it) for nearly all
        assert np.mean(np.abs(g - ref) <= 2.0 ** -8 * np.abs(ref) + slack) > 0.999


# ------------------------------------------------------- small packs, full ---

SMALL_PACKS = [
    ("tiny_pack", WORKLOADS[0]),
    ("ragged_d128", Workload("ragged_d128", ((77, 12, 20, 1), (0, 9, 15, 1), (5, 1, 1, 1),
                                             (200, 8, 8, 2)), heads=3, head_dim=128, seed=11)),
    ("ragged_d64", Workload("ragged_d64", ((13, 10, 13, 1), (128, 1, 1, 1), (0, 16, 8, 1)),
                            heads=2, head_dim=64, seed=12)),
    ("tile_edges", Workload("tile_edges", ((0, 1, 1, 1), (0, 1, 127, 1), (0, 1, 128, 1),
                                           (0, 1, 129, 1), (1, 16, 16, 1), (0, 1, 257, 1)),
                            heads=2, head_dim=128, seed=13)),
    ("config2_shapes_h1", WORKLOADS[2].with_heads(1)),
    # sample ends at and one past the 32-row boundaries of a softmax warp's
    # output rows (the epilogue stores a warp's rows together)
    ("warp_edges", Workload("warp_edges", ((31, 1, 1, 1), (32, 1, 1, 1), (62, 1, 1, 1),
                                           (63, 1, 1, 1), (95, 1, 1, 1), (0, 1, 97, 1),
                                           (0, 8, 20, 1)), heads=2, head_dim=128, seed=16)),
    ("warp_edges_d64", Workload("warp_edges_d64", ((31, 1, 1, 1), (0, 1, 33, 1), (63, 1, 1, 1),
                                                   (0, 5, 19, 1)), heads=3, head_dim=64, seed=17)),
]


@pytest.mark.parametrize("name,w", SMALL_PACKS, ids=[n for n, _ in SMALL_PACKS])
def test_small_pack_full_compare(cuda_device, name, w):
    inp = make_inputs(w)
    _, _, out = run_gpu(w, inp, cuda_device)
    ref = oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps)
    got = bf16_to_f64(out)
    assert np.all(np.isfinite(got))
    max_abs, rel_rms = errors(got, ref)
    assert max_abs <= MAX_ABS and rel_rms <= REL_RMS, (max_abs, rel_rms)


def test_long_sample_sampled_rows(cuda_device):
    """One sample of 131,072 tokens: 512 work items of 1,024 key steps each,
    on sampled rows (the first, the last, 96 random tokens, both heads)."""
    w = Workload("long_131k", ((0, 256, 512, 1),), heads=2, head_dim=128, seed=19)
    inp = make_inputs(w)
    _, _, out = run_gpu(w, inp, cuda_device)
    rng = np.random.default_rng(11)
    toks = np.unique(np.concatenate([[0, 1, w.total_tokens - 1],
                                     rng.choice(w.total_tokens, 96, replace=False)]))
    rows = (toks[:, None] * w.heads + np.arange(w.heads)[None, :]).reshape(-1)
    ref = oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps, rows=rows)
    got = bf16_to_f64(out).reshape(-1, w.head_dim)[rows]
    max_abs, rel_rms = errors(got, ref)
    assert max_abs <= MAX_ABS and rel_rms <= REL_RMS, (max_abs, rel_rms)


@pytest.mark.parametrize("trial", range(4))
def test_random_packs_full_compare(cuda_device, trial):
    rng = np.random.default_rng(500 + trial)
    samples = random_pack(rng, int(rng.integers(1, 7)), 300, 24, 2)
    w = Workload(f"random_{trial}", samples, heads=int(rng.integers(1, 4)),
                 head_dim=(64, 128)[trial % 2], seed=600 + trial)
    inp = make_inputs(w)
    _, _, out = run_gpu(w, inp, cuda_device)
    ref = oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps)
    max_abs, rel_rms = errors(bf16_to_f64(out), ref)
    assert max_abs <= MAX_ABS and rel_rms <= REL_RMS, (max_abs, rel_rms)


@pytest.mark.parametrize("d", (64, 128))
def test_many_small_samples_every_element(cuda_device, d):
    """A pack of 600 samples of 1 to ~100 tokens (text only, grid only and
    both; one and two frames), so that thousands of segment boundaries fall
    inside warps, tiles and prologue blocks (600 work items per head): every
    element against the oracle."""
    rng = np.random.default_rng(9100 + d)
    samples = random_pack(rng, 600, 12, 7, 2)
    w = Workload(f"many_{d}", samples, heads=3, head_dim=d, seed=9200 + d)
    assert len(w.seg_lens) == 600 and min(w.seg_lens) >= 1
    inp = make_inputs(w)
    _, _, out = run_gpu(w, inp, cuda_device)
    ref = oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps)
    max_abs, rel_rms = errors(bf16_to_f64(out), ref)
    assert max_abs <= MAX_ABS and rel_rms <= REL_RMS, (max_abs, rel_rms)


# ------------------------------------------------ full-size packs, sampled ---

@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_full_size_config_sampled_rows(cuda_device, cfg):
    w = WORKLOADS[cfg]
    inp = make_inputs(w)
    _, _, out = run_gpu(w, inp, cuda_device)
    got_all = bf16_to_f64(out)
    assert np.all(np.isfinite(got_all))
    rng = np.random.default_rng(cfg)
    rows = sample_rows(w, rng)
    ref = oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps, rows=rows)
    got = got_all.reshape(-1, w.head_dim)[rows]
    max_abs, rel_rms = errors(got, ref)
    report = os.environ.get("MF_PARITY_REPORT")  # optional: append the figures to a JSON-lines file
    if report:
        with open(report, "a") as f:
            f.write(json.dumps({"config": cfg, "workload": w.name, "rows": int(len(rows)),
                                "max_abs": max_abs, "rel_rms": rel_rms}) + "\n")
    assert max_abs <= MAX_ABS and rel_rms <= REL_RMS, (max_abs, rel_rms)


# ----------------------------------------- full-size packs, every element ---

CACHE_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), ".oracle_cache")


def _cache_key(w: Workload) -> str:
    """Changes whenever the oracle's code, the input generator or the workload
    (shapes, seed, value recipe) changes."""
    h = hashlib.sha256(repr(w).encode())
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for rel in ("oracle/oracle.cpp", "packed_attention_b200/synth.py",
                "packed_attention_b200/workloads.py"):
        with open(os.path.join(root, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def oracle_full_output(w: Workload, inp):
    """The oracle's whole ``[T, H, d]`` output for workload ``w`` (fp64
    arithmetic on all host cores), cached on disk as fp32 under
    ``tests/.oracle_cache`` so that a rerun on the same machine only reads it
    back. fp32 storage moves a value by at most 2^-24 relative, five orders of
    magnitude below the tolerances it is compared at."""
    path = os.path.join(CACHE_DIR, f"{w.name}-{_cache_key(w)}.npy")
    if os.path.exists(path):
        return np.load(path).astype(np.float64), 0.0
    t0 = time.perf_counter()
    ref = oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps,
                            frame_dims=w.rope_frame_dims)
    sec = time.perf_counter() - t0
    os.makedirs(CACHE_DIR, exist_ok=True)
    tmp = path + f".tmp{os.getpid()}.npy"
    np.save(tmp, ref.astype(np.float32))
    os.replace(tmp, path)
    return ref, sec


def compare_every_element(w: Workload, inp, out, tag):
    """Every element of ``out`` (bf16 [T, H, d] on the GPU) against the
    oracle: the bar over all T*H*d elements, and the same bar on each head
    alone (so that an error confined to some heads cannot hide in the
    average)."""
    got = out.float().cpu().numpy()
    assert np.all(np.isfinite(got))
    ref, oracle_s = oracle_full_output(w, inp)
    sq_diff = sq_ref = 0.0
    max_abs = 0.0
    per_head = []
    for h in range(w.heads):
        d = got[:, h, :].astype(np.float64) - ref[:, h, :]
        r = ref[:, h, :]
        hd, hr, hm = float(np.sum(d * d)), float(np.sum(r * r)), float(np.max(np.abs(d)))
        per_head.append((hm, float(np.sqrt(hd / hr))))
        sq_diff += hd
        sq_ref += hr
        max_abs = max(max_abs, hm)
    rel_rms = float(np.sqrt(sq_diff / sq_ref))
    report = os.environ.get("MF_PARITY_REPORT")
    if report:
        with open(report, "a") as f:
            f.write(json.dumps({"config": tag, "workload": w.name, "compared": "every element",
                                "elements": int(got.size), "max_abs": max_abs,
                                "rel_rms": rel_rms,
                                "worst_head_rel_rms": max(r for _, r in per_head),
                                "oracle_seconds": oracle_s}) + "\n")
    assert max_abs <= MAX_ABS and rel_rms <= REL_RMS, (max_abs, rel_rms)
    bad = [(h, m, r) for h, (m, r) in enumerate(per_head) if m > MAX_ABS or r > REL_RMS]
    assert not bad, bad


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_full_size_config_every_element(cuda_device, cfg):
    """Every element of the full-size pack's output against the oracle."""
    w = WORKLOADS[cfg]
    inp = make_inputs(w)
    _, _, out = run_gpu(w, inp, cuda_device)
    compare_every_element(w, inp, out, cfg)


# --------------------------------------------------------------- hygiene ---

def test_canary_rows_untouched_and_deterministic(cuda_device):
    w = SMALL_PACKS[1][1]
    inp = make_inputs(w)
    T, H, d = w.total_tokens, w.heads, w.head_dim
    guard = 200
    buf = torch.full(((T + 2 * guard) * H * d,), -1000.0, dtype=torch.bfloat16, device=cuda_device)
    out = buf[guard * H * d:(guard + T) * H * d].view(T, H, d)
    _, _, out = run_gpu(w, inp, cuda_device, out=out)
    first = out.clone()
    torch.cuda.synchronize()
    pre, post = buf[:guard * H * d], buf[(guard + T) * H * d:]
    assert torch.all(pre == -1000.0) and torch.all(post == -1000.0)
    _, _, out = run_gpu(w, inp, cuda_device, out=out)
    assert torch.equal(first.view(torch.int16), out.view(torch.int16))


def test_host_buffer_path_matches_device_path(cuda_device):
    w = SMALL_PACKS[2][1]
    inp = make_inputs(w)
    plan, t, out = run_gpu(w, inp, cuda_device)
    host = {n: t[n].cpu().pin_memory() for n in ("q", "k", "v", *pa.GAMMA_NAMES)}
    res = pa.joint_attention_host(host["q"], host["k"], host["v"], host, plan, eps=w.eps)
    torch.cuda.synchronize()
    assert torch.equal(res.view(torch.int16), out.cpu().view(torch.int16))


def test_key_outliers_are_harmless(cuda_device):
    # Config 4's recipe (1% of raw K rows x8) on a small pack: parity holds.
    w = Workload("outliers", ((64, 12, 12, 1), (30, 6, 24, 1)), heads=2, head_dim=128, seed=21,
                 outlier_frac=0.01, outlier_scale=8.0)
    inp = make_inputs(w)
    assert len(inp["outlier_rows"]) == round(0.01 * w.total_tokens)
    _, _, out = run_gpu(w, inp, cuda_device)
    ref = oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps)
    max_abs, rel_rms = errors(bf16_to_f64(out), ref)
    assert max_abs <= MAX_ABS and rel_rms <= REL_RMS


def test_explicit_softmax_scale(cuda_device):
    w = Workload("scaled", ((10, 8, 9, 1), (3, 5, 5, 1)), heads=2, head_dim=64, seed=22)
    inp = make_inputs(w)
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, device=cuda_device)
    t = to_dev(inp, cuda_device)
    for scale in (0.05, 0.3):
        out = pa.joint_attention(t["q"], t["k"], t["v"], t, plan, eps=w.eps, softmax_scale=scale)
        ref = oracle.joint_attn(inp["q"], inp["k"], inp["v"], inp, w.samples, eps=w.eps, scale=scale)
        max_abs, rel_rms = errors(bf16_to_f64(out), ref)
        assert max_abs <= MAX_ABS and rel_rms <= REL_RMS, (scale, max_abs, rel_rms)


def test_softmax_exp2_accuracy(cuda_device):
    """The exponential the softmax uses (the MUFU unit's approximate exp2)
    against fp64: relative error below 1e-5 wherever the result is a normal
    number, i.e. far below the 2^-9 relative rounding of P to bf16, so the
    approximation costs nothing measurable in the attention output. Results
    below the normal range flush to zero (the softmax's masked keys use -inf)."""
    import ctypes
    from packed_attention_b200 import _native
    xs = np.concatenate([np.linspace(-125.0, 8.0, 1_000_001), np.arange(-125, 9, dtype=np.float64),
                         np.arange(-125, 9) + 0.5, [0.0, -0.0, 7.999999, -1e-7, 1e-7]])
    x = torch.tensor(xs, dtype=torch.float32, device=cuda_device)
    y = torch.empty_like(x)
    st = torch.cuda.current_stream()
    assert _native.lib().mf_selftest_exp2(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()),
                                          x.numel(), ctypes.c_void_p(st.cuda_stream)) == 0
    got = y.cpu().numpy().astype(np.float64)
    ref = np.exp2(x.cpu().numpy().astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1e-5, rel.max()
    x2 = torch.tensor([-130.0, -200.0, -float("inf"), -3e38], dtype=torch.float32, device=cuda_device)
    y2 = torch.empty_like(x2)
    assert _native.lib().mf_selftest_exp2(ctypes.c_void_p(x2.data_ptr()), ctypes.c_void_p(y2.data_ptr()),
                                          4, ctypes.c_void_p(st.cuda_stream)) == 0
    assert np.all(y2.cpu().numpy() == 0.0)


def test_host_pipeline_matches_device_path(cuda_device):
    """HostPipeline (uploads, forwards and read-backs overlapped on three
    streams) gives every batch exactly what the device call gives it."""
    w = Workload("pipe", ((30, 12, 12, 1), (5, 7, 9, 2)), heads=3, head_dim=128, seed=40)
    sets = []
    for seed in (40, 41, 42):
        inp = make_inputs(Workload(w.name, w.samples, w.heads, w.head_dim, seed))
        host = {n: torch.from_numpy(inp[n].view(np.int16)).view(torch.bfloat16).pin_memory()
                for n in ("q", "k", "v")}
        host.update({n: torch.from_numpy(inp[n]).pin_memory() for n in pa.GAMMA_NAMES})
        sets.append((inp, host))
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, device=cuda_device)
    pipe = pa.HostPipeline(plan)
    outs = []
    for i in range(7):
        _, host = sets[i % 3]
        o = torch.empty((w.total_tokens, w.heads, w.head_dim), dtype=torch.bfloat16, pin_memory=True)
        outs.append(pipe.submit(host["q"], host["k"], host["v"], host, o))
    pipe.synchronize()
    assert pa.device_error() == 0
    for i, o in enumerate(outs):
        inp, _ = sets[i % 3]
        _, _, ref = run_gpu(Workload(w.name, w.samples, w.heads, w.head_dim, 40 + i % 3), inp,
                            cuda_device)
        assert torch.equal(o.view(torch.int16), ref.cpu().view(torch.int16)), i
