"""The checked build (libmfattn_checked.so, -DMF_CHECKED) on the GPU.

Its kernels compare every global index they compute with the extent of its
buffer before the access and record MF_ERR_BOUNDS instead of making it. Run
on the edge-length packs (samples of 1, 31-33, 63, 95, 97, 127-129 and 257
tokens, warp and tile boundaries) and on random small packs, forward and
backward: no check may fire, and every output must be bit for bit the
product build's (the checks change no arithmetic). One test hands the
attention kernel a work item that names a sample past the end of the pack:
the check must catch it, and the context must stay usable.
"""
import numpy as np
import pytest
import torch

import packed_attention_b200 as pa
from packed_attention_b200 import _native
from packed_attention_b200.workloads import Workload, make_inputs, random_pack
from test_gpu_backward import SMALL as BWD_PACKS, dout_bits, run_fwd_bwd
from test_gpu_parity import SMALL_PACKS, run_gpu

pytestmark = pytest.mark.gpu

MF_ERR_BOUNDS = -8


def _random_packs():
    packs = []
    for trial in range(4):
        rng = np.random.default_rng(7100 + trial)
        samples = random_pack(rng, int(rng.integers(1, 7)), 200, 20, 2)
        packs.append(Workload(f"checked_random_{trial}", samples, heads=int(rng.integers(1, 4)),
                              head_dim=(64, 128)[trial % 2], seed=7200 + trial,
                              rope_frame_dims=(0, 0, 16, 8)[trial]))
    return packs


FWD_PACKS = [w for _, w in SMALL_PACKS] + _random_packs()


@pytest.mark.parametrize("w", FWD_PACKS, ids=lambda w: w.name)
def test_checked_forward_matches_product(cuda_device, w):
    inp = make_inputs(w)
    _, _, ref = run_gpu(w, inp, cuda_device)
    with _native.checked_build():
        _, _, got = run_gpu(w, inp, cuda_device)  # asserts no device error
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("w", BWD_PACKS + _random_packs()[:2], ids=lambda w: w.name)
def test_checked_backward_matches_product(cuda_device, w):
    inp = make_inputs(w)
    dob = dout_bits(w)
    _, _, out_r, lse_r, g_r = run_fwd_bwd(w, inp, dob, cuda_device)
    with _native.checked_build():
        _, _, out_c, lse_c, g_c = run_fwd_bwd(w, inp, dob, cuda_device)  # asserts no error
    assert torch.equal(out_c.view(torch.int16), out_r.view(torch.int16))
    assert torch.equal(lse_c, lse_r)
    for key in ("dq", "dk", "dv") + pa.GAMMA_NAMES:
        a, b = g_c[key], g_r[key]
        if a.dtype == torch.bfloat16:
            a, b = a.view(torch.int16), b.view(torch.int16)
        assert torch.equal(a, b), key


def test_checked_build_reports_a_bad_sample_index(cuda_device):
    """A work item whose sample index is one past the pack's last sample:
    the checked kernel records MF_ERR_BOUNDS, reads sample 0 in its place
    (every role of the kernel does the same, so its pipeline stays in step)
    and touches nothing outside its buffers; the next call runs clean."""
    w = Workload("checked_bad_seg", ((10, 6, 6, 1), (4, 5, 7, 1)), heads=2, head_dim=128, seed=7300)
    inp = make_inputs(w)
    from test_gpu_parity import to_dev
    t = to_dev(inp, cuda_device)
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, device=cuda_device, ctas=0)
    work = plan.work.clone()
    assert int(work[0, 2]) == 0  # q_tile 0 exists in every sample
    work[0, 0] = len(w.samples)
    with _native.checked_build():
        ws = plan.new_workspace()
        out = torch.empty_like(t["q"])
        pa.qk_prologue(t["q"], t["k"], t, plan, ws, eps=w.eps)
        L = _native.lib()
        st = torch.cuda.current_stream()
        import ctypes
        P = ctypes.c_void_p
        rc = L.mf_packed_attention(P(t["v"].data_ptr()), P(plan.segs.data_ptr()), len(w.samples),
                                   P(work.data_ptr()), work.shape[0], w.total_tokens, w.heads,
                                   w.head_dim, 0.0, P(out.data_ptr()), P(ws.data_ptr()),
                                   ws.numel(), P(st.cuda_stream))
        assert rc == 0
        assert pa.device_error() == MF_ERR_BOUNDS
        assert pa.device_error() == 0  # read and cleared
        _, _, again = run_gpu(w, inp, cuda_device)
    _, _, ref = run_gpu(w, inp, cuda_device)
    assert torch.equal(again.view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("cfg", (1, 2, 3, 4))
def test_checked_forward_full_size(cuda_device, cfg):
    """The checked build on the full-size configs (every global index of the
    prologue and the attention kernel compared with its buffer's extent at
    the real sizes): no check fires, and the output is bit for bit the
    product build's."""
    from packed_attention_b200.workloads import WORKLOADS
    w = WORKLOADS[cfg]
    inp = make_inputs(w)
    _, _, ref = run_gpu(w, inp, cuda_device)
    with _native.checked_build():
        _, _, got = run_gpu(w, inp, cuda_device)  # asserts no device error
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_checked_backward_full_size(cuda_device):
    """The checked build's backward on the full-size 1024² editing pack: no
    check fires, and every gradient is bit for bit the product build's."""
    from packed_attention_b200.workloads import WORKLOADS
    w = WORKLOADS[3]
    inp = make_inputs(w)
    dob = dout_bits(w)
    _, _, out_r, lse_r, g_r = run_fwd_bwd(w, inp, dob, cuda_device)
    with _native.checked_build():
        _, _, out_c, lse_c, g_c = run_fwd_bwd(w, inp, dob, cuda_device)  # asserts no error
    assert torch.equal(out_c.view(torch.int16), out_r.view(torch.int16))
    assert torch.equal(lse_c, lse_r)
    for key in ("dq", "dk", "dv") + pa.GAMMA_NAMES:
        a, b = g_c[key], g_r[key]
        if a.dtype == torch.bfloat16:
            a, b = a.view(torch.int16), b.view(torch.int16)
        assert torch.equal(a, b), key
