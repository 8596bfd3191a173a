"""Failure detection on the GPU without a fault: a pipeline wait that runs out
of time must be reported through the device error word, and the context
must stay usable afterwards. The wait that runs out is the attention
kernel's own bounded wait, driven by a diagnostic kernel on an mbarrier that
nothing arrives on; nothing traps, faults or hangs."""
import ctypes

import numpy as np
import pytest
import torch

import packed_attention_b200 as pa
from packed_attention_b200 import _native
from packed_attention_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(cuda_device):
    lib = _native.lib()
    st = torch.cuda.current_stream()
    assert pa.device_error() == 0
    assert lib.mf_selftest_timeout(50_000_000, ctypes.c_void_p(st.cuda_stream)) == 0  # 50 ms
    assert pa.device_error(st) == -7          # MF_ERR_TIMEOUT, read and cleared
    assert pa.device_error(st) == 0           # cleared
    # the context is healthy: a forward still runs and matches itself
    w = WORKLOADS[0]
    inp = make_inputs(w)
    t = {n: torch.from_numpy(inp[n].view(np.int16)).view(torch.bfloat16).to(cuda_device)
         for n in ("q", "k", "v")}
    t.update({n: torch.from_numpy(inp[n]).to(cuda_device) for n in pa.GAMMA_NAMES})
    plan = pa.PackedPlan(w.samples, w.heads, w.head_dim, device=cuda_device)
    a = pa.joint_attention(t["q"], t["k"], t["v"], t, plan)
    b = pa.joint_attention(t["q"], t["k"], t["v"], t, plan)
    assert pa.device_error() == 0
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))

