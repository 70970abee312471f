"""sla_forward_noalloc: the forward for callers that cannot allocate device
memory (for example a plugin inside a host program that owns the whole GPU
memory pool, or a loop that must never call cudaMalloc). It takes its scratch
from the library's static device array instead of a caller workspace.

Checked through the C ABI against sla_forward (caller-allocated workspace) on
two calls in a row with different shapes and variants, so the second call runs
on the array the first one left behind. Both paths run the same deterministic
kernels on the same inputs, so their outputs must agree bit for bit; the first
case is also held to the float64 oracle at the bf16 contract, and the array's
status word (read with a NULL workspace) must be clear after each call. This
file is collected last so that a run stopping at the first failure has already
run every other test."""

import ctypes

import pytest

import workloads as W
from tests.gpu_helpers import assert_close, device_inputs, from_dev_bf16, oracle_head


def _noalloc(sla, inp, dev):
    import torch

    w = inp.w
    p = sla.make_params(w.B, w.H, w.N, w.d, variant=w.variant, k_crit=w.k_crit, k_neg=w.k_neg,
                        w_proj=dev["w_proj"], proj_q=dev["proj_q"], proj_k=dev["proj_k"],
                        alpha=dev["alpha"])
    assert sla.workspace_size(p) <= sla.NOALLOC_WORKSPACE_BYTES
    out = torch.zeros_like(dev["q"])
    st = sla.load().sla_forward_noalloc(dev["q"].data_ptr(), dev["k"].data_ptr(),
                                        dev["v"].data_ptr(), out.data_ptr(), ctypes.byref(p),
                                        torch.cuda.current_stream().cuda_stream)
    assert st == sla.SLA_OK, sla.status_string(st)
    assert sla.read_device_status(None) == sla.SLA_OK  # the static array's status word
    torch.cuda.synchronize()
    return out


def _with_workspace(sla, inp, dev):
    import torch

    w = inp.w
    p = sla.make_params(w.B, w.H, w.N, w.d, variant=w.variant, k_crit=w.k_crit, k_neg=w.k_neg,
                        w_proj=dev["w_proj"], proj_q=dev["proj_q"], proj_k=dev["proj_k"],
                        alpha=dev["alpha"])
    out = torch.zeros_like(dev["q"])
    ws = sla.allocate_workspace(p)
    sla.forward(dev["q"], dev["k"], dev["v"], out=out, workspace=ws, params=p)
    assert sla.read_device_status(ws) == sla.SLA_OK
    return out


@pytest.mark.gpu
def test_noalloc_matches_sla_forward_on_two_calls_in_a_row(cuda_lib):
    import torch

    cases = [
        W.make_workload("noalloc_sla", 1, 4, 64 * 40 + 17, 128, "sla", k_crit=3, k_neg=5, seed=21),
        W.make_workload("noalloc_sla2", 2, 2, 64 * 23 + 50, 64, "sla2", k_crit=2, k_neg=0, seed=22),
    ]
    for n, w in enumerate(cases):
        inp = W.make_inputs(w)
        dev = device_inputs(inp)
        ref = _with_workspace(cuda_lib, inp, dev)
        got = _noalloc(cuda_lib, inp, dev)
        N = w.N
        assert torch.equal(got[:, :, :N].view(torch.int16), ref[:, :, :N].view(torch.int16)), \
            f"noalloc differs from sla_forward ({w.name})"
        if n == 0:  # and the float64 oracle, at the bf16 contract
            o = from_dev_bf16(got)
            for idx, (b, h) in enumerate(inp.heads):
                assert_close(o[b, h, :N], oracle_head(inp, idx)["O"], what=f"noalloc vs oracle head {h}")


@pytest.mark.gpu
def test_noalloc_rejects_problems_above_the_static_size(cuda_lib):
    w = W.WORKLOADS["sla_wan13b_b1h12n32768d128_s95"]
    p = cuda_lib.make_params(w.B, w.H, w.N, w.d, variant="sla", k_crit=w.k_crit, k_neg=w.k_neg)
    assert cuda_lib.workspace_size(p) > cuda_lib.NOALLOC_WORKSPACE_BYTES
    # rejected on the host before anything is enqueued (the tensor pointers are never touched)
    st = cuda_lib.load().sla_forward_noalloc(0x10000, 0x20000, 0x30000, 0x40000, ctypes.byref(p),
                                             None)
    assert st == cuda_lib.SLA_ERR_WORKSPACE
