"""sla_forward_noalloc: the forward for callers that cannot allocate device
memory (for example a plugin inside a host program that owns the whole GPU
memory pool, or a loop that must never call cudaMalloc). It takes its scratch
from the library's static device array instead of a caller workspace.

Checked through the C ABI against sla_forward (caller-allocated workspace) on
two calls in a row with different shapes and variants, so the second call runs
on the array the first one left behind. This file is collected last so that a
run stopping at the first failure has already run every other test."""

import ctypes

import numpy as np
import pytest

import workloads as W
from tests.gpu_helpers import assert_close, device_inputs, from_dev_bf16, run_library


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
    torch.cuda.synchronize()
    return from_dev_bf16(out)


@pytest.mark.gpu
def test_noalloc_matches_sla_forward_on_two_calls_in_a_row(cuda_lib):
    cases = [
        W.make_workload("noalloc_sla", 1, 4, 64 * 40 + 17, 128, "sla", k_crit=3, k_neg=5, seed=21),
        W.make_workload("noalloc_sla2", 2, 2, 64 * 23 + 50, 64, "sla2", k_crit=2, k_neg=0, seed=22),
    ]
    for w in cases:
        inp = W.make_inputs(w)
        dev = device_inputs(inp)
        ref = run_library(cuda_lib, inp, dev=dev)["O"][:, :, :w.N]
        got = _noalloc(cuda_lib, inp, dev)[:, :, :w.N]
        assert_close(got, ref, what=f"noalloc vs sla_forward ({w.name})")


@pytest.mark.gpu
def test_noalloc_rejects_problems_above_the_static_size(cuda_lib):
    w = W.WORKLOADS["sla_wan13b_b1h12n32768d128_s95"]
    p = cuda_lib.make_params(w.B, w.H, w.N, w.d, variant="sla", k_crit=w.k_crit, k_neg=w.k_neg)
    assert cuda_lib.workspace_size(p) > cuda_lib.NOALLOC_WORKSPACE_BYTES
    # rejected on the host before anything is enqueued (the tensor pointers are never touched)
    st = cuda_lib.load().sla_forward_noalloc(0x10000, 0x20000, 0x30000, 0x40000, ctypes.byref(p),
                                             None)
    assert st == cuda_lib.SLA_ERR_WORKSPACE
