"""Failure detection on the GPU without a fault: a bounded in-kernel wait is
made to expire on purpose (sla_check_wait_timeout waits on an mbarrier that
nothing arrives on, with a short limit and no copy or tensor-core product in
flight). The kernel must give up, record the timeout in the workspace's status
word and return, so that sla_read_device_status reports
SLA_ERR_DEVICE_TIMEOUT and the context stays usable: the next forward on the
same workspace clears the word and still matches the oracle."""

import pytest

import workloads as W
from tests.gpu_helpers import assert_close, device_inputs, oracle_head

pytestmark = pytest.mark.gpu


def test_expired_wait_reports_timeout_and_context_stays_usable(cuda_lib):
    import torch

    sla = cuda_lib
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert sla.read_device_status(ws) == sla.SLA_OK
    assert sla.check_wait_timeout(ws, 100_000) == sla.SLA_OK
    assert sla.read_device_status(ws) == sla.SLA_ERR_DEVICE_TIMEOUT
    torch.cuda.synchronize()  # no CUDA error is pending

    # a forward workspace: the self-test marks it, the next forward clears it
    w = W.make_workload("after_timeout", 1, 2, 64 * 9 + 21, 128, "sla2", k_crit=2, k_neg=0, seed=41)
    inp = W.make_inputs(w)
    dev = device_inputs(inp)
    p = sla.make_params(w.B, w.H, w.N, w.d, variant="sla2", k_crit=w.k_crit, proj_q=dev["proj_q"],
                        proj_k=dev["proj_k"], alpha=dev["alpha"])
    fws = sla.allocate_workspace(p)
    assert sla.check_wait_timeout(fws, 50_000) == sla.SLA_OK
    assert sla.read_device_status(fws) == sla.SLA_ERR_DEVICE_TIMEOUT
    out, _ = sla.forward(dev["q"], dev["k"], dev["v"], workspace=fws, params=p)
    assert sla.read_device_status(fws) == sla.SLA_OK
    from tests.gpu_helpers import from_dev_bf16

    got = from_dev_bf16(out)
    for idx in range(len(inp.heads)):
        ref = oracle_head(inp, idx)
        assert_close(got[0, idx, :w.N], ref["O"], what=f"forward after an expired wait, head {idx}")


def test_wait_limit_is_checked_on_the_host(cuda_lib):
    import torch

    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert cuda_lib.check_wait_timeout(ws, 0) == cuda_lib.SLA_ERR_INVALID_ARG
    assert cuda_lib.check_wait_timeout(ws, 4_000_000_001) == cuda_lib.SLA_ERR_INVALID_ARG
    assert cuda_lib.read_device_status(ws) == cuda_lib.SLA_OK  # nothing was enqueued
