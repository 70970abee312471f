"""GPU parity of the SoftTop-k router forward (sla_router_soft_topk) against the
oracle's soft_topk on the same float32 pooled scores.

SoftTop-k (SLA2 article, two-stage training paragraphs; SLA2 L3 synthesis,
section 3): M_ij = sigmoid((Pc_ij - lambda_i) / tau) with lambda_i per row by
bisection so that sum_j M_ij = k_crit. The scores s_ij are bit-identical on
both sides (the mask-stage float32 specification); the oracle then takes Pc
and lambda in float64, the kernel in float32.

Tolerances, from the float32 arithmetic:
  * Pc: relative 2e-5 (2^x on the MUFU unit and one division per entry).
  * M: absolute 1e-4. An error e in the float32 row-sum residual moves each
    M_ij by at most e (dM_j = sigma_j (1 - sigma_j) dlambda / tau and
    dlambda = e tau / sum_j sigma_j (1 - sigma_j)); e is a few 1e-6 per row here.
    An error in Pc moves the sigmoid argument by dPc / tau, at most 1e-6 at
    the temperatures used.
  * lambda, where the row fixes it weakly (saturated sigmoids), is checked
    through its residual: the float64 row sum at the kernel's lambda is within
    1e-3 of k_crit.
"""

import numpy as np
import pytest

import workloads as W
from tests.gpu_helpers import device_inputs

pytestmark = pytest.mark.gpu

PC_RTOL = 2e-5
M_ATOL = 1e-4
SUM_TOL = 1e-3


def residual_f64(pc, lam, tau, k):
    """sum_j sigmoid((pc_j - lam) / tau) - k in float64, from the sigmoid tails."""
    x = (pc - lam[:, None]) / tau
    e = np.exp(-np.abs(x))
    t = e / (1.0 + e)
    pos = x > 0
    return (pos.sum(axis=1) - k) + np.where(pos, -t, t).sum(axis=1)


def run_router(sla, inp, tau, use_router=True):
    import torch

    w = inp.w
    dev = device_inputs(inp)
    B, H = inp.q.shape[:2]
    p = sla.make_params(B, H, w.N, w.d, variant=w.variant, k_crit=w.k_crit, k_neg=w.k_neg,
                        proj_q=dev["proj_q"] if use_router else None,
                        proj_k=dev["proj_k"] if use_router else None, alpha=dev["alpha"])
    m, lam, pc, ws = sla.router_soft_topk(dev["q"], dev["k"], tau=tau, params=p, want_pc=True)
    torch.cuda.synchronize()
    return m.cpu().numpy().astype(np.float64), lam.cpu().numpy().astype(np.float64), \
        pc.cpu().numpy().astype(np.float64)


def check_head(inp, idx, tau, M, lam, Pc, use_router=True):
    from oracle import sla_oracle as O

    w = inp.w
    b, h = inp.heads[idx]
    full = len(inp.heads) == w.B * w.H
    sel = (b, h) if full else (idx, 0)
    r = O.router_soft_topk_head(inp.q[sel], inp.k[sel], w.N, w.k_crit, tau,
                                inp.proj_q if use_router else None, inp.proj_k if use_router else None)
    np.testing.assert_allclose(Pc[sel], r["Pc"], rtol=PC_RTOL, atol=1e-30, err_msg=f"Pc head {idx}")
    np.testing.assert_allclose(M[sel], r["M"], rtol=0, atol=M_ATOL, err_msg=f"M head {idx}")
    np.testing.assert_allclose(M[sel].sum(axis=1), w.k_crit, rtol=0, atol=SUM_TOL)
    Nb = w.Nb
    if w.k_crit == Nb:
        assert np.all(np.isneginf(lam[sel])) and np.all(M[sel] == 1.0)
        return
    res = residual_f64(r["Pc"], lam[sel], tau, w.k_crit)
    assert np.abs(res).max() <= SUM_TOL, f"head {idx}: row-sum residual {np.abs(res).max():.3e} at the kernel's lambda"


CASES = [
    # name, B, H, N, d, variant, k_crit, tau
    ("sla2_router_ragged", 1, 2, 64 * 12 + 13, 128, "sla2", 2, 0.05),
    ("sla2_router_cold", 1, 2, 64 * 12 + 13, 128, "sla2", 3, 1e-3),
    ("sla_d64_no_proj", 2, 1, 64 * 20, 64, "sla", 4, 0.01),
    ("one_block_all_selected", 1, 2, 37, 128, "sla2", 1, 0.1),
    ("all_but_one_selected", 1, 1, 64 * 9, 64, "sla", 8, 0.02),
    ("many_tiles_hot", 1, 3, 64 * 300 + 5, 128, "sla2", 9, 0.5),
    ("nb1500_vpl64", 1, 1, 64 * 1500, 64, "sla", 45, 1e-3),
    ("nb2100_vpl128", 1, 1, 64 * 2100 - 20, 64, "sla", 63, 1e-3),
    ("sla2_batch2_heads3", 2, 3, 64 * 9 + 5, 128, "sla2", 3, 0.02),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_soft_topk_small(cuda_lib, case):
    name, B, H, N, d, variant, kc, tau = case
    w = W.make_workload(name, B, H, N, d, variant, k_crit=kc, k_neg=0, seed=41)
    inp = W.make_inputs(w)
    M, lam, Pc = run_router(cuda_lib, inp, tau)
    for idx in range(B * H):
        check_head(inp, idx, tau, M, lam, Pc)


def test_soft_topk_full_size_sla2_32k(cuda_lib):
    """The SLA2 32k-token, 12-head workload (k_crit = 15 of 512 blocks), two
    temperatures; the oracle checks two heads, every row."""
    w = W.WORKLOADS["sla2_b1h12n32768d128_s97"]
    inp = W.make_inputs(w)
    for tau in (1e-2, 1e-4):
        M, lam, Pc = run_router(cuda_lib, inp, tau)
        assert np.isfinite(M).all() and np.isfinite(lam).all()
        np.testing.assert_allclose(M.sum(axis=-1), w.k_crit, rtol=0, atol=SUM_TOL)
        for idx in (0, 7):
            check_head(inp, idx, tau, M, lam, Pc)


def test_soft_topk_rejects_bad_temperature(cuda_lib):
    import torch

    w = W.make_workload("bad_tau", 1, 1, 256, 64, "sla", k_crit=1, k_neg=0, seed=1)
    dev = device_inputs(W.make_inputs(w))
    p = cuda_lib.make_params(1, 1, w.N, w.d, variant="sla", k_crit=1)
    for tau in (0.0, -1.0, float("inf"), float("nan"), 1e-45):
        with pytest.raises(cuda_lib.SLAError) as e:
            cuda_lib.router_soft_topk(dev["q"], dev["k"], tau=tau, params=p)
        assert e.value.status == cuda_lib.SLA_ERR_INVALID_ARG
    torch.cuda.synchronize()
