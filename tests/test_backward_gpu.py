"""GPU parity of the backward pass (sla_forward_train + sla_backward) against
the float64 oracle's backward_head, with the mask of the forward held fixed.

The sparse path is the softmax-attention backward on the critical pairs; the
linear path is the chain rule through num / den, H_i, Z_i and phi (SLA
walkthrough, section 2.3). The library keeps bf16 operands for every tensor
core product (Q, K, V, dO, P, dS, dnum, phi, H_i, A_j) with fp32 accumulation
and returns bf16 gradients, so each gradient carries bf16 rounding of its
operands: a relative error of about 2^-9 per operand, averaging down over
the sums: measured rel-L2 4e-3 to 7.4e-3 and max-abs 5e-3 to 7.7e-3 of the
tensor's largest entry over the cases below, the 32k-token workloads
included. The tolerances (rel-L2 GRAD_REL_L2, max-abs against the tensor's
own largest entry GRAD_MAX_REL) sit at about twice that. dW and dalpha are
checked as exact reductions of the saved activations, and against the oracle
(check_param_grad).

The saved activations are checked too: O^s and O^l within the bf16 output
contract, lse within LSE_ABS (fp32 log2 arithmetic), den within DEN_REL (phi
rounded to bf16 before the dot with Z_i, as in the forward).
"""

import numpy as np
import pytest

import workloads as W
from tests.gpu_helpers import MAX_ABS, REL_L2, assert_close, device_inputs, from_dev_bf16, to_dev

pytestmark = pytest.mark.gpu

GRAD_REL_L2 = 1.5e-2
GRAD_MAX_REL = 1.5e-2
DW_REL = 1e-2
PARAM_REL = 5e-2   # dalpha against the oracle (a cancelling sum; see check_param_grad)
REDUCE_REL = 1e-5  # the library's float32 reductions against float64 on the same saved values
LSE_ABS = 2e-3
DEN_REL = 1e-2


def rel_l2(got, want):
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))


def check_grad(got, want, what, record=None):
    r = rel_l2(got, want)
    m = float(np.abs(got - want).max() / max(np.abs(want).max(), 1e-30))
    if record is not None:
        record(f"{what}_rel_l2", r)
        record(f"{what}_max_rel", m)
    assert r <= GRAD_REL_L2, f"{what}: rel-L2 {r:.3e}"
    assert m <= GRAD_MAX_REL, f"{what}: max-abs / max {m:.3e}"


def run_train(sla, inp, dO_bits, use_w=True):
    import torch

    w = inp.w
    dev = device_inputs(inp)
    B, H = inp.q.shape[:2]
    p = sla.make_params(B, H, w.N, w.d, variant=w.variant, k_crit=w.k_crit, k_neg=w.k_neg, phi=w.phi,
                        w_proj=dev["w_proj"] if use_w else None, proj_q=dev["proj_q"], proj_k=dev["proj_k"],
                        alpha=dev["alpha"])
    do = to_dev(dO_bits)
    O, saved, fws = sla.forward_train(dev["q"], dev["k"], dev["v"], params=p)
    dq, dk, dv, pg, bws = sla.backward(dev["q"], dev["k"], dev["v"], do, params=p, saved=saved, fwd_workspace=fws)
    torch.cuda.synchronize()
    return dict(dev=dev, p=p, do=do, O=O, saved=saved, fws=fws, bws=bws, dq=dq, dk=dk, dv=dv, pg=pg)


def oracle_bwd(inp, idx, dO_bits, use_w=True):
    from oracle import sla_oracle as O

    w = inp.w
    b, h = inp.heads[idx]
    sel = (b, h)
    do = W.bf16_bits_to_f32(dO_bits[sel]).astype(np.float64)
    return O.backward_head(inp.q[sel], inp.k[sel], inp.v[sel], do, w.N, variant=w.variant, k_crit=w.k_crit,
                           k_neg=w.k_neg, w_proj_bits=inp.w_proj if use_w else None, proj_q_bits=inp.proj_q,
                           proj_k_bits=inp.proj_k, alpha_h=None if inp.alpha is None else float(inp.alpha[h]),
                           phi_kind=w.phi)


def check_head(res, inp, idx, dO_bits, use_w=True, record=None):
    w = inp.w
    N = w.N
    b, h = inp.heads[idx]
    r = oracle_bwd(inp, idx, dO_bits, use_w)
    sv = res["saved"]
    assert_close(from_dev_bf16(sv["o_s"])[b, h][:N], r["O_s"], MAX_ABS, REL_L2, what=f"O^s head {idx}")
    assert_close(from_dev_bf16(sv["o_l"])[b, h][:N], r["O_l"], MAX_ABS, REL_L2, what=f"O^l head {idx}")
    lse = sv["lse"].cpu().numpy()[b, h][:N].astype(np.float64)
    np.testing.assert_allclose(lse, r["lse"], rtol=0, atol=LSE_ABS, err_msg=f"lse head {idx}")
    den = sv["den"].cpu().numpy()[b, h][:N].astype(np.float64)
    np.testing.assert_allclose(den, r["den"], rtol=DEN_REL, atol=1e-30, err_msg=f"den head {idx}")
    for name, key in (("dQ", "dq"), ("dK", "dk"), ("dV", "dv")):
        g = from_dev_bf16(res[key])[b, h]
        check_grad(g[:N], r[name], f"{name}_head{idx}", record)
        assert np.all(g[N:] == 0.0), f"{name} head {idx}: rows past N not zero"
    return r


CASES = [
    # name, B, H, N, d, variant, k_crit, k_neg, phi, use_w
    ("bw_sla_ragged", 1, 2, 64 * 12 + 13, 128, "sla", 3, 2, "softmax", True),
    ("bw_sla2_ragged", 1, 2, 64 * 12 + 13, 128, "sla2", 2, 0, "softmax", True),
    ("bw_sla_d64_many_tiles", 2, 1, 64 * 37 + 63, 64, "sla", 5, 7, "softmax", True),
    ("bw_sla2_elu1", 1, 2, 64 * 10 + 1, 128, "sla2", 2, 0, "elu1", True),
    ("bw_sla_elu1_d64", 1, 2, 64 * 9, 64, "sla", 2, 3, "elu1", True),
    ("bw_all_critical", 1, 2, 64 * 5 + 7, 128, "sla", 6, 0, "softmax", True),
    ("bw_sla_no_w", 1, 1, 64 * 8 + 40, 128, "sla", 2, 1, "softmax", False),
    ("bw_one_partial_block", 1, 2, 37, 64, "sla2", 1, 0, "softmax", True),
    ("bw_sla2_batch2_heads3", 2, 3, 64 * 7 + 21, 128, "sla2", 2, 0, "softmax", True),
    ("bw_sla2_with_negligible", 1, 2, 64 * 10, 128, "sla2", 2, 3, "softmax", True),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_backward_small(cuda_lib, case, record_property):
    name, B, H, N, d, variant, kc, kn, phi, use_w = case
    w = W.make_workload(name, B, H, N, d, variant, k_crit=kc, k_neg=kn, seed=51, phi=phi)
    inp = W.make_inputs(w)
    dO_bits = W.grad_output(w)
    res = run_train(cuda_lib, inp, dO_bits, use_w)
    assert cuda_lib.read_device_status(res["fws"]) == 0
    per_head = [check_head(res, inp, idx, dO_bits, use_w, record_property) for idx in range(B * H)]
    check_param_grad(res, inp, dO_bits, per_head)


def check_param_grad(res, inp, dO_bits, per_head):
    """dW (SLA) and dalpha (SLA2) are sums over every row of products of the
    saved bf16 activations with dO. They are checked as the exact reductions
    of what the training forward saved (float64 here against the library's
    float32 sums: REDUCE_REL of the sum of the terms' magnitudes), the saved
    activations themselves having been checked against the oracle. dalpha
    cancels (random-sign dO), so the activations' bf16-level errors reach it
    at about 1 % relative; it is held to PARAM_REL against the oracle. dW does
    not cancel that way and stays within DW_REL."""
    w = inp.w
    N = w.N
    got = res["pg"].cpu().numpy().astype(np.float64)
    Os = from_dev_bf16(res["saved"]["o_s"])[:, :, :N]
    Ol = from_dev_bf16(res["saved"]["o_l"])[:, :, :N]
    dO = W.bf16_bits_to_f32(dO_bits[:, :, :N]).astype(np.float64)
    if w.variant == "sla":
        exact = np.einsum("bhnc,bhne->ce", Ol, dO)
        scale = np.einsum("bhnc,bhne->ce", np.abs(Ol), np.abs(dO))
        assert np.all(np.abs(got - exact) <= REDUCE_REL * scale + 1e-6), "dW is not the reduction of O^l^T dO"
        dW = sum(r["dW"] for r in per_head)
        assert rel_l2(got, dW) <= DW_REL, f"dW rel-L2 {rel_l2(got, dW):.3e}"
    else:
        terms = dO * (Os - Ol)
        exact = terms.sum(axis=(0, 2, 3))
        scale = np.abs(terms).sum(axis=(0, 2, 3))
        assert np.all(np.abs(got - exact) <= REDUCE_REL * scale + 1e-6), (got, exact)
        for h in range(w.H):
            want = sum(pr["dalpha"] for j, pr in enumerate(per_head) if inp.heads[j][1] == h)
            assert got[h] == pytest.approx(want, rel=PARAM_REL, abs=1e-3), f"dalpha head {h}"


def test_training_forward_output_and_determinism(cuda_lib):
    """The training forward's O is the plain forward's, bit for bit, and two
    backward runs give bitwise identical gradients; NaN in dO's pad rows stays out."""
    import torch

    w = W.make_workload("bw_det", 1, 2, 64 * 11 + 9, 128, "sla", k_crit=3, k_neg=2, seed=52)
    inp = W.make_inputs(w)
    dO_bits = W.grad_output(w)
    dO_bits[:, :, w.N:] = 0x7FC0  # NaN pad rows
    res = run_train(cuda_lib, inp, dO_bits)
    dev, p = res["dev"], res["p"]
    O2, _ = cuda_lib.forward(dev["q"], dev["k"], dev["v"], params=p)
    assert torch.equal(res["O"].view(torch.int16)[:, :, :w.N], O2.view(torch.int16)[:, :, :w.N])
    again = cuda_lib.backward(dev["q"], dev["k"], dev["v"], res["do"], params=p, saved=res["saved"],
                              fwd_workspace=res["fws"])
    torch.cuda.synchronize()
    for a, b in ((res["dq"], again[0]), (res["dk"], again[1]), (res["dv"], again[2]), (res["pg"], again[3])):
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                           b.view(torch.int16) if b.dtype == torch.bfloat16 else b)
    for t in (res["dq"], res["dk"], res["dv"], res["pg"]):
        assert torch.isfinite(t.float()).all()
    check_head(res, inp, 0, dO_bits)


@pytest.mark.parametrize("name", ["sla_wan13b_b1h12n32768d128_s95", "sla2_b1h12n32768d128_s97"])
def test_backward_full_size(cuda_lib, name, record_property):
    """The 32k-token, 12-head workloads: gradients of one head against the oracle."""
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w)
    dO_bits = W.grad_output(w)
    res = run_train(cuda_lib, inp, dO_bits)
    assert cuda_lib.read_device_status(res["fws"]) == 0
    check_head(res, inp, 5, dO_bits, record=record_property)


def test_autograd_function_matches_sla_backward(cuda_lib):
    """attention() through torch.autograd gives sla_backward's gradients, bit for bit."""
    import torch

    w = W.make_workload("bw_autograd", 1, 2, 64 * 6 + 9, 64, "sla2", k_crit=2, k_neg=0, seed=53)
    inp = W.make_inputs(w)
    dO_bits = W.grad_output(w)
    res = run_train(cuda_lib, inp, dO_bits)
    dev = res["dev"]
    q, k, v = (dev[x].clone().requires_grad_(True) for x in ("q", "k", "v"))
    alpha = dev["alpha"].clone().requires_grad_(True)
    o = cuda_lib.attention(q, k, v, N=w.N, variant="sla2", k_crit=w.k_crit, alpha=alpha,
                           proj_q=dev["proj_q"], proj_k=dev["proj_k"])
    assert torch.equal(o.view(torch.int16)[:, :, :w.N], res["O"].view(torch.int16)[:, :, :w.N])
    o.backward(res["do"])
    torch.cuda.synchronize()
    for t, ref in ((q, res["dq"]), (k, res["dk"]), (v, res["dv"])):
        assert torch.equal(t.grad.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(alpha.grad, res["pg"])
