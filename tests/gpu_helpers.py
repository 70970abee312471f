"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
library through its C ABI, and compare with the oracle."""

import math

import numpy as np

import workloads as W

# bf16 output contract (unrounded float64 oracle output as the reference)
MAX_ABS = 2e-2
REL_L2 = 1e-2


def to_dev(bits):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def from_dev_bf16(t):
    import torch

    u = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return W.bf16_bits_to_f32(u).astype(np.float64)


def device_inputs(inp):
    import torch

    d = dict(q=to_dev(inp.q), k=to_dev(inp.k), v=to_dev(inp.v))
    d["w_proj"] = to_dev(inp.w_proj) if inp.w_proj is not None else None
    d["proj_q"] = to_dev(inp.proj_q) if inp.proj_q is not None else None
    d["proj_k"] = to_dev(inp.proj_k) if inp.proj_k is not None else None
    d["alpha"] = torch.from_numpy(inp.alpha).cuda() if inp.alpha is not None else None
    return d


def run_library(sla, inp, dev=None, use_w=True, use_router=True, out_fill=None, ws_fill=None):
    """sla_forward on a workloads.Inputs, in the workload's precision. Returns
    dict with O (float64 numpy, [B,H,N_pad,d]), Mc, crit, neg (numpy), the
    params and the raw tensors."""
    import torch

    w = inp.w
    dev = dev or device_inputs(inp)
    B, H = inp.q.shape[:2]
    p = sla.make_params(B, H, w.N, w.d, variant=w.variant, precision=w.precision, k_crit=w.k_crit,
                        k_neg=w.k_neg, phi=w.phi, w_proj=dev["w_proj"] if use_w else None,
                        proj_q=dev["proj_q"] if use_router else None,
                        proj_k=dev["proj_k"] if use_router else None, alpha=dev["alpha"])
    out = torch.empty_like(dev["q"])
    if out_fill is not None:
        out.view(torch.int16).fill_(out_fill)
    ws = sla.allocate_workspace(p)
    if ws_fill is not None:
        ws.fill_(ws_fill)
    sla.forward(dev["q"], dev["k"], dev["v"], out=out, workspace=ws, params=p)
    mc, crit, neg = sla.get_mask(p, ws)
    st = sla.read_device_status(ws)
    torch.cuda.synchronize()
    return dict(O=from_dev_bf16(out), O_raw=out, Mc=mc.cpu().numpy(), crit=crit.cpu().numpy(),
                neg=neg.cpu().numpy(), params=p, ws=ws, status=st, dev=dev)


def oracle_head(inp, idx, use_w=True, use_router=True, quantized=False):
    """Oracle for entry idx (b, h) of inp.heads (with quantized=True also the
    emulated low-bit sparse branch, O_sq, and the output built from it, O_q)."""
    from oracle import sla_oracle as O

    w = inp.w
    b, h = inp.heads[idx]
    full = inp.q.shape[:2] == (w.B, w.H) and len(inp.heads) == w.B * w.H
    sel = (b, h) if full else (idx, 0)
    return O.forward_head(
        inp.q[sel], inp.k[sel], inp.v[sel], w.N, variant=w.variant, k_crit=w.k_crit, k_neg=w.k_neg,
        w_proj_bits=inp.w_proj if use_w else None,
        proj_q_bits=inp.proj_q if use_router else None,
        proj_k_bits=inp.proj_k if use_router else None,
        alpha_h=None if inp.alpha is None else float(inp.alpha[h]), quantized=quantized,
        phi_kind=w.phi)


def oracle_mask_only(inp, idx, use_router=True):
    from oracle import sla_oracle as O

    w = inp.w
    b, h = inp.heads[idx]
    full = inp.q.shape[:2] == (w.B, w.H) and len(inp.heads) == w.B * w.H
    sel = (b, h) if full else (idx, 0)
    pq = O.bf16_to_f32(inp.proj_q) if (use_router and inp.proj_q is not None) else None
    pk = O.bf16_to_f32(inp.proj_k) if (use_router and inp.proj_k is not None) else None
    return O.mask_f32_spec(O.bf16_to_f32(inp.q[sel]), O.bf16_to_f32(inp.k[sel]), w.N, w.k_crit,
                           w.k_neg, pq, pk)


def errors(got, want):
    e = got - want
    return float(np.abs(e).max()), float(np.linalg.norm(e) / max(np.linalg.norm(want), 1e-30))


def assert_close(got, want, max_abs=MAX_ABS, rel_l2=REL_L2, what=""):
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    ma, rl = errors(got, want)
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max-abs {ma:.3e} (<= {max_abs}), rel-L2 {rl:.3e} (<= {rel_l2})"
    return ma, rl
