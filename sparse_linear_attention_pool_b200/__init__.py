"""Python binding of the B200 SLA / SLA2 forward-pass library (libsla_b200.so).

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels. PyTorch supplies device memory and the stream. There is no CPU
fallback: if the compiled library is missing, load() raises.

    import sparse_linear_attention_pool_b200 as sla
    o = sla.forward(q, k, v, N=N, variant="sla2", k_crit=15, alpha=alpha,
                    proj_q=wq, proj_k=wk)

    # training: the forward that keeps its activations, then the gradients
    p = sla.make_params(B, H, N, d, variant="sla2", k_crit=15, alpha=alpha, proj_q=wq, proj_k=wk)
    o, saved, ws = sla.forward_train(q, k, v, params=p)
    dq, dk, dv, dalpha, _ = sla.backward(q, k, v, do, params=p, saved=saved, fwd_workspace=ws)

    # SLA2's SoftTop-k router (first training stage)
    m, lam, pc, _ = sla.router_soft_topk(q, k, tau=0.01, params=p, want_pc=True)

q, k, v: [B, H, N_pad, d] torch.bfloat16 CUDA tensors, N_pad = 64 * ceil(N / 64).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsla_b200.so")

SLA_OK, SLA_ERR_INVALID_ARG, SLA_ERR_UNSUPPORTED, SLA_ERR_WORKSPACE, SLA_ERR_ALIGNMENT, \
    SLA_ERR_CUDA, SLA_ERR_DEVICE_TIMEOUT, SLA_ERR_DEVICE_CHECK = range(8)
VARIANTS = {"sla": 0, "sla2": 1}
PRECISIONS = {"bf16": 0, "i8qk_f8pv": 1}
PHIS = {"softmax": 0, "elu1": 1}  # feature map of the linear branch
BLOCK = 64

# every symbol include/sla.h declares
EXPORTS = ("sla_abi_version", "sla_status_string", "sla_validate", "sla_workspace_size",
           "sla_forward", "sla_get_mask", "sla_get_pooled", "sla_read_device_status",
           "sla_dense_forward", "sla_stage_timing", "sla_stage_times", "sla_forward_noalloc",
           "sla_get_quantized", "sla_router_soft_topk", "sla_forward_train", "sla_backward_workspace_size",
           "sla_backward", "sla_check_wait_timeout")
NOALLOC_WORKSPACE_BYTES = 32 << 20
NUM_STAGES = 6
STAGES = ("pool", "phik_hz", "scores", "classify", "hz_reduce", "attention")


class Params(ctypes.Structure):
    """Mirror of struct sla_params."""
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int),
        ("block_q", ctypes.c_int), ("block_kv", ctypes.c_int),
        ("variant", ctypes.c_int), ("precision", ctypes.c_int),
        ("k_crit", ctypes.c_int), ("k_neg", ctypes.c_int),
        ("softmax_scale", ctypes.c_float),
        ("w_proj", ctypes.c_void_p), ("proj_q", ctypes.c_void_p), ("proj_k", ctypes.c_void_p),
        ("alpha", ctypes.c_void_p),
        ("phi", ctypes.c_int),
    ]


class Saved(ctypes.Structure):
    """Mirror of struct sla_saved (device pointers)."""
    _fields_ = [("o_s", ctypes.c_void_p), ("o_l", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("den", ctypes.c_void_p)]


class SLAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib: Optional[ctypes.CDLL] = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the compiled library (once). Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} not built; run python -m sparse_linear_attention_pool_b200.build")
    lib = ctypes.CDLL(path)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    P = ctypes.POINTER(Params)
    sig = {
        "sla_abi_version": (i, []),
        "sla_status_string": (ctypes.c_char_p, [i]),
        "sla_validate": (i, [P]),
        "sla_workspace_size": (sz, [P]),
        "sla_forward": (i, [vp, vp, vp, vp, P, vp, sz, vp]),
        "sla_get_mask": (i, [P, vp, vp, vp, vp, vp]),
        "sla_get_pooled": (i, [P, vp, vp, vp, vp]),
        "sla_read_device_status": (i, [vp, vp]),
        "sla_dense_forward": (i, [vp, vp, vp, vp, i, i, i, i, ctypes.c_float, vp]),
        "sla_forward_noalloc": (i, [vp, vp, vp, vp, P, vp]),
        "sla_get_quantized": (i, [P, vp, vp, vp, vp, vp, vp, vp, vp]),
        "sla_router_soft_topk": (i, [vp, vp, P, ctypes.c_float, vp, vp, vp, vp, sz, vp]),
        "sla_forward_train": (i, [vp, vp, vp, vp, P, ctypes.POINTER(Saved), vp, sz, vp]),
        "sla_backward_workspace_size": (sz, [P]),
        "sla_backward": (i, [vp, vp, vp, vp, P, ctypes.POINTER(Saved), vp, sz, vp, vp, vp, vp, vp, vp, sz, vp]),
        "sla_check_wait_timeout": (i, [vp, sz, ctypes.c_longlong, vp]),
        "sla_stage_timing": (i, [i]),
        "sla_stage_times": (i, [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().sla_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != SLA_OK:
        raise SLAError(status, what)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def make_params(B, H, N, d, *, variant="sla", precision="bf16", k_crit, k_neg=0,
                softmax_scale=0.0, w_proj=None, proj_q=None, proj_k=None, alpha=None,
                phi="softmax") -> Params:
    return Params(B=B, H=H, N=N, d=d, block_q=BLOCK, block_kv=BLOCK,
                  variant=VARIANTS[variant], precision=PRECISIONS[precision],
                  k_crit=int(k_crit), k_neg=int(k_neg), softmax_scale=float(softmax_scale),
                  w_proj=_ptr(w_proj), proj_q=_ptr(proj_q), proj_k=_ptr(proj_k), alpha=_ptr(alpha),
                  phi=PHIS[phi])


def validate(p: Params) -> int:
    return load().sla_validate(ctypes.byref(p))


def workspace_size(p: Params) -> int:
    n = load().sla_workspace_size(ctypes.byref(p))
    if n == 0:
        _check(validate(p), "sla_workspace_size")
    return n


def allocate_workspace(p: Params, device=None):
    """A uint8 CUDA tensor of sla_workspace_size bytes (torch allocations are 256-aligned)."""
    import torch

    return torch.empty(workspace_size(p), dtype=torch.uint8, device=device or "cuda")


def forward(q, k, v, *, N: Optional[int] = None, variant: str = "sla", precision: str = "bf16",
            k_crit: Optional[int] = None, k_neg: int = 0, softmax_scale: float = 0.0, w_proj=None,
            proj_q=None, proj_k=None, alpha=None, phi: str = "softmax", out=None, workspace=None,
            stream=None, params=None):
    """O = SLA / SLA2 forward of q, k, v ([B, H, N_pad, d] bf16 CUDA tensors).

    Returns (O, workspace); the workspace holds the mask and lists afterwards."""
    import torch

    B, H, Np, d = q.shape
    N = Np if N is None else int(N)
    if params is None and k_crit is None:
        raise ValueError("forward() needs k_crit or params")
    p = params or make_params(B, H, N, d, variant=variant, precision=precision, k_crit=k_crit,
                              k_neg=k_neg, softmax_scale=softmax_scale, w_proj=w_proj,
                              proj_q=proj_q, proj_k=proj_k, alpha=alpha, phi=phi)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = allocate_workspace(p, q.device)
    st = load().sla_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), ctypes.byref(p),
                            _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "sla_forward")
    return out, workspace


def get_mask(p: Params, workspace, stream=None):
    """(Mc [B,H,Nb,Nb] int8, crit [B,H,Nb,kc] int32, neg [B,H,Nb,kn] int32) on the device."""
    import torch

    Nb = (p.N + BLOCK - 1) // BLOCK
    dev = workspace.device
    mc = torch.empty((p.B, p.H, Nb, Nb), dtype=torch.int8, device=dev)
    crit = torch.empty((p.B, p.H, Nb, p.k_crit), dtype=torch.int32, device=dev)
    neg = torch.empty((p.B, p.H, Nb, p.k_neg), dtype=torch.int32, device=dev)
    st = load().sla_get_mask(ctypes.byref(p), _ptr(workspace), _ptr(mc), _ptr(crit),
                             _ptr(neg) if p.k_neg > 0 else None, _stream(stream))
    _check(st, "sla_get_mask")
    return mc, crit, neg


def get_pooled(p: Params, workspace, stream=None):
    """(qbar, kbar) [B,H,Nb,d] float32: the vectors the mask was ranked on."""
    import torch

    Nb = (p.N + BLOCK - 1) // BLOCK
    qb = torch.empty((p.B, p.H, Nb, p.d), dtype=torch.float32, device=workspace.device)
    kb = torch.empty_like(qb)
    _check(load().sla_get_pooled(ctypes.byref(p), _ptr(workspace), _ptr(qb), _ptr(kb),
                                 _stream(stream)), "sla_get_pooled")
    return qb, kb


def read_device_status(workspace, stream=None) -> int:
    """Status word of the last forward on `workspace` (None: the last
    sla_forward_noalloc on the current device); syncs the stream."""
    return load().sla_read_device_status(_ptr(workspace), _stream(stream))


def check_wait_timeout(workspace, limit_cycles: int, stream=None) -> int:
    """sla_check_wait_timeout: one bounded in-kernel wait that nothing ends,
    given up after limit_cycles; its status lands in the workspace's status word."""
    return load().sla_check_wait_timeout(_ptr(workspace), workspace.numel(), int(limit_cycles), _stream(stream))


def dense_forward(q, k, v, *, N: Optional[int] = None, softmax_scale: float = 0.0, out=None,
                  stream=None):
    """Dense softmax attention with the same kernel machinery (the baseline)."""
    import torch

    B, H, Np, d = q.shape
    N = Np if N is None else int(N)
    if out is None:
        out = torch.empty_like(q)
    st = load().sla_dense_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d,
                                  float(softmax_scale), _stream(stream))
    _check(st, "sla_dense_forward")
    return out


def stage_timing(max_calls: int):
    """Record per-stage CUDA events for up to max_calls sla_forward calls (0 stops)."""
    _check(load().sla_stage_timing(int(max_calls)), "sla_stage_timing")


def stage_times() -> tuple[dict, int]:
    """(summed ms per stage name, number of calls) since the last read."""
    ms = (ctypes.c_float * NUM_STAGES)()
    n = ctypes.c_int(0)
    _check(load().sla_stage_times(ms, ctypes.byref(n)), "sla_stage_times")
    return {name: float(ms[i]) for i, name in enumerate(STAGES)}, n.value


def forward_noalloc(q, k, v, *, params: Params, out=None, stream=None):
    """sla_forward_noalloc: the forward with the library's static scratch array
    instead of a caller-supplied workspace (for callers that cannot allocate).
    Calls on one device share that array: do not let their GPU work overlap."""
    import torch

    if out is None:
        out = torch.empty_like(q)
    st = load().sla_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), ctypes.byref(params),
                                    _stream(stream))
    _check(st, "sla_forward_noalloc")
    return out


def get_quantized(p: Params, workspace, stream=None):
    """Codes and scales of the quantised sparse branch, on the device:
    (qcode, kcode int8 [B,H,N_pad,d], vcode uint8 e4m3 bits [B,H,N_pad,d],
    qscale, kscale, vscale float32 [B,H,Nb])."""
    import torch

    Nb = (p.N + BLOCK - 1) // BLOCK
    dev = workspace.device
    shp = (p.B, p.H, Nb * BLOCK, p.d)
    qc = torch.empty(shp, dtype=torch.int8, device=dev)
    kc = torch.empty(shp, dtype=torch.int8, device=dev)
    vc = torch.empty(shp, dtype=torch.uint8, device=dev)
    qs, ks, vs = (torch.empty((p.B, p.H, Nb), dtype=torch.float32, device=dev) for _ in range(3))
    _check(load().sla_get_quantized(ctypes.byref(p), _ptr(workspace), _ptr(qc), _ptr(kc), _ptr(vc),
                                    _ptr(qs), _ptr(ks), _ptr(vs), _stream(stream)), "sla_get_quantized")
    return qc, kc, vc, qs, ks, vs


def router_soft_topk(q, k, *, tau: float, params: Params, workspace=None, want_pc: bool = False,
                     stream=None):
    """SoftTop-k router forward (sla_router_soft_topk): the pooled, router-projected
    scores, Pc = softmax(scale s) per row and M = sigmoid((Pc - lambda) / tau) with
    each row of M summing to params.k_crit.
    Returns (M [B,H,Nb,Nb] float32, lambda [B,H,Nb] float32, Pc or None, workspace)."""
    import torch

    Nb = (params.N + BLOCK - 1) // BLOCK
    dev = q.device
    m = torch.empty((params.B, params.H, Nb, Nb), dtype=torch.float32, device=dev)
    lam = torch.empty((params.B, params.H, Nb), dtype=torch.float32, device=dev)
    pc = torch.empty_like(m) if want_pc else None
    if workspace is None:
        workspace = allocate_workspace(params, dev)
    st = load().sla_router_soft_topk(_ptr(q), _ptr(k), ctypes.byref(params), float(tau), _ptr(m), _ptr(lam),
                                     _ptr(pc), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "sla_router_soft_topk")
    return m, lam, pc, workspace


def forward_train(q, k, v, *, params: Params, out=None, workspace=None, saved=None, stream=None):
    """sla_forward_train: the forward pass that also keeps what the backward reads.
    Returns (O, saved dict of tensors o_s, o_l, lse, den, workspace)."""
    import torch

    B, H, Np, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = allocate_workspace(params, q.device)
    if saved is None:
        saved = dict(o_s=torch.empty_like(q), o_l=torch.empty_like(q),
                     lse=torch.empty((B, H, Np), dtype=torch.float32, device=q.device),
                     den=torch.empty((B, H, Np), dtype=torch.float32, device=q.device))
    sv = Saved(o_s=_ptr(saved["o_s"]), o_l=_ptr(saved["o_l"]), lse=_ptr(saved["lse"]), den=_ptr(saved["den"]))
    st = load().sla_forward_train(_ptr(q), _ptr(k), _ptr(v), _ptr(out), ctypes.byref(params), ctypes.byref(sv),
                                  _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "sla_forward_train")
    return out, saved, workspace


def backward_workspace_size(p: Params) -> int:
    n = load().sla_backward_workspace_size(ctypes.byref(p))
    if n == 0:
        _check(validate(p), "sla_backward_workspace_size")
    return n


def backward(q, k, v, do, *, params: Params, saved: dict, fwd_workspace, want_param_grad: bool = True,
             workspace=None, stream=None):
    """sla_backward: gradients of <dO, O> for the forward of forward_train (mask fixed).
    Returns (dQ, dK, dV, dW or dalpha or None, workspace)."""
    import torch

    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    sla2 = params.variant == VARIANTS["sla2"]
    dW = dalpha = None
    if want_param_grad:
        if sla2:
            dalpha = torch.empty(params.H, dtype=torch.float32, device=q.device)
        else:
            dW = torch.empty((params.d, params.d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(backward_workspace_size(params), dtype=torch.uint8, device=q.device)
    sv = Saved(o_s=_ptr(saved["o_s"]), o_l=_ptr(saved["o_l"]), lse=_ptr(saved["lse"]), den=_ptr(saved["den"]))
    st = load().sla_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(do), ctypes.byref(params), ctypes.byref(sv),
                             _ptr(fwd_workspace), fwd_workspace.numel(), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dW),
                             _ptr(dalpha), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "sla_backward")
    return dq, dk, dv, (dalpha if sla2 else dW), workspace


def attention(q, k, v, *, N: Optional[int] = None, variant: str = "sla", k_crit: int, k_neg: int = 0,
              softmax_scale: float = 0.0, w_proj=None, proj_q=None, proj_k=None, alpha=None,
              phi: str = "softmax"):
    """Differentiable SLA / SLA2 attention for PyTorch: the forward through
    sla_forward_train and, on .backward(), the gradients through sla_backward
    (mask held fixed) for q, k, v and, when they require grad, SLA's w_proj
    and SLA2's alpha. Arguments as for forward(); every tensor on the GPU."""
    import torch

    class _SLAFunction(torch.autograd.Function):
        @staticmethod
        def forward(ctx, q_, k_, v_, w_, a_):
            B, H, Np, d = q_.shape
            n = Np if N is None else int(N)
            p = make_params(B, H, n, d, variant=variant, k_crit=k_crit, k_neg=k_neg,
                            softmax_scale=softmax_scale, w_proj=w_, proj_q=proj_q, proj_k=proj_k, alpha=a_,
                            phi=phi)
            q_, k_, v_ = q_.contiguous(), k_.contiguous(), v_.contiguous()
            out, saved, ws = forward_train(q_, k_, v_, params=p)
            ctx.p, ctx.saved, ctx.ws = p, saved, ws
            ctx.save_for_backward(q_, k_, v_, w_, a_)
            return out

        @staticmethod
        def backward(ctx, do):
            q_, k_, v_, w_, a_ = ctx.saved_tensors
            dq, dk, dv, pg, _ = backward(q_, k_, v_, do.contiguous(), params=ctx.p, saved=ctx.saved,
                                         fwd_workspace=ctx.ws)
            dw = pg.to(w_.dtype) if (w_ is not None and variant == "sla" and ctx.needs_input_grad[3]) else None
            da = pg if (a_ is not None and variant == "sla2" and ctx.needs_input_grad[4]) else None
            return dq, dk, dv, dw, da

    return _SLAFunction.apply(q, k, v, w_proj, alpha)
