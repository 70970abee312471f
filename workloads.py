"""Seeded synthetic inputs for the SLA / SLA2 forward pass.

This module holds input generation only: shapes, seeds, value distributions
and the block-count convention for the critical / negligible fractions. It
contains none of the method's arithmetic, and it is the one piece of code
that both the CUDA path (through the Python binding) and the float64 oracle
use.

Workloads stand in for the Wan2.1 attention inputs that the SLA and SLA2
pages measure on (Wan2.1-1.3B at 480p: H=12, d=128, about 32k tokens;
Wan2.1-14B-720P: H=40, d=128, 75600 tokens). Real activations are not
available, so Q and K are block-clustered Gaussians: every 64-token block
draws a mean mu ~ N(0, s^2 I_d) and every token adds N(0, I_d) noise; Q and K
draw independent means. V ~ N(0, 1). The d x d weights (SLA's output
projection, SLA2's router proj_q / proj_k) are N(0, 1/d); SLA2's per-head
mixing weight alpha is U(0.6, 0.95). Every value is drawn in float32 and
rounded to bfloat16 (round to nearest even).

Random streams are keyed per (tensor, batch, head) with
``SeedSequence(seed, spawn_key=(tensor, b, h))`` so that a single sampled
head can be regenerated without drawing the others.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Iterable, Optional

import numpy as np

BLOCK = 64  # bq = bkv = 64 tokens per block

# stream ids for SeedSequence spawn keys
_T_Q, _T_K, _T_V, _T_WPROJ, _T_PROJQ, _T_PROJK, _T_ALPHA, _T_DO = range(8)

# value written into the rows past N of a padded tensor; a kernel that reads
# them by mistake produces visibly wrong results
DEFAULT_PAD_VALUE = 64.0


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (RNE); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    out = (rounded >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def n_pad(N: int) -> int:
    return BLOCK * ((N + BLOCK - 1) // BLOCK)


def block_counts(Nb: int, crit_pct: float, neg_pct: float) -> tuple[int, int]:
    """Convert kh % / kl % to whole blocks per row.

    The pages give the fractions only (kh = 5 %, kl = 10 % for SLA; 3 %
    critical for SLA2 at 97 % sparsity); the count per row is
    k_crit = clamp(floor(kh * Nb), 1, Nb) and k_neg = floor(kl * Nb), with
    k_crit + k_neg <= Nb. Percentages are handled as exact rationals.
    """
    from fractions import Fraction

    kc = math.floor(Fraction(str(crit_pct)) * Nb / 100)
    kn = math.floor(Fraction(str(neg_pct)) * Nb / 100)
    kc = max(1, min(Nb, kc))
    kn = max(0, min(Nb - kc, kn))
    return kc, kn


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    variant: str  # "sla" | "sla2"
    precision: str  # "bf16" | "i8qk_f8pv"
    k_crit: int
    k_neg: int
    cluster_scale: float
    seed: int
    pad_value: float = DEFAULT_PAD_VALUE
    phi: str = "softmax"  # feature map of the linear branch: "softmax" | "elu1"

    @property
    def N_pad(self) -> int:
        return n_pad(self.N)

    @property
    def Nb(self) -> int:
        return self.N_pad // BLOCK

    @property
    def sparsity(self) -> float:
        """Fraction of (query block, key block) pairs not computed exactly."""
        return 1.0 - self.k_crit / self.Nb

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def make_workload(name, B, H, N, d, variant, crit_pct=None, neg_pct=0.0, k_crit=None,
                  k_neg=None, cluster_scale=2.0, seed=0, precision="bf16", phi="softmax") -> Workload:
    Nb = n_pad(N) // BLOCK
    if k_crit is None:
        k_crit, k_neg = block_counts(Nb, crit_pct, neg_pct)
    return Workload(name=name, B=B, H=H, N=N, d=d, variant=variant, precision=precision,
                    k_crit=int(k_crit), k_neg=int(k_neg or 0), cluster_scale=float(cluster_scale),
                    seed=int(seed), phi=phi)


# ---------------------------------------------------------------------------
# The workloads, restated from the benchmark configuration list.
# ---------------------------------------------------------------------------

WORKLOADS: dict[str, Workload] = {
    # SLA, B=1 H=2 N=1024 d=64, 16 blocks: 2 critical, 2 negligible per row
    "sla_b1h2n1024d64": make_workload("sla_b1h2n1024d64", 1, 2, 1024, 64, "sla", k_crit=2,
                                      k_neg=2, cluster_scale=1.0, seed=0),
    # SLA on a Wan2.1-1.3B-shaped call: kh=5 % critical, kl=10 % negligible
    "sla_wan13b_b1h12n32768d128_s95": make_workload(
        "sla_wan13b_b1h12n32768d128_s95", 1, 12, 32768, 128, "sla", crit_pct=5, neg_pct=10,
        cluster_scale=2.0, seed=1),
    # SLA2 at 97 % sparsity: 3 % critical, the rest linear, per-head alpha
    "sla2_b1h12n32768d128_s97": make_workload(
        "sla2_b1h12n32768d128_s97", 1, 12, 32768, 128, "sla2", crit_pct=3, neg_pct=0,
        cluster_scale=2.0, seed=2),
    # SLA2 with the INT8 (Q,K) / FP8 e4m3 (P,V) sparse branch, Wan2.1-14B-720P-shaped
    "sla2_q_wan14b_b1h40n75600d128_s97": make_workload(
        "sla2_q_wan14b_b1h40n75600d128_s97", 1, 40, 75600, 128, "sla2", crit_pct=3, neg_pct=0,
        cluster_scale=2.0, seed=3, precision="i8qk_f8pv"),
}

SWEEP_N = (4096, 16384, 32768, 65536, 131072)
SWEEP_SPARSITY = (90, 95, 97)


def sweep_workload(N: int, sparsity_pct: int, variant: str) -> Workload:
    """The sequence-length / sparsity sweep (H=12, d=128, seed 4).

    SLA keeps kl = 10 % negligible blocks; SLA2 has none. 0 % sparsity is the
    dense baseline kernel, not a SLA workload.
    """
    neg = 10 if variant == "sla" else 0
    return make_workload(f"{variant}_sweep_b1h12n{N}d128_s{sparsity_pct}", 1, 12, N, 128, variant,
                         crit_pct=100 - sparsity_pct, neg_pct=neg, cluster_scale=2.0, seed=4)


# ---------------------------------------------------------------------------
# Generation
# ---------------------------------------------------------------------------

def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=key)))


def head_tensor(w: Workload, tensor: str, b: int, h: int) -> np.ndarray:
    """One head of Q, K or V: uint16 bf16 bits, shape [N_pad, d]; rows >= N hold pad_value."""
    tid = {"q": _T_Q, "k": _T_K, "v": _T_V}[tensor]
    rng = _rng(w.seed, tid, b, h)
    Np, d = w.N_pad, w.d
    if tensor == "v":
        x = rng.standard_normal((Np, d), dtype=np.float32)
    else:
        mu = rng.standard_normal((w.Nb, d), dtype=np.float32) * np.float32(w.cluster_scale)
        x = rng.standard_normal((Np, d), dtype=np.float32)
        x += np.repeat(mu, BLOCK, axis=0)
    if Np > w.N:
        x[w.N:] = np.float32(w.pad_value)
    return f32_to_bf16_bits(x)


def head_grad_output(w: Workload, b: int, h: int) -> np.ndarray:
    """Upstream gradient dO of one head for the backward pass: N(0, 1), bf16
    bits [N_pad, d]; rows >= N hold pad_value (the backward must ignore them)."""
    rng = _rng(w.seed, _T_DO, b, h)
    x = rng.standard_normal((w.N_pad, w.d), dtype=np.float32)
    if w.N_pad > w.N:
        x[w.N:] = np.float32(w.pad_value)
    return f32_to_bf16_bits(x)


def grad_output(w: Workload, heads: Optional[Iterable[tuple[int, int]]] = None) -> np.ndarray:
    """dO for every head ([B, H, N_pad, d]) or for a list of heads ([len, 1, N_pad, d])."""
    full = heads is None
    hl = [(b, h) for b in range(w.B) for h in range(w.H)] if full else list(heads)
    out = np.empty(((w.B, w.H) if full else (len(hl), 1)) + (w.N_pad, w.d), dtype=np.uint16)
    for idx, (b, h) in enumerate(hl):
        out[(b, h) if full else (idx, 0)] = head_grad_output(w, b, h)
    return out


def weight(w: Workload, which: str) -> np.ndarray:
    """d x d bf16 bits, N(0, 1/d): 'w_proj' (SLA), 'proj_q' / 'proj_k' (SLA2 router)."""
    tid = {"w_proj": _T_WPROJ, "proj_q": _T_PROJQ, "proj_k": _T_PROJK}[which]
    rng = _rng(w.seed, tid, 0, 0)
    x = rng.standard_normal((w.d, w.d), dtype=np.float32) * np.float32(1.0 / math.sqrt(w.d))
    return f32_to_bf16_bits(x)


def alpha(w: Workload) -> np.ndarray:
    """SLA2 per-head mixing weights, float32 [H], U(0.6, 0.95)."""
    rng = _rng(w.seed, _T_ALPHA, 0, 0)
    return rng.uniform(0.6, 0.95, size=w.H).astype(np.float32)


@dataclasses.dataclass
class Inputs:
    w: Workload
    q: np.ndarray  # uint16 [B, H, N_pad, d]
    k: np.ndarray
    v: np.ndarray
    w_proj: Optional[np.ndarray]  # uint16 [d, d] (SLA)
    proj_q: Optional[np.ndarray]  # uint16 [d, d] (SLA2)
    proj_k: Optional[np.ndarray]
    alpha: Optional[np.ndarray]  # float32 [H] (SLA2)
    heads: list  # list of (b, h) that q/k/v hold, in order


def make_inputs(w: Workload, heads: Optional[Iterable[tuple[int, int]]] = None) -> Inputs:
    """Generate the inputs of a workload.

    With ``heads=None`` every (b, h) is generated and q/k/v have shape
    [B, H, N_pad, d]. With an explicit list, q/k/v have shape
    [len(heads), 1, N_pad, d] (one entry per requested head, same values as the
    full generation).
    """
    full = heads is None
    hl = [(b, h) for b in range(w.B) for h in range(w.H)] if full else list(heads)
    shape = (w.B, w.H) if full else (len(hl), 1)
    out = {}
    for t in ("q", "k", "v"):
        arr = np.empty(shape + (w.N_pad, w.d), dtype=np.uint16)
        for idx, (b, h) in enumerate(hl):
            dst = arr[b, h] if full else arr[idx, 0]
            dst[...] = head_tensor(w, t, b, h)
        out[t] = arr
    sla2 = w.variant == "sla2"
    return Inputs(w=w, q=out["q"], k=out["k"], v=out["v"],
                  w_proj=None if sla2 else weight(w, "w_proj"),
                  proj_q=weight(w, "proj_q") if sla2 else None,
                  proj_k=weight(w, "proj_k") if sla2 else None,
                  alpha=alpha(w) if sla2 else None, heads=hl)
