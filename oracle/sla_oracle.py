"""Float64 CPU oracle for the SLA / SLA2 sparse-linear attention forward and backward passes.

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline / reference leg may import this module. The product path (the CUDA
library and its binding) never calls it, and this module shares no code with
it: the only common dependency is the seeded input generator in workloads.py.

Sources (cited by page title and section):
  [SLA-sum]   "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable
              Sparse-Linear Attention" -- structured summary (aipaper.cc),
              section 4 "Methodology", "Mathematical formulas & key details",
              formulas 1-4.
  [SLA-walk]  "SLA paper walkthrough: 95 % sparsity, 20x fewer FLOPs"
              (intelliparadigm.com), sections 1.2, 2.2, 2.3 and 3.2.
  [SLA2-notes] "SLA2 -- L3 Cross-Paper Synthesis" (zhaifeiyue.github.io),
              sections 2 and 3.
  [SLA2-art]  popular article on SLA2, arXiv 2602.12675 (mcffsbgs.com),
              paragraphs on the mixing formula, the router, quantisation and
              the two-stage training.

What the pages fix, and the readings taken where they are silent:
  * pool(.) is a mean over each 64-token block ([SLA-sum] formula 1,
    "average pooling along the sequence"; bq = bkv = 64 in [SLA-walk] 2.2).
    The last block of a padded sequence is averaged over its valid rows.
  * Pc = softmax(pool(Q) pool(K)^T / sqrt(d)) ([SLA-sum] formula 1). Softmax
    and the positive scale are strictly increasing, so the per-row ranking is
    taken on the raw pooled dot products.
  * Mc[i,j] = 1 for the top kh % of row i, -1 for the bottom kl %, 0 otherwise
    ([SLA-sum] formula 2). Ties: one total order, score descending then block
    index ascending; the first k_crit are critical, the last k_neg negligible.
  * SLA2's router applies learnable proj_q / proj_k to Q and K before pooling
    ([SLA2-notes] section 2 and [SLA2-art]). Pooling is linear, so projecting
    the pooled vectors is the same map; the float32 specification pools first.
  * phi(x) = softmax over the head dimension ([SLA-walk] 3.2 "phi: Softmax";
    [SLA2-notes] section 3 item 3); optionally elu(x) + 1 elementwise, the
    alternative [SLA-sum] section 4 names and its Table 2 ablates.
  * Sparse branch: softmax attention restricted to the keys of critical
    blocks, scale 1/sqrt(d) ([SLA-sum] step 3; [SLA-walk] 2.2 online softmax).
  * Linear branch: H_i = sum_{Mc[i,j]=0} phi(K_j)^T V_j,
    Z_i = sum_{Mc[i,j]=0} rowsum(phi(K_j)^T), O^l_i = phi(Q_i) H_i / phi(Q_i) Z_i
    ([SLA-sum] formula 3; [SLA-walk] 2.2 pseudo-code). Z_i is a d-vector and
    the denominator a scalar per query row.
  * SLA combine O = O^s + Proj(O^l), Proj a learnable linear map without bias,
    written y = x W with W [d_in, d_out] shared by all heads ([SLA-sum]
    formula 4).
  * SLA2 combine O = alpha O^s + (1 - alpha) O^l with one alpha per head
    ([SLA2-art] mixing-formula paragraph; [SLA2-notes] section 2).
  * Empty sets: no critical block -> O^s = 0; no marginal block -> O^l = 0.
  * Quantised sparse branch ([SLA2-art] quantisation paragraphs: Q, K, P, V
    go to low-bit values with scaling before and restoring after): see
    quantize_* and sparse_branch_quantized below for the exact scheme.
  * SoftTop-k, the differentiable stand-in for Top-k in the first training
    stage of SLA2's router ([SLA2-art] two-stage training; [SLA2-notes]
    section 3): sigmoid((Pc_ij - lambda_i) / tau) on the router's Pc, the
    matrix the hard Top-k ranks, with lambda_i found by bisection so that
    every row sums to k = k_crit. The pages give no value for the
    temperature tau: it is an argument.
  * Backward pass ([SLA-walk] section 2.3): the gradients of <dO, O> with the
    mask held fixed (it is a hard Top-k of pooled scores). The sparse branch
    is softmax attention over the critical keys, differentiated as such; the
    linear branch by the chain rule through num / den, H_i, Z_i and phi.

The bit-exact mask rests on one float32 operation order, emulated here op by
op in NumPy float32 (each elementwise NumPy float32 operation is a single IEEE
round-to-nearest operation; nothing is fused):
  pooled[c] = (((0 + x_0[c]) + x_1[c]) + ... + x_{n-1}[c]), then * 2^-6 for a
              full block or / n (one rounded division) for a partial one;
  router    = sum over k ascending of (pooled[k] * W[k][c]), accumulated from 0;
  score     = sum over k ascending of (qbar_i[k] * kbar_j[k]), accumulated from 0.
The float64 path (pool_f64 ...) gives the exact-arithmetic ranking, used only
as a diagnostic.

Parity pins: every function here is checked in tests/test_oracle_pins.py
against closed forms, brute force on tiny inputs, library routines on the
special cases that reduce to them, and the hand-derived fixtures in
tests/golden/.
"""

from __future__ import annotations

import math
from typing import Optional

import numpy as np

BLOCK = 64


# ---------------------------------------------------------------------------
# bf16 widening
# ---------------------------------------------------------------------------

def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_to_f32(bits).astype(np.float64)


def valid_rows(N: int, Nb: int) -> np.ndarray:
    """n_i: number of real (non-pad) tokens in each 64-token block."""
    return np.minimum(BLOCK, N - BLOCK * np.arange(Nb)).astype(np.int64)


# ---------------------------------------------------------------------------
# float32 specification of the mask scores
# ---------------------------------------------------------------------------

def pool_f32_spec(x32: np.ndarray, N: int) -> np.ndarray:
    """Block mean in the specified float32 order. x32: [N_pad, d] float32 -> [Nb, d]."""
    Np, d = x32.shape
    Nb = Np // BLOCK
    xb = x32.reshape(Nb, BLOCK, d)
    n = valid_rows(N, Nb)
    acc = np.zeros((Nb, d), dtype=np.float32)
    for t in range(BLOCK):
        live = n > t
        acc[live] = acc[live] + xb[live, t, :]
    out = np.empty_like(acc)
    full = n == BLOCK
    out[full] = acc[full] * np.float32(1.0 / 64.0)
    for i in np.nonzero(~full)[0]:
        out[i] = acc[i] / np.float32(n[i])
    return out


def project_f32_spec(xbar: np.ndarray, W32: np.ndarray) -> np.ndarray:
    """Router projection xbar @ W in the specified float32 order (k ascending)."""
    d = xbar.shape[1]
    acc = np.zeros((xbar.shape[0], W32.shape[1]), dtype=np.float32)
    for k in range(d):
        acc = acc + (xbar[:, k:k + 1] * W32[k:k + 1, :])
    return acc


def scores_f32_spec(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """s_ij = sum_k qbar_i[k] * kbar_j[k] in the specified float32 order."""
    d = qbar.shape[1]
    acc = np.zeros((qbar.shape[0], kbar.shape[0]), dtype=np.float32)
    for k in range(d):
        acc = acc + np.multiply.outer(qbar[:, k], kbar[:, k])
    return acc


def classify(scores: np.ndarray, k_crit: int, k_neg: int):
    """Three-way block classification of each row of the compressed scores.

    Order every row by (score descending, block index ascending); the first
    k_crit blocks are critical (1), the last k_neg negligible (-1), the rest
    marginal (0). Returns Mc int8 [R, Nb], crit int32 [R, k_crit] and neg int32
    [R, k_neg], both lists ascending by block index.
    """
    R, Nb = scores.shape
    assert 0 <= k_crit and 0 <= k_neg and k_crit + k_neg <= Nb
    idx = np.broadcast_to(np.arange(Nb), (R, Nb))
    # lexsort: last key is primary; -score ascending == score descending
    order = np.lexsort((idx, -scores.astype(np.float64)), axis=-1)
    Mc = np.zeros((R, Nb), dtype=np.int8)
    rows = np.arange(R)[:, None]
    if k_crit:
        Mc[rows, order[:, :k_crit]] = 1
    if k_neg:
        Mc[rows, order[:, Nb - k_neg:]] = -1
    crit = np.sort(order[:, :k_crit], axis=1).astype(np.int32)
    neg = np.sort(order[:, Nb - k_neg:], axis=1).astype(np.int32) if k_neg else \
        np.zeros((R, 0), dtype=np.int32)
    return Mc, crit, neg


def mask_f32_spec(q32: np.ndarray, k32: np.ndarray, N: int, k_crit: int, k_neg: int,
                  proj_q32: Optional[np.ndarray] = None, proj_k32: Optional[np.ndarray] = None):
    """Pooled scores in the float32 specification and the resulting mask for one head."""
    qbar = pool_f32_spec(q32, N)
    kbar = pool_f32_spec(k32, N)
    if proj_q32 is not None:
        qbar = project_f32_spec(qbar, proj_q32)
        kbar = project_f32_spec(kbar, proj_k32)
    s = scores_f32_spec(qbar, kbar)
    Mc, crit, neg = classify(s, k_crit, k_neg)
    return dict(qbar=qbar, kbar=kbar, scores=s, Mc=Mc, crit=crit, neg=neg)


# ---------------------------------------------------------------------------
# float64 definition
# ---------------------------------------------------------------------------

def pool_f64(x: np.ndarray, N: int) -> np.ndarray:
    """pool(X): mean over the valid rows of each 64-token block, float64."""
    Np, d = x.shape
    Nb = Np // BLOCK
    n = valid_rows(N, Nb)
    out = np.empty((Nb, d), dtype=np.float64)
    for i in range(Nb):
        out[i] = x[i * BLOCK:i * BLOCK + n[i]].mean(axis=0)
    return out


def mask_f64(q: np.ndarray, k: np.ndarray, N: int, k_crit: int, k_neg: int,
             proj_q: Optional[np.ndarray] = None, proj_k: Optional[np.ndarray] = None):
    """Exact-arithmetic (float64) ranking: a diagnostic for the float32 specification."""
    qbar, kbar = pool_f64(q, N), pool_f64(k, N)
    if proj_q is not None:
        qbar, kbar = qbar @ proj_q, kbar @ proj_k
    s = qbar @ kbar.T
    Mc, crit, neg = classify(s, k_crit, k_neg)
    return dict(scores=s, Mc=Mc, crit=crit, neg=neg)


# ---------------------------------------------------------------------------
# SoftTop-k router (stage-1 training of SLA2's router)
# ---------------------------------------------------------------------------

def compressed_softmax(scores: np.ndarray, scale: float) -> np.ndarray:
    """Pc = softmax over each row of scale * s ([SLA-sum] formula 1), float64."""
    x = np.asarray(scores, dtype=np.float64) * scale
    e = np.exp(x - x.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def soft_topk(P: np.ndarray, k: int, tau: float):
    """SoftTop-k of each row of P: M_ij = sigmoid((P_ij - lambda_i) / tau), with
    lambda_i the root of sum_j M_ij = k ([SLA2-art] two-stage training: a
    sigmoid with a temperature in place of Top-k; [SLA2-notes] section 3: a
    binary search for lambda_i per row meets the row-sum constraint).

    The row sum f(lambda) = sum_j sigmoid((P_ij - lambda) / tau) falls strictly
    from n to 0, so the root is unique. Every term is >= k/n once
    lambda <= min_j P_ij - tau logit(k/n), and <= k/n once
    lambda >= max_j P_ij - tau logit(k/n): those two points bracket it. Bisection
    halves the bracket until its midpoint equals an end (no float64 lies
    between). The residual f - k is summed as (#{x_j > 0} - k) plus the signed
    tails t_j = sigmoid(-|x_j|) (-t_j for x_j > 0, +t_j otherwise): each term
    is then small and exact to rounding, where sigmoid(x_j) itself would
    round to 1 and leave f flat around the root. k = n has no finite root:
    M = 1 and lambda = -inf.
    Returns (M [R, n] float64, lambda [R] float64).
    """
    P = np.asarray(P, dtype=np.float64)
    R, n = P.shape
    assert 1 <= k <= n and tau > 0
    if k == n:
        return np.ones((R, n)), np.full(R, -np.inf)

    def split(lam):
        x = (P - lam[:, None]) / tau
        e = np.exp(-np.abs(x))
        return x > 0, e / (1.0 + e)   # sigmoid(x) = 1 - t for x > 0, t otherwise

    off = tau * np.log(k / (n - k))
    lo = P.min(axis=1) - off
    hi = P.max(axis=1) - off
    for _ in range(4000):
        mid = 0.5 * (lo + hi)
        live = (mid > lo) & (mid < hi)
        if not live.any():
            break
        pos, t = split(mid)
        resid = (pos.sum(axis=1) - k) + np.where(pos, -t, t).sum(axis=1)
        above = live & (resid > 0)   # f(mid) > k: the root lies right of mid
        below = live & ~(resid > 0)
        lo = np.where(above, mid, lo)
        hi = np.where(below, mid, hi)
    lam = 0.5 * (lo + hi)
    pos, t = split(lam)
    return np.where(pos, 1.0 - t, t), lam


def router_soft_topk_head(q_bits: np.ndarray, k_bits: np.ndarray, N: int, k: int, tau: float,
                          proj_q_bits: Optional[np.ndarray] = None,
                          proj_k_bits: Optional[np.ndarray] = None,
                          scale: Optional[float] = None) -> dict:
    """Router forward of one head with SoftTop-k in place of the hard Top-k:
    the pooled (and, for SLA2, projected) scores in the float32 specification,
    Pc = softmax(scale s) with scale 1/sqrt(d) by default, then soft_topk(Pc, k, tau).
    Returns dict(scores, Pc, M, lam)."""
    d = q_bits.shape[1]
    pq = bf16_to_f32(proj_q_bits) if proj_q_bits is not None else None
    pk = bf16_to_f32(proj_k_bits) if proj_k_bits is not None else None
    spec = mask_f32_spec(bf16_to_f32(q_bits), bf16_to_f32(k_bits), N, 1, 0, pq, pk)
    Pc = compressed_softmax(spec["scores"], 1.0 / np.sqrt(d) if scale is None else scale)
    M, lam = soft_topk(Pc, k, tau)
    return dict(scores=spec["scores"], Pc=Pc, M=M, lam=lam)


PHI_KINDS = ("softmax", "elu1")


def phi(x: np.ndarray, kind: str = "softmax") -> np.ndarray:
    """Feature map of the linear branch.

    'softmax': softmax over the head dimension (last axis), max-subtracted; the
    map SLA and SLA2 use (SLA walkthrough, section 3.2).
    'elu1': elu(x) + 1 elementwise, i.e. x + 1 for x > 0 and exp(x) otherwise;
    the SLA structured summary (section 4) names it beside softmax and its
    Table 2 ablates it as "SLA (elu+1)".
    """
    if kind == "softmax":
        m = x.max(axis=-1, keepdims=True)
        e = np.exp(x - m)
        return e / e.sum(axis=-1, keepdims=True)
    if kind == "elu1":
        return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))
    raise ValueError(f"unknown phi {kind!r}")


def _block_tokens(blocks: np.ndarray, N: int) -> np.ndarray:
    t = (np.asarray(blocks, dtype=np.int64)[:, None] * BLOCK + np.arange(BLOCK)[None, :]).ravel()
    return t[t < N]


def sparse_branch(q: np.ndarray, k: np.ndarray, v: np.ndarray, Mc: np.ndarray, N: int,
                  scale: float) -> np.ndarray:
    """O^s: for each query row of block i, softmax over the keys of the critical blocks
    of row i of Mc (scores q.k * scale), two-pass (max, then normalised sum). [N, d]."""
    Nb = Mc.shape[0]
    d = v.shape[1]
    out = np.zeros((N, d), dtype=np.float64)
    for i in range(Nb):
        r0, r1 = i * BLOCK, min(N, (i + 1) * BLOCK)
        keys = _block_tokens(np.nonzero(Mc[i] == 1)[0], N)
        if keys.size == 0:
            continue
        s = (q[r0:r1] @ k[keys].T) * scale
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        out[r0:r1] = (p @ v[keys]) / p.sum(axis=1, keepdims=True)
    return out


def linear_terms(k: np.ndarray, v: np.ndarray, N: int, phi_kind: str = "softmax"):
    """Per key block j: h_j = phi(K_j)^T V_j [d, d] and z_j = rowsum(phi(K_j)^T) [d],
    over the block's valid tokens."""
    Np, d = k.shape
    Nb = Np // BLOCK
    pk = phi(k[:N], phi_kind)
    h = np.zeros((Nb, d, d), dtype=np.float64)
    z = np.zeros((Nb, d), dtype=np.float64)
    for j in range(Nb):
        t0, t1 = j * BLOCK, min(N, (j + 1) * BLOCK)
        h[j] = pk[t0:t1].T @ v[t0:t1]
        z[j] = pk[t0:t1].sum(axis=0)
    return h, z


def linear_branch(q: np.ndarray, k: np.ndarray, v: np.ndarray, Mc: np.ndarray, N: int,
                  phi_kind: str = "softmax") -> np.ndarray:
    """O^l_i = phi(Q_i) H_i / (phi(Q_i) Z_i) with H_i, Z_i summed over the marginal
    blocks (Mc == 0) of row i. Rows whose marginal set is empty get O^l = 0. [N, d]."""
    Nb = Mc.shape[0]
    d = v.shape[1]
    h, z = linear_terms(k, v, N, phi_kind)
    marg = (Mc == 0).astype(np.float64)  # [Nb, Nb]; H_i = sum_j marg[i, j] h_j
    H = (marg @ h.reshape(Nb, d * d)).reshape(Nb, d, d)
    Z = marg @ z
    out = np.zeros((N, d), dtype=np.float64)
    pq = phi(q[:N], phi_kind)
    for i in range(Nb):
        if not marg[i].any():
            continue
        r0, r1 = i * BLOCK, min(N, (i + 1) * BLOCK)
        num = pq[r0:r1] @ H[i]
        den = pq[r0:r1] @ Z[i]
        out[r0:r1] = num / den[:, None]
    return out


def combine_sla(o_s: np.ndarray, o_l: np.ndarray, w_proj: np.ndarray) -> np.ndarray:
    """SLA: O = O^s + Proj(O^l), Proj(x) = x W (no bias)."""
    return o_s + o_l @ w_proj


def combine_sla2(o_s: np.ndarray, o_l: np.ndarray, alpha_h: float) -> np.ndarray:
    """SLA2: O = alpha O^s + (1 - alpha) O^l."""
    return alpha_h * o_s + (1.0 - alpha_h) * o_l


# ---------------------------------------------------------------------------
# backward pass (gradients of the forward above, the mask held fixed)
# ---------------------------------------------------------------------------
#
# [SLA-walk] section 2.3: the sparse path follows the FlashAttention backward on
# the Mc = 1 blocks; the linear path obtains the gradients of phi(Q), phi(K)
# and V by the chain rule, accumulated block by block. The mask is a hard
# Top-k of the pooled scores and has no gradient. Each function below is the
# chain rule of the matching forward function written out; rows past N get
# zero gradient.

def phi_vjp(x: np.ndarray, dy: np.ndarray, kind: str = "softmax") -> np.ndarray:
    """dx for y = phi(x) and upstream dy (row-wise Jacobian of the feature map)."""
    if kind == "softmax":
        y = phi(x, kind)
        return y * (dy - (dy * y).sum(axis=-1, keepdims=True))
    if kind == "elu1":
        return np.where(x > 0, dy, dy * np.exp(np.minimum(x, 0.0)))
    raise ValueError(f"unknown phi {kind!r}")


def sparse_branch_backward(q, k, v, Mc, N, scale, do_s):
    """Gradients of O^s for upstream do_s [N, d]: (dq, dk, dv) [N, d] each, and
    lse [N], the natural-log normaliser log sum exp(scale q.k) of each row over
    its critical keys (-inf for a row without critical blocks)."""
    Nb = Mc.shape[0]
    d = v.shape[1]
    dq, dk, dv = (np.zeros((N, d)) for _ in range(3))
    lse = np.full(N, -np.inf)
    for i in range(Nb):
        r0, r1 = i * BLOCK, min(N, (i + 1) * BLOCK)
        keys = _block_tokens(np.nonzero(Mc[i] == 1)[0], N)
        if keys.size == 0:
            continue
        s = (q[r0:r1] @ k[keys].T) * scale
        mx = s.max(axis=1, keepdims=True)
        e = np.exp(s - mx)
        l = e.sum(axis=1, keepdims=True)
        p = e / l
        lse[r0:r1] = (mx + np.log(l))[:, 0]
        g = do_s[r0:r1]
        dv[keys] += p.T @ g
        dp = g @ v[keys].T
        ds = p * (dp - (dp * p).sum(axis=1, keepdims=True))
        dq[r0:r1] += scale * (ds @ k[keys])
        dk[keys] += scale * (ds.T @ q[r0:r1])
    return dq, dk, dv, lse


def linear_branch_backward(q, k, v, Mc, N, do_l, phi_kind="softmax"):
    """Gradients of O^l for upstream do_l [N, d]. With num = phi(Q_i) H_i,
    den = phi(Q_i) Z_i and O^l = num / den:
      dnum = do_l / den,  dden = -rowsum(do_l * O^l) / den,
      dphi(Q_i) = dnum H_i^T + dden Z_i^T,
      dH_i = phi(Q_i)^T dnum,  dZ_i = phi(Q_i)^T dden,
    and, with A_j = sum of dH_i and b_j = sum of dZ_i over the rows i that have
    j marginal, dphi(K_j) = V_j A_j^T + 1 b_j^T and dV_j = phi(K_j) A_j.
    Returns (dq, dk, dv) [N, d] and den [N] (0 where the row has no marginal block)."""
    Nb = Mc.shape[0]
    d = v.shape[1]
    h, z = linear_terms(k, v, N, phi_kind)
    marg = (Mc == 0).astype(np.float64)
    H = (marg @ h.reshape(Nb, d * d)).reshape(Nb, d, d)
    Z = marg @ z
    pq = phi(q[:N], phi_kind)
    pk = phi(k[:N], phi_kind)
    dpq = np.zeros((N, d))
    dH = np.zeros((Nb, d, d))
    dZ = np.zeros((Nb, d))
    den_all = np.zeros(N)
    for i in range(Nb):
        if not marg[i].any():
            continue
        r0, r1 = i * BLOCK, min(N, (i + 1) * BLOCK)
        num = pq[r0:r1] @ H[i]
        den = pq[r0:r1] @ Z[i]
        o = num / den[:, None]
        den_all[r0:r1] = den
        g = do_l[r0:r1]
        dnum = g / den[:, None]
        dden = -(g * o).sum(axis=1) / den
        dpq[r0:r1] = dnum @ H[i].T + dden[:, None] * Z[i][None, :]
        dH[i] = pq[r0:r1].T @ dnum
        dZ[i] = pq[r0:r1].T @ dden
    A = (marg.T @ dH.reshape(Nb, d * d)).reshape(Nb, d, d)
    b = marg.T @ dZ
    dpk = np.zeros((N, d))
    dv = np.zeros((N, d))
    for j in range(Nb):
        t0, t1 = j * BLOCK, min(N, (j + 1) * BLOCK)
        dpk[t0:t1] = v[t0:t1] @ A[j].T + b[j][None, :]
        dv[t0:t1] = pk[t0:t1] @ A[j]
    dq = phi_vjp(q[:N], dpq, phi_kind)
    dk = phi_vjp(k[:N], dpk, phi_kind)
    return dq, dk, dv, den_all


def backward_head(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray, do: np.ndarray, N: int, *,
                  variant: str, k_crit: int, k_neg: int, softmax_scale: Optional[float] = None,
                  w_proj_bits: Optional[np.ndarray] = None, proj_q_bits: Optional[np.ndarray] = None,
                  proj_k_bits: Optional[np.ndarray] = None, alpha_h: Optional[float] = None,
                  phi_kind: str = "softmax") -> dict:
    """Backward pass of one (b, h) head: gradients of <dO, O> for upstream do
    [N, d] (float64), O the forward_head output, with the mask of the forward.
    SLA (O = O^s + O^l W): dO^s = dO, dO^l = dO W^T, dW = O^l^T dO.
    SLA2 (O = a O^s + (1 - a) O^l): dO^s = a dO, dO^l = (1 - a) dO,
    da = sum(dO * (O^s - O^l)).
    Returns dQ, dK, dV [N, d], dW [d, d] (SLA) or dalpha (SLA2), the forward's
    O_s, O_l, the sparse row normaliser lse [N], the linear denominator den [N]
    and the mask."""
    fw = forward_head(q_bits, k_bits, v_bits, N, variant=variant, k_crit=k_crit, k_neg=k_neg,
                      softmax_scale=softmax_scale, w_proj_bits=w_proj_bits, proj_q_bits=proj_q_bits,
                      proj_k_bits=proj_k_bits, alpha_h=alpha_h, phi_kind=phi_kind)
    d = q_bits.shape[1]
    scale = (1.0 / math.sqrt(d)) if not softmax_scale else float(softmax_scale)
    W = None
    if variant == "sla":
        W = bf16_to_f64(w_proj_bits) if w_proj_bits is not None else np.eye(d)
    res = backward_f64(bf16_to_f64(q_bits), bf16_to_f64(k_bits), bf16_to_f64(v_bits), fw["Mc"], do, N,
                       variant=variant, scale=scale, W=W, alpha_h=alpha_h, phi_kind=phi_kind)
    res.update(O=fw["O"], Mc=fw["Mc"], crit=fw["crit"], neg=fw["neg"])
    return res


def backward_f64(q, k, v, Mc, do, N, *, variant, scale, W=None, alpha_h=None, phi_kind="softmax") -> dict:
    """backward_head on float64 [N_pad, d] arrays with a given mask."""
    do = np.asarray(do, dtype=np.float64)[:N]
    o_s = sparse_branch(q, k, v, Mc, N, scale)
    o_l = linear_branch(q, k, v, Mc, N, phi_kind)
    res = dict(O_s=o_s, O_l=o_l)
    if variant == "sla":
        do_s, do_l = do, do @ W.T
        res["dW"] = o_l.T @ do
    else:
        a = float(alpha_h)
        do_s, do_l = a * do, (1.0 - a) * do
        res["dalpha"] = float((do * (o_s - o_l)).sum())
    dq_s, dk_s, dv_s, lse = sparse_branch_backward(q, k, v, Mc, N, scale, do_s)
    dq_l, dk_l, dv_l, den = linear_branch_backward(q, k, v, Mc, N, do_l, phi_kind)
    res.update(dQ=dq_s + dq_l, dK=dk_s + dk_l, dV=dv_s + dv_l, lse=lse, den=den)
    return res


# ---------------------------------------------------------------------------
# quantised sparse branch (INT8 Q, K; FP8 e4m3 P, V)
# ---------------------------------------------------------------------------
#
# Scheme (the pages say only that Q, K, P, V are quantised with a scale before
# the products and restored after; the granularities below are this
# implementation's reading):
#   * Q, K: symmetric INT8 per 64-token block of a head. s = absmax / 127
#     (float32, one rounded division; absmax over the block's valid rows and
#     all d columns; s = 1 if absmax = 0). code = clamp(rint(x / s), -127, 127)
#     with x / s one rounded float32 division and rint round-half-even.
#   * V: FP8 e4m3 per 64-token block, s_v = absmax / 448, code = e4m3(v / s_v)
#     (round to nearest even, saturating at +-448, subnormals kept).
#   * S = (Qc Kc^T exact integer) * s_q * s_k * softmax_scale.
#   * P~ = 2^(x - m) with x = S log2(e) and m = ceil(max_j x) the row max
#     rounded up to an integer, so P~ is in (0, 1] and its largest entry in
#     (1/2, 1]. The pages fix only that P is scaled before the product and
#     restored after; the scale of a row is taken as a power of two because
#     e4m3 rounding commutes with multiplication by 2^k for values that stay
#     normal and below the saturation bound: quantise(P 2^k) 2^-k is then the
#     same value for every such k, so the scale adds no rounding of its own
#     and the result does not depend on how the offset is reached. The offset
#     puts the row's largest P~ in (1/2, 1], i.e. its code (after the 2^8
#     multiplier below) in (128, 256], inside e4m3's normal range and below 448.
#   * Each key block's V scale is folded into P relative to the largest V
#     scale of the head, r_j = s_v,j / max_j s_v,j (one float32 division), and
#     P enters the PV product as e4m3(P~ * r_j * 2^8); the row sum l uses the
#     unquantised P~. O^s = (sum e4m3(P~ r 2^8) Vc) * max s_v / 2^8 / l.

E4M3_MAX = 448.0
LOG2E = 1.0 / math.log(2.0)


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Nearest OCP FP8 E4M3 value (bias 7, 3 mantissa bits, no infinities, max
    normal 1.75 * 2^8 = 448, min normal 2^-6, subnormal step 2^-9), ties to even,
    saturating to +-448. Returned as float64 values."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    out = np.zeros_like(a)
    nz = a > 0
    _, ex = np.frexp(np.where(nz, a, 1.0))  # a = m 2^ex, m in [0.5, 1): binade exponent ex - 1
    e = np.maximum(ex.astype(np.float64) - 1.0, -6.0)  # subnormals share the 2^-6 quantum
    quantum = np.exp2(e - 3.0)
    q = np.rint(a / quantum) * quantum  # a / quantum is exact (power of two)
    out[nz] = q[nz]
    out = np.minimum(out, E4M3_MAX)
    return np.copysign(out, x)


def quantize_int8_blocks(x32: np.ndarray, N: int):
    """Per-block symmetric INT8 of a float32 [N_pad, d] head; pad rows -> 0.
    Returns (codes int8 [N_pad, d], scales float32 [Nb])."""
    Np, d = x32.shape
    Nb = Np // BLOCK
    n = valid_rows(N, Nb)
    codes = np.zeros((Np, d), dtype=np.int8)
    scales = np.ones(Nb, dtype=np.float32)
    for i in range(Nb):
        blk = x32[i * BLOCK:i * BLOCK + n[i]]
        amax = np.float32(np.abs(blk).max())
        s = np.float32(amax / np.float32(127.0)) if amax > 0 else np.float32(1.0)
        scales[i] = s
        y = (blk / s).astype(np.float32)
        codes[i * BLOCK:i * BLOCK + n[i]] = np.clip(np.rint(y), -127, 127).astype(np.int8)
    return codes, scales


def quantize_e4m3_blocks(x32: np.ndarray, N: int):
    """Per-block FP8 e4m3 of a float32 [N_pad, d] head (values returned as float64),
    scale absmax / 448 per block; pad rows -> 0."""
    Np, d = x32.shape
    Nb = Np // BLOCK
    n = valid_rows(N, Nb)
    vals = np.zeros((Np, d), dtype=np.float64)
    scales = np.ones(Nb, dtype=np.float32)
    for i in range(Nb):
        blk = x32[i * BLOCK:i * BLOCK + n[i]]
        amax = np.float32(np.abs(blk).max())
        s = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
        scales[i] = s
        vals[i * BLOCK:i * BLOCK + n[i]] = e4m3_round((blk / s).astype(np.float32))
    return vals, scales


def sparse_branch_quantized(q32: np.ndarray, k32: np.ndarray, v32: np.ndarray, Mc: np.ndarray,
                            N: int, scale: float) -> np.ndarray:
    """Emulation of the INT8 / FP8 sparse branch (scheme above). [N, d] float64."""
    qc, sq = quantize_int8_blocks(q32, N)
    kc, sk = quantize_int8_blocks(k32, N)
    vq, sv = quantize_e4m3_blocks(v32, N)
    sv_max = float(sv.max())
    Nb = Mc.shape[0]
    out = np.zeros((N, v32.shape[1]), dtype=np.float64)
    qc64, kc64 = qc.astype(np.float64), kc.astype(np.float64)
    for i in range(Nb):
        r0, r1 = i * BLOCK, min(N, (i + 1) * BLOCK)
        cb = np.nonzero(Mc[i] == 1)[0]
        keys = _block_tokens(cb, N)
        if keys.size == 0:
            continue
        kblk = keys // BLOCK
        s = (qc64[r0:r1] @ kc64[keys].T) * (float(sq[i]) * sk[kblk].astype(np.float64)) * scale
        x = s * LOG2E
        p = np.exp2(x - np.ceil(x.max(axis=1, keepdims=True)))
        r = (sv[kblk] / np.float32(sv_max)).astype(np.float64)
        pq = e4m3_round(p * r[None, :] * 256.0)
        out[r0:r1] = (pq @ vq[keys]) * (sv_max / 256.0) / p.sum(axis=1, keepdims=True)
    return out


# ---------------------------------------------------------------------------
# whole forward for one head
# ---------------------------------------------------------------------------

def forward_head(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray, N: int, *,
                 variant: str, k_crit: int, k_neg: int, softmax_scale: Optional[float] = None,
                 w_proj_bits: Optional[np.ndarray] = None, proj_q_bits: Optional[np.ndarray] = None,
                 proj_k_bits: Optional[np.ndarray] = None, alpha_h: Optional[float] = None,
                 quantized: bool = False, with_f64_mask: bool = False,
                 phi_kind: str = "softmax") -> dict:
    """Forward pass of one (b, h) head from bf16 bit arrays [N_pad, d].

    Returns a dict with O [N, d] float64 (unrounded), O_s, O_l, the mask (Mc,
    crit, neg) from the float32 specification, the pooled float32 vectors and,
    optionally, the float64 ranking for diagnostics. With quantized=True, O_sq
    holds the emulated low-bit sparse branch and O_q the output built from it.
    """
    d = q_bits.shape[1]
    scale = (1.0 / math.sqrt(d)) if not softmax_scale else float(softmax_scale)
    q32, k32, v32 = bf16_to_f32(q_bits), bf16_to_f32(k_bits), bf16_to_f32(v_bits)
    pq32 = bf16_to_f32(proj_q_bits) if (variant == "sla2" and proj_q_bits is not None) else None
    pk32 = bf16_to_f32(proj_k_bits) if (variant == "sla2" and proj_k_bits is not None) else None
    m = mask_f32_spec(q32, k32, N, k_crit, k_neg, pq32, pk32)
    Mc = m["Mc"]
    q, k, v = q32.astype(np.float64), k32.astype(np.float64), v32.astype(np.float64)
    o_s = sparse_branch(q, k, v, Mc, N, scale)
    o_l = linear_branch(q, k, v, Mc, N, phi_kind)
    if variant == "sla":
        W = bf16_to_f64(w_proj_bits) if w_proj_bits is not None else np.eye(d)
        comb = lambda a, b: combine_sla(a, b, W)  # noqa: E731
    elif variant == "sla2":
        comb = lambda a, b: combine_sla2(a, b, float(alpha_h))  # noqa: E731
    else:
        raise ValueError(variant)
    res = dict(O=comb(o_s, o_l), O_s=o_s, O_l=o_l, **m)
    if quantized:
        o_sq = sparse_branch_quantized(q32, k32, v32, Mc, N, scale)
        res["O_sq"] = o_sq
        res["O_q"] = comb(o_sq, o_l)
    if with_f64_mask:
        pq64 = pq32.astype(np.float64) if pq32 is not None else None
        pk64 = pk32.astype(np.float64) if pk32 is not None else None
        res["f64"] = mask_f64(q, k, N, k_crit, k_neg, pq64, pk64)
    return res


def mask_disagreements(spec: dict, f64: dict, k_crit: int, k_neg: int) -> list:
    """Rows where the float32-spec ranking and the exact ranking give different
    masks, with the exact-arithmetic score gap at each boundary (diagnostic)."""
    out = []
    diff = np.nonzero((spec["Mc"] != f64["Mc"]).any(axis=1))[0]
    for i in diff:
        s = np.sort(f64["scores"][i])[::-1]
        gaps = []
        if k_crit and k_crit < s.size:
            gaps.append(float(s[k_crit - 1] - s[k_crit]))
        if k_neg:
            b = s.size - k_neg
            gaps.append(float(s[b - 1] - s[b]))
        out.append((int(i), gaps))
    return out


def forward(inputs, heads=None, quantized: bool = False) -> dict:
    """Run forward_head over the heads of a workloads.Inputs. Returns per-head results
    keyed by (b, h)."""
    w = inputs.w
    res = {}
    hl = inputs.heads if heads is None else heads
    full = inputs.q.shape[:2] == (w.B, w.H) and len(inputs.heads) == w.B * w.H
    for idx, (b, h) in enumerate(inputs.heads):
        if (b, h) not in hl:
            continue
        sel = (b, h) if full else (idx, 0)
        res[(b, h)] = forward_head(
            inputs.q[sel], inputs.k[sel], inputs.v[sel], w.N, variant=w.variant,
            k_crit=w.k_crit, k_neg=w.k_neg, w_proj_bits=inputs.w_proj,
            proj_q_bits=inputs.proj_q, proj_k_bits=inputs.proj_k,
            alpha_h=None if inputs.alpha is None else float(inputs.alpha[h]),
            quantized=quantized, phi_kind=w.phi)
    return res
