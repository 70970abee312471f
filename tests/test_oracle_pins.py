"""Pins for the float64 oracle: closed forms, brute force on tiny inputs,
library routines on the special cases that reduce to them, and the
hand-derived fixtures in tests/golden/. CPU only."""

import glob
import json
import math
import os

import numpy as np
import pytest

import workloads as W
from oracle import sla_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def bits(x):
    return W.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def head_from_blocks(blocks, N, pad):
    """Expand per-block row cycles into an [N_pad, d] float32 array."""
    Nb = len(blocks)
    d = len(blocks[0][0])
    x = np.empty((Nb * 64, d), dtype=np.float32)
    for i, cyc in enumerate(blocks):
        for t in range(64):
            x[i * 64 + t] = cyc[t % len(cyc)]
    x[N:] = pad
    return x


# ---------------------------------------------------------------------------
# hand-derived fixtures
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("path", sorted(glob.glob(os.path.join(GOLDEN, "*.json"))),
                         ids=lambda p: os.path.basename(p))
def test_golden_fixture(path):
    g = json.load(open(path))
    N = g["N"]
    q, k, v = (head_from_blocks(g[t], N, g["pad"]) for t in ("q", "k", "v"))
    kw = dict(variant=g["variant"], k_crit=g["k_crit"], k_neg=g["k_neg"])
    if g["variant"] == "sla":
        kw["w_proj_bits"] = bits(g["w_proj"])
    else:
        kw["alpha_h"] = g["alpha"]
    r = O.forward_head(bits(q), bits(k), bits(v), N, **kw)
    np.testing.assert_array_equal(r["Mc"], np.array(g["expected_Mc"], dtype=np.int8))
    e = math.e
    want = np.array([eval(x, {"e": e}) if isinstance(x, str) else x for x in g["expected_row"]])
    np.testing.assert_allclose(r["O"], np.broadcast_to(want, r["O"].shape), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# phi
# ---------------------------------------------------------------------------

def test_phi_is_softmax_over_head_dim():
    x = RNG.standard_normal((7, 5, 16)) * 3
    p = O.phi(x)
    assert np.all(p > 0)
    np.testing.assert_allclose(p.sum(axis=-1), 1.0, atol=1e-14)
    # invariant to a per-row shift, and ratios are exp of differences
    np.testing.assert_allclose(O.phi(x + 11.5), p, atol=1e-15)
    np.testing.assert_allclose(p[..., 3] / p[..., 9], np.exp(x[..., 3] - x[..., 9]), rtol=1e-12)
    # large inputs stay finite (max-subtracted)
    assert np.isfinite(O.phi(x * 1e3)).all()


def test_phi_elu1_is_elementwise_elu_plus_one():
    # elu(x) + 1: x + 1 above zero, exp(x) at or below it; elementwise, so an
    # entry depends on nothing else in its row, and rows are not normalised
    x = RNG.standard_normal((6, 16)) * 3
    p = O.phi(x, "elu1")
    assert np.all(p > 0)
    y = x.copy()
    y[:, 5] += 7.0
    q = O.phi(y, "elu1")
    np.testing.assert_array_equal(np.delete(q, 5, axis=1), np.delete(p, 5, axis=1))
    assert not np.allclose(p.sum(axis=-1), 1.0)
    # continuity at 0 (value 1 from both sides), slope 1 above, exp ratios below
    np.testing.assert_allclose(O.phi(np.array([-1e-12, 0.0, 1e-12]), "elu1"), 1.0, atol=1e-11)
    pos = np.abs(x) + 0.25
    np.testing.assert_allclose(O.phi(pos + 0.5, "elu1") - O.phi(pos, "elu1"), 0.5, atol=1e-13)
    neg = -np.abs(x) - 0.25
    np.testing.assert_allclose(O.phi(neg, "elu1") / O.phi(neg - 2.0, "elu1"), np.exp(2.0), rtol=1e-12)
    assert O.phi(np.array([-800.0]), "elu1")[0] == 0.0 and O.phi(np.array([800.0]), "elu1")[0] == 801.0
    with pytest.raises(ValueError):
        O.phi(x, "relu")


# ---------------------------------------------------------------------------
# float32 specification of the mask scores
# ---------------------------------------------------------------------------

def test_pool_spec_exact_on_integers():
    N = 64 * 5 + 23  # a partial last block of 23 rows
    x = RNG.integers(-20, 21, size=(64 * 6, 8)).astype(np.float32)
    got = O.pool_f32_spec(x, N)
    exact = O.pool_f64(x.astype(np.float64), N)
    # integer sums are exact in float32; full blocks divide by 64 exactly and the
    # partial block by 23 with one rounding: at most half an ulp of float32
    np.testing.assert_array_equal(got[:5], exact[:5].astype(np.float32))
    ulp = np.spacing(np.abs(got[5]).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(got[5] - exact[5]) <= 0.5 * ulp + 1e-30)


def test_pool_spec_close_to_mean_and_ignores_pad():
    N = 64 * 3 + 10
    x = RNG.standard_normal((64 * 4, 32)).astype(np.float32)
    a = O.pool_f32_spec(x, N)
    x2 = x.copy()
    x2[N:] = np.nan
    b = O.pool_f32_spec(x2, N)
    np.testing.assert_array_equal(a, b)
    ref = O.pool_f64(x.astype(np.float64), N)
    assert np.abs(a - ref).max() < 64 * 2.0 ** -24 * 4


def test_scores_and_router_spec_exact_on_small_integers():
    qb = RNG.integers(-8, 9, size=(9, 16)).astype(np.float32)
    kb = RNG.integers(-8, 9, size=(11, 16)).astype(np.float32)
    Wt = RNG.integers(-4, 5, size=(16, 16)).astype(np.float32)
    np.testing.assert_array_equal(O.scores_f32_spec(qb, kb), (qb.astype(np.float64) @ kb.T.astype(np.float64)))
    np.testing.assert_array_equal(O.project_f32_spec(qb, Wt), qb.astype(np.float64) @ Wt.astype(np.float64))


def test_scores_spec_is_sequential_float32_order():
    # Non-integer case: the specified order accumulates k ascending from +0 with
    # separately rounded products; check against a scalar loop on a few entries.
    qb = RNG.standard_normal((4, 24)).astype(np.float32)
    kb = RNG.standard_normal((5, 24)).astype(np.float32)
    s = O.scores_f32_spec(qb, kb)
    for i in range(4):
        for j in range(5):
            acc = np.float32(0.0)
            for c in range(24):
                acc = np.float32(acc + np.float32(qb[i, c] * kb[j, c]))
            assert s[i, j] == acc


# ---------------------------------------------------------------------------
# classification
# ---------------------------------------------------------------------------

def brute_force_mask(s, kc, kn):
    R, Nb = s.shape
    Mc = np.zeros((R, Nb), dtype=np.int8)
    for i in range(R):
        for j in range(Nb):
            rank = sum(1 for jj in range(Nb) if s[i, jj] > s[i, j] or (s[i, jj] == s[i, j] and jj < j))
            if rank < kc:
                Mc[i, j] = 1
            elif rank >= Nb - kn:
                Mc[i, j] = -1
    return Mc


@pytest.mark.parametrize("kc,kn", [(1, 0), (3, 2), (5, 11), (16, 0), (0, 4), (12, 4)])
def test_classify_matches_rank_count_with_ties(kc, kn):
    s = RNG.integers(-3, 4, size=(20, 16)).astype(np.float32)  # many ties
    s[0] = 0.0
    s[1, ::2] = -0.0  # signed zeros compare equal
    Mc, crit, neg = O.classify(s, kc, kn)
    np.testing.assert_array_equal(Mc, brute_force_mask(s, kc, kn))
    for i in range(20):
        assert list(crit[i]) == sorted(np.nonzero(Mc[i] == 1)[0])
        assert list(neg[i]) == sorted(np.nonzero(Mc[i] == -1)[0])
    # all-equal row: lowest indices critical, highest negligible
    assert list(np.nonzero(Mc[0] == 1)[0]) == list(range(kc))
    assert list(np.nonzero(Mc[0] == -1)[0]) == list(range(16 - kn, 16))


def test_all_critical_and_constant_query():
    s = RNG.standard_normal((6, 10)).astype(np.float32)
    Mc, _, _ = O.classify(s, 10, 0)
    assert np.all(Mc == 1)
    s2 = np.broadcast_to(RNG.standard_normal(10).astype(np.float32), (6, 10))
    Mc2, _, _ = O.classify(np.array(s2), 3, 2)
    assert np.all(Mc2 == Mc2[0])


def test_spec_mask_agrees_with_exact_ranking_on_tiny_workload():
    w = W.WORKLOADS["sla_b1h2n1024d64"]
    inp = W.make_inputs(w)
    for h in range(w.H):
        r = O.forward_head(inp.q[0, h], inp.k[0, h], inp.v[0, h], w.N, variant="sla",
                           k_crit=w.k_crit, k_neg=w.k_neg, w_proj_bits=inp.w_proj,
                           with_f64_mask=True)
        for row, gaps in O.mask_disagreements(r, r["f64"], w.k_crit, w.k_neg):
            assert min(gaps) < 1e-4, (row, gaps)


def test_router_projection_commutes_with_pooling():
    x = RNG.standard_normal((64 * 4, 16))
    Wt = RNG.standard_normal((16, 16))
    N = 64 * 3 + 5
    np.testing.assert_allclose(O.pool_f64(x @ Wt, N), O.pool_f64(x, N) @ Wt, atol=1e-12)


# ---------------------------------------------------------------------------
# sparse branch
# ---------------------------------------------------------------------------

def rand_head(N, d, Np=None, scale=1.0):
    Np = Np or 64 * ((N + 63) // 64)
    x = (RNG.standard_normal((Np, d)) * scale).astype(np.float32)
    return W.bf16_bits_to_f32(bits(x)).astype(np.float64)


def test_sparse_all_critical_is_exact_softmax_attention():
    import torch

    N, d = 200, 16
    q, k, v = rand_head(N, d, scale=2.0), rand_head(N, d, scale=2.0), rand_head(N, d)
    Nb = q.shape[0] // 64
    Mc = np.ones((Nb, Nb), dtype=np.int8)
    scale = 1 / math.sqrt(d)
    got = O.sparse_branch(q, k, v, Mc, N, scale)
    # textbook dense softmax attention, full N x N
    S = q[:N] @ k[:N].T * scale
    P = np.exp(S - S.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(got, P @ v[:N], atol=1e-12)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a[:N]))[None, None]  # noqa: E731
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v))[0, 0].numpy()
    np.testing.assert_allclose(got, ref, atol=1e-12)


def test_sparse_branch_masks_exactly_the_noncritical_blocks():
    N, d = 64 * 4, 8
    q, k, v = rand_head(N, d), rand_head(N, d), rand_head(N, d)
    Mc = np.array([[1, 0, -1, 1], [0, 0, 1, 0], [1, 1, 1, 1], [-1, 0, 0, 1]], dtype=np.int8)
    got = O.sparse_branch(q, k, v, Mc, N, 0.3)
    for r in range(N):
        i = r // 64
        keys = [t for t in range(N) if Mc[i, t // 64] == 1]
        s = np.array([q[r] @ k[t] * 0.3 for t in keys])
        p = np.exp(s - s.max())
        want = (p[:, None] * v[keys]).sum(0) / p.sum()
        np.testing.assert_allclose(got[r], want, atol=1e-12)


# ---------------------------------------------------------------------------
# linear branch
# ---------------------------------------------------------------------------

def brute_force_linear(q, k, v, Mc, N, phi_kind="softmax"):
    pq, pk = O.phi(q[:N], phi_kind), O.phi(k[:N], phi_kind)
    out = np.zeros((N, v.shape[1]))
    for r in range(N):
        i = r // 64
        num = np.zeros(v.shape[1])
        den = 0.0
        for t in range(N):
            if Mc[i, t // 64] == 0:
                wgt = float(pq[r] @ pk[t])
                num += wgt * v[t]
                den += wgt
        out[r] = num / den if den > 0 else 0.0
    return out


@pytest.mark.parametrize("phi_kind", ["softmax", "elu1"])
def test_linear_branch_matches_token_level_brute_force(phi_kind):
    N, d = 64 * 3 + 17, 12
    q, k, v = rand_head(N, d, scale=2), rand_head(N, d, scale=2), rand_head(N, d)
    Mc = np.array([[1, 0, -1, 0], [0, 0, 0, 0], [1, 1, 1, 0], [-1, 1, 1, 1]], dtype=np.int8)
    got = O.linear_branch(q, k, v, Mc, N, phi_kind)
    np.testing.assert_allclose(got, brute_force_linear(q, k, v, Mc, N, phi_kind), atol=1e-12)
    assert np.all(got[3 * 64:N] == 0.0)  # row 3 has no marginal block


def test_no_critical_block_gives_pure_linear_attention():
    # SLA with W = I and an empty critical set: O is linear attention over the
    # non-negligible blocks; with k_neg = 0, over every token.
    N, d = 64 * 4, 8
    qb, kb, vb = bits(rand_head(N, d, scale=2)), bits(rand_head(N, d, scale=2)), bits(rand_head(N, d))
    eye = bits(np.eye(d))
    for kn in (0, 1):
        r = O.forward_head(qb, kb, vb, N, variant="sla", k_crit=0, k_neg=kn, w_proj_bits=eye)
        q, k, v = (W.bf16_bits_to_f32(b).astype(np.float64) for b in (qb, kb, vb))
        np.testing.assert_allclose(r["O"], brute_force_linear(q, k, v, r["Mc"], N), atol=1e-12)
        assert np.all(r["O_s"] == 0)
    # k_neg = 0: every block marginal, plain linear attention over all tokens
    pq, pk = O.phi(q), O.phi(k)
    A = pq @ pk.T
    r0 = O.forward_head(qb, kb, vb, N, variant="sla", k_crit=0, k_neg=0, w_proj_bits=eye)
    np.testing.assert_allclose(r0["O"], (A @ v) / A.sum(1, keepdims=True), atol=1e-12)


def test_elu1_forward_without_critical_blocks_is_plain_linear_attention():
    # the same identity with phi = elu + 1: every block marginal, W = I, so O is
    # kernelised linear attention with k(q, k) = phi(q) . phi(k) over all tokens
    N, d = 64 * 4 + 9, 8
    qb, kb, vb = bits(rand_head(N, d, scale=2)), bits(rand_head(N, d, scale=2)), bits(rand_head(N, d))
    r = O.forward_head(qb, kb, vb, N, variant="sla", k_crit=0, k_neg=0, w_proj_bits=bits(np.eye(d)),
                       phi_kind="elu1")
    q, k, v = (W.bf16_bits_to_f32(b)[:N].astype(np.float64) for b in (qb, kb, vb))
    eq = np.where(q > 0, q + 1, np.exp(np.minimum(q, 0)))
    ek = np.where(k > 0, k + 1, np.exp(np.minimum(k, 0)))
    A = eq @ ek.T
    np.testing.assert_allclose(r["O"], (A @ v) / A.sum(1, keepdims=True), atol=1e-12)


def test_sla2_alpha_extremes_and_empty_marginal():
    N, d = 64 * 3, 16
    qb, kb, vb = bits(rand_head(N, d, scale=2)), bits(rand_head(N, d, scale=2)), bits(rand_head(N, d))
    full = O.forward_head(qb, kb, vb, N, variant="sla2", k_crit=3, k_neg=0, alpha_h=1.0)
    q, k, v = (W.bf16_bits_to_f32(b).astype(np.float64) for b in (qb, kb, vb))
    S = q @ k.T / math.sqrt(d)
    P = np.exp(S - S.max(1, keepdims=True))
    np.testing.assert_allclose(full["O"], (P / P.sum(1, keepdims=True)) @ v, atol=1e-12)
    assert np.all(full["O_l"] == 0)  # no marginal block
    zero = O.forward_head(qb, kb, vb, N, variant="sla2", k_crit=1, k_neg=0, alpha_h=0.0)
    np.testing.assert_allclose(zero["O"], zero["O_l"], atol=0)


def test_branch_outputs_are_convex_combinations_of_v():
    w = W.WORKLOADS["sla_b1h2n1024d64"]
    inp = W.make_inputs(w)
    r = O.forward_head(inp.q[0, 0], inp.k[0, 0], inp.v[0, 0], w.N, variant="sla",
                       k_crit=w.k_crit, k_neg=w.k_neg, w_proj_bits=inp.w_proj)
    v = W.bf16_bits_to_f32(inp.v[0, 0])[:w.N].astype(np.float64)
    for name, label in (("O_s", 1), ("O_l", 0)):
        for i in range(w.Nb):
            blocks = np.nonzero(r["Mc"][i] == label)[0]
            rows = np.concatenate([v[j * 64:(j + 1) * 64] for j in blocks])
            o = r[name][i * 64:(i + 1) * 64]
            assert np.all(o <= rows.max(0) + 1e-12) and np.all(o >= rows.min(0) - 1e-12)


def test_padding_rows_do_not_matter():
    w = W.make_workload("pad", 1, 1, 64 * 5 + 9, 32, "sla", k_crit=2, k_neg=1, seed=9)
    outs = []
    for pad in (64.0, 0.0, float("nan"), -3e4):
        inp = W.make_inputs(w.replace(pad_value=pad))
        outs.append(O.forward(inp)[(0, 0)])
    for o in outs[1:]:
        np.testing.assert_array_equal(o["Mc"], outs[0]["Mc"])
        np.testing.assert_array_equal(o["O"], outs[0]["O"])
        assert np.isfinite(o["O"]).all()


# ---------------------------------------------------------------------------
# quantisation helpers
# ---------------------------------------------------------------------------

def e4m3_grid():
    """All finite non-negative e4m3 values, from the format's definition."""
    vals = [m * 2.0 ** -9 for m in range(8)]  # subnormals (exponent field 0)
    for e in range(1, 16):
        for m in range(8):
            if e == 15 and m == 7:
                continue  # the NaN code
            vals.append((1 + m / 8) * 2.0 ** (e - 7))
    return np.array(sorted(vals))


def test_e4m3_round_is_nearest_even_on_the_grid():
    grid = e4m3_grid()
    assert grid[-1] == 448.0 and grid[8] == 2.0 ** -6
    x = np.concatenate([RNG.standard_normal(20000) * 10.0 ** RNG.uniform(-4, 2.5, 20000), grid, -grid,
                        (grid[1:] + grid[:-1]) / 2, [500.0, -1e6]])
    y = O.e4m3_round(x)
    a = np.abs(x)
    assert np.all(np.isin(np.abs(y), grid))
    # nearest: no grid point is strictly closer
    idx = np.clip(np.searchsorted(grid, np.minimum(a, 448.0)), 1, grid.size - 1)
    best = np.minimum(np.abs(grid[idx] - np.minimum(a, 448.0)), np.abs(grid[idx - 1] - np.minimum(a, 448.0)))
    assert np.all(np.abs(np.abs(y) - np.minimum(a, 448.0)) <= best + 0.0)
    assert np.all(np.abs(O.e4m3_round([500.0, -1e6])) == 448.0)
    # ties go to the even code (mantissa lsb 0): 1 + 1/16 lies between 1 and 1.125
    assert O.e4m3_round([1.0 + 1 / 16, 1.0 + 3 / 16])[0] == 1.0
    assert O.e4m3_round([1.0 + 3 / 16])[0] == 1.25


def test_e4m3_round_matches_torch_float8():
    import torch

    x = RNG.standard_normal(50000) * 10.0 ** RNG.uniform(-5, 2.6, 50000)
    x = x[np.abs(x) <= 448.0].astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.e4m3_round(x.astype(np.float64)), ref)


def test_int8_block_quantisation_bounds():
    N = 64 * 2 + 30
    x = (RNG.standard_normal((64 * 3, 16)) * 3).astype(np.float32)
    codes, s = O.quantize_int8_blocks(x, N)
    n = O.valid_rows(N, 3)
    for i in range(3):
        blk = x[i * 64:i * 64 + n[i]].astype(np.float64)
        c = codes[i * 64:i * 64 + n[i]].astype(np.float64)
        assert np.abs(c).max() == 127
        assert np.all(np.abs(blk - c * s[i]) <= s[i] / 2 * (1 + 1e-6))
    assert np.all(codes[N:] == 0)


def test_quantized_branch_exact_when_inputs_sit_on_the_grids():
    # Q, K integer-valued with block absmax 127 (INT8 scale exactly 1), keys
    # equal inside each block, V on the e4m3 grid with block absmax 448 (scale
    # 1, r_j = 1): every quantisation step is exact except P's. A row's scores
    # on its critical block are all equal to x (log2 units), so every P~ of the
    # row is c = 2^(x - ceil x) and every P code is e4m3(256 c): the branch is
    # the float64 sparse branch times e4m3(256 c) / (256 c), row by row.
    rng = np.random.default_rng(2024)  # own stream: independent of test order
    d, N = 8, 128
    q = rng.integers(-20, 21, size=(N, d)).astype(np.float32)
    q[0, 0] = 127
    q[64, 3] = -127
    k = np.zeros((N, d), dtype=np.float32)
    k[:64] = [127, 3, 0, 0, 0, 0, 0, 0]
    k[64:] = [-127, 5, 1, 0, 0, 0, 0, 0]
    grid = e4m3_grid()
    v = (rng.choice(grid[grid <= 448], size=(N, d)) * rng.choice([-1, 1], size=(N, d))).astype(np.float32)
    v[0, 0] = 448.0
    v[64, 1] = -448.0
    qb, kb, vb = bits(q), bits(k), bits(v)
    r = O.forward_head(qb, kb, vb, N, variant="sla2", k_crit=1, k_neg=0, alpha_h=1.0, quantized=True)
    assert (r["Mc"] == 1).sum() == 2
    crit_block = np.argmax(r["Mc"] == 1, axis=1)
    s = np.array([q[i].astype(np.float64) @ k[64 * crit_block[i // 64]] for i in range(N)])
    x = s / math.sqrt(d) / math.log(2.0)
    c = 2.0 ** (x - np.ceil(x))
    assert np.all((c > 0.5) & (c <= 1.0))
    factor = O.e4m3_round(256.0 * c) / (256.0 * c)
    assert np.any(factor != 1.0)  # the P step is really exercised
    # float64 rounding of the two sides only (one e4m3 step is 2^-4 relative)
    np.testing.assert_allclose(r["O_sq"], r["O_s"] * factor[:, None], rtol=1e-10, atol=1e-12)


def test_int8_block_quantisation_ties_go_to_even():
    # block absmax 127 makes the scale exactly 1, so x / s = x and the codes are
    # rint(x): halves go to the even neighbour (round-half-away would give
    # 3, 4, -3, 1, -1, 2 here instead of 2, 4, -2, 0, 0, 2)
    x = np.zeros((64, 8), dtype=np.float32)
    x[0, 0] = 127.0
    x[1, :6] = [2.5, 3.5, -2.5, 0.5, -0.5, 1.5]
    codes, s = O.quantize_int8_blocks(x, 64)
    assert s[0] == np.float32(1.0)
    assert list(codes[1, :6]) == [2, 4, -2, 0, 0, 2]
    assert codes[0, 0] == 127


def test_quantized_branch_folds_each_blocks_v_scale_into_p():
    # As the grid test above, but the two key blocks' V scales differ by a
    # factor that is not a power of two (s_v = 1 and 0.75: block 1 holds 0.75
    # times e4m3 grid values, absmax 336), so the fold r_j = s_v,j / max s_v is
    # exercised: P of a row whose critical block is j enters as
    # e4m3(256 r_j c), and O^s_q = O^s e4m3(256 r_j c) / (256 r_j c). A fold
    # inverted (1 / r_j) or left out (r_j = 1) changes at least one row.
    rng = np.random.default_rng(77)
    d, N = 8, 128
    q = rng.integers(-20, 21, size=(N, d)).astype(np.float32)
    q[0, 0] = 127
    q[64, 3] = -127
    k = np.zeros((N, d), dtype=np.float32)
    k[:64] = [127, 3, 0, 0, 0, 0, 0, 0]
    k[64:] = [-127, 5, 1, 0, 0, 0, 0, 0]
    grid = e4m3_grid()
    g = rng.choice(grid[grid <= 448], size=(N, d)) * rng.choice([-1, 1], size=(N, d))
    g[0, 0], g[64, 1] = 448.0, -448.0
    v = g.copy()
    v[64:] *= 0.75  # exact in float32: grid values have at most 4 significant bits
    v = v.astype(np.float32)
    r = O.forward_head(bits(q), bits(k), bits(v), N, variant="sla2", k_crit=1, k_neg=0, alpha_h=1.0,
                       quantized=True)
    _, sv = O.quantize_e4m3_blocks(O.bf16_to_f32(bits(v)), N)
    assert list(sv) == [1.0, 0.75]
    crit_block = np.argmax(r["Mc"] == 1, axis=1)
    assert set(crit_block.tolist()) == {0, 1}  # both folds are used
    s = np.array([q[i].astype(np.float64) @ k[64 * crit_block[i // 64]] for i in range(N)])
    x = s / math.sqrt(d) / math.log(2.0)
    c = 2.0 ** (x - np.ceil(x))
    rj = np.array([1.0, 0.75])[crit_block[np.arange(N) // 64]]

    def factor(rr):
        return O.e4m3_round(256.0 * rr * c) / (256.0 * rr * c)

    np.testing.assert_allclose(r["O_sq"], r["O_s"] * factor(rj)[:, None], rtol=1e-10, atol=1e-12)
    assert np.any(factor(1.0 / rj) != factor(rj)) and np.any(factor(np.ones(N)) != factor(rj))


def test_e4m3_p_and_v_alone_exceed_the_low_bit_tolerance_on_the_14b_shape():
    # A finding about the low-bit scheme itself, not a check of the kernel.
    # With the scores computed exactly (no INT8 Q or K at all), e4m3 P (the
    # scheme's power-of-two row scale and V-scale fold) and e4m3 V alone move
    # the sparse branch by more than the 5e-2 max-abs tolerance stated for the
    # INT8 / FP8 branch on this workload's peaked rows: three mantissa bits
    # carry up to 2^-4 relative error per element, and a row dominated by a
    # few keys passes that error straight to its output. O = alpha O^s +
    # (1 - alpha) O^l, so O moves by alpha times as much.
    w = W.WORKLOADS["sla2_q_wan14b_b1h40n75600d128_s97"]
    inp = W.make_inputs(w, heads=[(0, 5)])
    q32, k32, v32 = (O.bf16_to_f32(x[0, 0]) for x in (inp.q, inp.k, inp.v))
    N = w.N
    m = O.mask_f32_spec(q32, k32, N, w.k_crit, 0, O.bf16_to_f32(inp.proj_q), O.bf16_to_f32(inp.proj_k))
    vq, sv = O.quantize_e4m3_blocks(v32, N)
    q, k, v = (x.astype(np.float64) for x in (q32, k32, v32))
    scale = 1.0 / math.sqrt(w.d)
    errs, refs = [], []
    for i in range(0, w.Nb, 30):  # 40 of the 1182 query blocks
        r0, r1 = i * 64, min(N, (i + 1) * 64)
        keys = O._block_tokens(np.nonzero(m["Mc"][i] == 1)[0], N)
        x = (q[r0:r1] @ k[keys].T) * scale * O.LOG2E
        p = np.exp2(x - np.ceil(x.max(axis=1, keepdims=True)))
        exact = (p @ v[keys]) / p.sum(axis=1, keepdims=True)
        rj = (sv[keys // 64] / np.float32(sv.max())).astype(np.float64)
        pq = O.e4m3_round(p * rj[None, :] * 256.0)
        low = (pq @ vq[keys]) * (float(sv.max()) / 256.0) / p.sum(axis=1, keepdims=True)
        errs.append(low - exact)
        refs.append(exact)
    e, ref = np.concatenate(errs), np.concatenate(refs)
    alpha = float(inp.alpha[5])
    assert alpha * np.abs(e).max() > 5e-2
    assert np.linalg.norm(e) / np.linalg.norm(ref) > 3e-2


def test_quantized_sparse_branch_error_is_quantisation_sized():
    # Diagnostic scale only: on the tiny workload (128 critical keys per row)
    # the low-bit branch stays within a few percent of the exact branch.
    w = W.WORKLOADS["sla_b1h2n1024d64"]
    inp = W.make_inputs(w)
    r = O.forward_head(inp.q[0, 1], inp.k[0, 1], inp.v[0, 1], w.N, variant="sla",
                       k_crit=w.k_crit, k_neg=w.k_neg, w_proj_bits=inp.w_proj, quantized=True)
    err = r["O_sq"] - r["O_s"]
    assert 0 < np.linalg.norm(err) / np.linalg.norm(r["O_s"]) < 0.1


# ---------------------------------------------------------------------------
# SoftTop-k router
# ---------------------------------------------------------------------------

def test_soft_topk_uniform_row_closed_form():
    # every entry equal: each M_ij = k / n and lambda = c - tau log(k / (n - k))
    for n, k, tau, c in [(16, 3, 0.05, 0.0625), (512, 25, 1e-3, 1.0 / 512), (7, 6, 2.0, -3.0)]:
        M, lam = O.soft_topk(np.full((2, n), c), k, tau)
        np.testing.assert_allclose(M, k / n, rtol=1e-12)
        np.testing.assert_allclose(lam, c - tau * math.log(k / (n - k)), rtol=1e-12, atol=1e-15)


def test_soft_topk_two_entries_root_is_the_midpoint():
    # n = 2, k = 1: sigmoid(a) + sigmoid(-a) = 1 puts lambda halfway between the entries
    P = np.array([[0.9, 0.1], [0.25, 0.75], [0.5, 0.5]])
    for tau in (0.01, 0.3, 5.0):
        M, lam = O.soft_topk(P, 1, tau)
        np.testing.assert_allclose(lam, P.mean(axis=1), rtol=1e-13)
        want = 1.0 / (1.0 + np.exp(-(P[:, 0] - P[:, 1]) / (2 * tau)))
        np.testing.assert_allclose(M[:, 0], want, rtol=1e-12)
        np.testing.assert_allclose(M.sum(axis=1), 1.0, rtol=1e-13)


def test_soft_topk_root_matches_brentq():
    from scipy.optimize import brentq
    from scipy.special import expit

    rng = np.random.default_rng(77)
    for n, k, tau in [(64, 3, 0.02), (300, 40, 1e-3), (33, 32, 0.5)]:
        P = rng.dirichlet(np.full(n, 0.3), size=4)
        M, lam = O.soft_topk(P, k, tau)
        for r in range(P.shape[0]):
            root = brentq(lambda x: expit((P[r] - x) / tau).sum() - k, -10.0, 10.0, xtol=1e-15, rtol=1e-15)
            assert lam[r] == pytest.approx(root, rel=1e-10, abs=1e-13)
        np.testing.assert_allclose(M.sum(axis=1), k, rtol=1e-10)
        assert np.all((M >= 0) & (M <= 1))


def test_soft_topk_small_temperature_is_the_hard_topk():
    # distinct entries, gaps far above tau: the soft mask is the Top-k indicator
    rng = np.random.default_rng(5)
    n, k = 40, 6
    P = np.stack([rng.permutation(n) for _ in range(5)]).astype(np.float64) / n
    M, _ = O.soft_topk(P, k, 1e-4)
    Mc, _, _ = O.classify(P, k, 0)
    np.testing.assert_allclose(M, (Mc == 1).astype(np.float64), atol=1e-9)


def test_soft_topk_shift_and_scale():
    rng = np.random.default_rng(9)
    P = rng.random((3, 50))
    M, lam = O.soft_topk(P, 7, 0.05)
    M2, lam2 = O.soft_topk(P + 0.375, 7, 0.05)
    np.testing.assert_allclose(M2, M, atol=1e-12)
    np.testing.assert_allclose(lam2, lam + 0.375, rtol=1e-12)
    M3, lam3 = O.soft_topk(4.0 * P, 7, 0.2)
    np.testing.assert_allclose(M3, M, atol=1e-12)
    np.testing.assert_allclose(lam3, 4.0 * lam, rtol=1e-12)


def test_soft_topk_every_block_selected():
    M, lam = O.soft_topk(np.random.default_rng(2).random((2, 9)), 9, 0.1)
    assert np.all(M == 1.0) and np.all(np.isneginf(lam))


def test_router_pc_is_scaled_softmax_of_pooled_scores():
    # integer block means pool exactly; Pc = softmax(qbar kbar^T / sqrt(d)) per row
    from scipy.special import softmax

    rng = np.random.default_rng(21)
    Nb, d = 6, 16
    qm = rng.integers(-2, 3, size=(Nb, d)).astype(np.float32)
    km = rng.integers(-2, 3, size=(Nb, d)).astype(np.float32)
    q = np.repeat(qm, 64, axis=0)
    k = np.repeat(km, 64, axis=0)
    r = O.router_soft_topk_head(bits(q), bits(k), Nb * 64, 2, 0.05)
    s = qm.astype(np.float64) @ km.T.astype(np.float64)
    np.testing.assert_array_equal(r["scores"], s)
    np.testing.assert_allclose(r["Pc"], softmax(s / 4.0, axis=1), rtol=1e-13)
    np.testing.assert_allclose(r["M"].sum(axis=1), 2.0, rtol=1e-10)
    # the router projections act on the pooled vectors
    Wq = np.eye(d, dtype=np.float32)[::-1].copy()  # reverse the features of qbar
    r2 = O.router_soft_topk_head(bits(q), bits(k), Nb * 64, 2, 0.05, bits(Wq), bits(np.eye(d, dtype=np.float32)))
    np.testing.assert_array_equal(r2["scores"], qm[:, ::-1].astype(np.float64) @ km.T.astype(np.float64))


# ---------------------------------------------------------------------------
# backward pass
# ---------------------------------------------------------------------------

def _bwd_case(variant, phi_kind, N=64 * 4 + 9, d=8, kc=2, kn=1, seed=0):
    rng = np.random.default_rng(seed)
    Np = 64 * ((N + 63) // 64)
    q, k, v = (rng.standard_normal((Np, d)) for _ in range(3))
    Nb = Np // 64
    Mc, _, _ = O.classify(rng.standard_normal((Nb, Nb)), kc, kn if variant == "sla" else 0)
    W = rng.standard_normal((d, d)) / math.sqrt(d)
    alpha = 0.7
    do = rng.standard_normal((N, d))
    return q, k, v, Mc, W, alpha, do


def _forward_fixed_mask(q, k, v, Mc, N, variant, W, alpha, phi_kind):
    scale = 1.0 / math.sqrt(q.shape[1])
    o_s = O.sparse_branch(q, k, v, Mc, N, scale)
    o_l = O.linear_branch(q, k, v, Mc, N, phi_kind)
    return O.combine_sla(o_s, o_l, W) if variant == "sla" else O.combine_sla2(o_s, o_l, alpha)


@pytest.mark.parametrize("variant", ["sla", "sla2"])
@pytest.mark.parametrize("phi_kind", ["softmax", "elu1"])
def test_backward_matches_central_differences(variant, phi_kind):
    N = 64 * 4 + 9
    q, k, v, Mc, W, alpha, do = _bwd_case(variant, phi_kind, N)
    scale = 1.0 / math.sqrt(q.shape[1])
    g = O.backward_f64(q, k, v, Mc, do, N, variant=variant, scale=scale, W=W, alpha_h=alpha, phi_kind=phi_kind)
    loss = lambda q_, k_, v_, W_, a_: float((do * _forward_fixed_mask(q_, k_, v_, Mc, N, variant, W_, a_,  # noqa: E731
                                                                       phi_kind)).sum())
    rng = np.random.default_rng(11)
    eps = 1e-5
    for name, grad in (("q", g["dQ"]), ("k", g["dK"]), ("v", g["dV"])):
        delta = np.zeros_like(q)
        delta[:N] = rng.standard_normal((N, q.shape[1]))
        args = dict(q=q, k=k, v=v)
        plus = dict(args, **{name: args[name] + eps * delta})
        minus = dict(args, **{name: args[name] - eps * delta})
        fd = (loss(plus["q"], plus["k"], plus["v"], W, alpha) - loss(minus["q"], minus["k"], minus["v"], W, alpha)) / (2 * eps)
        an = float((grad * delta[:N]).sum())
        assert an == pytest.approx(fd, rel=1e-6, abs=1e-8), name
    if variant == "sla":
        dW = rng.standard_normal(W.shape)
        fd = (loss(q, k, v, W + eps * dW, alpha) - loss(q, k, v, W - eps * dW, alpha)) / (2 * eps)
        assert float((g["dW"] * dW).sum()) == pytest.approx(fd, rel=1e-7, abs=1e-9)
    else:
        fd = (loss(q, k, v, W, alpha + eps) - loss(q, k, v, W, alpha - eps)) / (2 * eps)
        assert g["dalpha"] == pytest.approx(fd, rel=1e-7, abs=1e-9)


@pytest.mark.parametrize("variant,phi_kind,kc,kn", [("sla", "softmax", 2, 1), ("sla2", "softmax", 3, 0),
                                                    ("sla", "elu1", 1, 2), ("sla", "softmax", 5, 0)])
def test_backward_matches_autograd_of_token_level_formulation(variant, phi_kind, kc, kn):
    """Independent formulation: masked dense softmax over critical keys and the
    token-level linear attention sum_t phi(q).phi(k_t) v_t / sum_t phi(q).phi(k_t)
    over marginal keys, differentiated by torch.autograd in float64."""
    import torch

    N = 64 * 4 + 9
    q, k, v, Mc, W, alpha, do = _bwd_case(variant, phi_kind, N, kc=kc, kn=kn, seed=5)
    d = q.shape[1]
    g = O.backward_f64(q, k, v, Mc, do, N, variant=variant, scale=1.0 / math.sqrt(d), W=W, alpha_h=alpha,
                       phi_kind=phi_kind)
    blk = np.arange(N) // 64
    crit_tok = torch.from_numpy(Mc[blk][:, blk] == 1)
    marg_tok = torch.from_numpy(Mc[blk][:, blk] == 0).double()
    T = lambda a: torch.tensor(a[:N], dtype=torch.float64, requires_grad=True)  # noqa: E731
    tq, tk, tv = T(q), T(k), T(v)
    tW = torch.tensor(W, requires_grad=True)
    ta = torch.tensor(alpha, dtype=torch.float64, requires_grad=True)
    s = (tq @ tk.T) / math.sqrt(d)
    p = torch.softmax(s.masked_fill(~crit_tok, float("-inf")), dim=1)
    o_s = torch.nan_to_num(p) @ tv
    f = (lambda x: torch.softmax(x, dim=1)) if phi_kind == "softmax" else (lambda x: torch.where(x > 0, x + 1, torch.exp(torch.clamp(x, max=0.0))))
    a = (f(tq) @ f(tk).T) * marg_tok
    den = a.sum(dim=1, keepdim=True)
    has = den > 0
    o_l = torch.where(has, (a @ tv) / torch.where(has, den, torch.ones_like(den)), torch.zeros_like(o_s))
    o = o_s + o_l @ tW if variant == "sla" else ta * o_s + (1 - ta) * o_l
    (o * torch.from_numpy(do)).sum().backward()
    np.testing.assert_allclose(g["dQ"], tq.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(g["dK"], tk.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(g["dV"], tv.grad.numpy(), rtol=1e-9, atol=1e-11)
    if variant == "sla":
        np.testing.assert_allclose(g["dW"], tW.grad.numpy(), rtol=1e-10, atol=1e-12)
    else:
        assert g["dalpha"] == pytest.approx(float(ta.grad), rel=1e-10)


def test_backward_all_critical_is_softmax_attention_gradient():
    """Every block critical (no linear branch): the gradients are those of exact
    softmax attention, here torch's scaled_dot_product_attention in float64."""
    import torch

    N, d = 64 * 3, 16
    rng = np.random.default_rng(8)
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    Mc = np.ones((3, 3), dtype=np.int8)
    do = rng.standard_normal((N, d))
    g = O.backward_f64(q, k, v, Mc, do, N, variant="sla2", scale=1.0 / math.sqrt(d), alpha_h=1.0)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq[None], tk[None], tv[None])[0]
    (o * torch.from_numpy(do)).sum().backward()
    for name, got, want in (("q", g["dQ"], tq.grad), ("k", g["dK"], tk.grad), ("v", g["dV"], tv.grad)):
        np.testing.assert_allclose(got, want.numpy(), rtol=1e-9, atol=1e-11, err_msg=name)
    assert np.isfinite(g["lse"]).all()
    np.testing.assert_allclose(g["lse"], np.log(np.exp(q @ k.T / math.sqrt(d)).sum(axis=1)), rtol=1e-12)
