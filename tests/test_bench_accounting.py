"""The benchmark's work accounting, checked against identities that hold
independently of its formulas (CPU only)."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads as W  # noqa: E402


def all_critical(N=64 * 16, H=3, d=128, variant="sla2"):
    Nb = N // 64
    return W.make_workload("acc", 1, H, N, d, variant, k_crit=Nb, k_neg=0, seed=0)


def test_all_critical_sparse_work_is_dense_attention():
    # every (query block, key block) pair critical: 4 B H N^2 d, the dense count
    w = all_critical()
    sparse, rest = bench.attention_split_flops(w)
    assert sparse == pytest.approx(bench.dense_eq_flops(w), rel=1e-15)
    assert rest == 0.0  # no marginal block: no linear branch; SLA2: no projection


def test_backward_of_dense_attention_is_two_and_a_half_forwards():
    # the attention backward takes five products of the forward's two
    w = all_critical()
    assert bench.backward_flops(w) == pytest.approx(2.5 * bench.dense_eq_flops(w), rel=1e-15)


def test_pair_tiles_issue_twice_the_sparse_work():
    # M = 128 pair tiles compute both query blocks' scores against both key
    # blocks: executed sparse work is twice the algorithmic one (Nb even)
    w = all_critical()
    assert bench.executed_flops(w) == pytest.approx(2 * bench.attention_split_flops(w)[0], rel=1e-15)


def test_linear_and_projection_terms():
    w = W.WORKLOADS["sla_wan13b_b1h12n32768d128_s95"]
    BH, N, d = w.B * w.H, w.N, w.d
    sparse, rest = bench.attention_split_flops(w)
    assert rest == pytest.approx(2 * (2.0 * BH * N * d * d), rel=1e-15)  # phi(Q) H and O^l W
    w2 = W.WORKLOADS["sla2_b1h12n32768d128_s97"]
    assert bench.attention_split_flops(w2)[1] == pytest.approx(2.0 * BH * N * d * d, rel=1e-15)
    # the correction: one d x d x 64 product per excluded (query block, key block) pair
    assert bench.correction_flops(w) == pytest.approx(BH * w.Nb * (w.k_crit + w.k_neg) * 4.0 * 64 * 64 * d)


def test_job_value_counts_every_rank():
    w = W.WORKLOADS["sla_b1h2n1024d64"]
    assert bench.job_value(w, 4, 2.0) == pytest.approx(4 * bench.job_value(w, 1, 2.0))


def test_attention_tile_traffic_follows_the_load_schedule():
    # per CTA of two query blocks, in 16 KB tiles (64 rows x d = 128 bf16):
    # SLA 95 %: Q pair 2 + 25 critical steps x (K, V, phi(K) pairs) 6 + 51 negligible
    # steps x (phi(K), V pairs) 4 + W (128 x 128 bf16 = 2 tiles) = 358
    w = W.WORKLOADS["sla_wan13b_b1h12n32768d128_s95"]
    ctas = w.B * w.H * w.Nb // 2
    assert bench.attention_tile_bytes(w) == ctas * 358 * 16384
    # SLA2 97 %: Q pair 2 + 15 x 6 + the precomputed phi(Q) pair 2 = 94
    w2 = W.WORKLOADS["sla2_b1h12n32768d128_s97"]
    assert bench.attention_tile_bytes(w2) == ctas * 94 * 16384
    assert bench.attention_tile_bytes(W.WORKLOADS["sla2_q_wan14b_b1h40n75600d128_s97"]) is None
    f = bench.l2_fill(w, 1.0, {"sm_mhz": 1000.0}, 100)
    assert f["B_per_cycle_per_SM"] == pytest.approx(bench.attention_tile_bytes(w) / (1e-3 * 1e9 * 100), rel=1e-3)
    assert bench.l2_fill(w, 1.0, None, 100)["frac"] is None
