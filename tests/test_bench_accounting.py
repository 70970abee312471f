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
