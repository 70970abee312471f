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
    # the correction: one d x 64 x d product per excluded (query block, key block) pair
    assert bench.correction_flops(w) == pytest.approx(BH * w.Nb * (w.k_crit + w.k_neg) * 2.0 * 64 * d * d)
    w64 = W.make_workload("c64", 1, 2, 64 * 20, 64, "sla", k_crit=2, k_neg=3, seed=0)
    assert bench.correction_flops(w64) == pytest.approx(2 * 20 * 5 * 2.0 * 64 * 64 * 64)
    assert bench.correction_flops(all_critical()) == 0.0  # no marginal block, no H_i


def test_useful_work_of_the_sla2_97_workload():
    # sparse pairs 12 heads x 512 blocks x 15 x 4 x 64 x 64 x 128 = 1.933e11, the
    # complement as much again (d = 128), phi(Q) H 2 N d^2 per head = 1.29e10
    w = W.WORKLOADS["sla2_b1h12n32768d128_s97"]
    sparse = 12 * 512 * 15 * 4.0 * 64 * 64 * 128
    assert bench.useful_flops(w) == pytest.approx(2 * sparse + 12 * 2.0 * 32768 * 128 * 128, rel=1e-12)
    # issued work adds the masked halves: the sparse pairs and phi(Q) H twice, the complement once
    assert bench.executed_flops(w) == pytest.approx(3 * sparse + 2 * 12 * 2.0 * 32768 * 128 * 128, rel=1e-12)


def test_launch_count_per_forward():
    # pool, scores, classify, phi(K)/h/z, reduction, attention; + Z_i when precomputed
    assert bench.forward_launches(W.WORKLOADS["sla_wan13b_b1h12n32768d128_s95"]) == 6  # 51 negligible
    assert bench.forward_launches(W.WORKLOADS["sla2_b1h12n32768d128_s97"]) == 7
    assert bench.forward_launches(W.WORKLOADS["sla2_q_wan14b_b1h40n75600d128_s97"]) == 7
    assert bench.forward_launches(all_critical()) == 6  # no linear branch


def test_peak_choice_follows_the_timed_region():
    pk = {"bf16_tflops": 1672.7, "bf16_tflops_sustained": 1414.8}
    assert bench.attention_peak(pk, "measured", 35.0)[0] == 1672.7
    assert bench.attention_peak(pk, "measured", 5000.0)[0] == 1414.8


def test_job_value_counts_every_rank():
    w = W.WORKLOADS["sla_b1h2n1024d64"]
    assert bench.job_value(w, 4, 2.0) == pytest.approx(4 * bench.job_value(w, 1, 2.0))


def test_attention_tile_traffic_follows_the_load_schedule():
    # per CTA of two query blocks, in 16 KB tiles (64 rows x d = 128 bf16):
    # SLA 95 %: Q pair 2 + 25 critical steps x (K, V, phi(K) pairs) 6 + 51 negligible
    # steps x (phi(K), V pairs) 4 + W and H_tot (128 x 128 bf16 = 2 tiles each) = 360
    w = W.WORKLOADS["sla_wan13b_b1h12n32768d128_s95"]
    ctas = w.B * w.H * w.Nb // 2
    assert bench.attention_tile_bytes(w) == ctas * 360 * 16384
    # SLA2 97 %: Q pair 2 + 15 x 6 + the precomputed phi(Q) pair 2 + H_tot 2 = 96
    w2 = W.WORKLOADS["sla2_b1h12n32768d128_s97"]
    assert bench.attention_tile_bytes(w2) == ctas * 96 * 16384
    assert bench.attention_tile_bytes(W.WORKLOADS["sla2_q_wan14b_b1h40n75600d128_s97"]) is None
    f = bench.l2_fill(w, 1.0, {"sm_mhz": 1000.0}, 100)
    assert f["B_per_cycle_per_SM"] == pytest.approx(bench.attention_tile_bytes(w) / (1e-3 * 1e9 * 100), rel=1e-3)
    assert bench.l2_fill(w, 1.0, None, 100)["frac"] is None
