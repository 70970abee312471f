"""GPU parity of the quantised sparse branch (INT8 Q, K; FP8 e4m3 P, V) against
the oracle's emulation of the same scheme.

Quantisation stage (SLA2 article, section 3.3, sparse + low-bit attention):
the INT8 codes and per-block scales of Q and K and the e4m3 codes and scales
of V are compared bit for bit with the oracle's quantize_int8_blocks /
quantize_e4m3_blocks. The mask is bit-exact as on the bf16 path. The output is
compared with O_q, the oracle's float64 emulation of the low-bit sparse branch
combined with the float64 linear branch. The kernel's P codes are the
emulation's shifted by a power of two (integer row max), except where the fp32
exponent and ex2.approx put a P value on the other side of an e4m3 rounding
midpoint than the float64 one (a rare event per element, frequent over a
full-size head): that code moves by one e4m3 step. Small cases stay within the
bf16 output contract; the full-size case is held to the low-bit output
tolerance (5e-2 max-abs, 3e-2 rel-L2) against that emulation. Against the
exact (unquantised) output the scheme's own error is checked against a
diagnostic bound (rel-L2 < 0.1); the stated low-bit tolerance against the
unquantised output is a strict xfail: the scheme misses it on this workload
whatever the kernel does (see the oracle pin on e4m3 P and V).
"""

import numpy as np
import pytest

import workloads as W
from tests.gpu_helpers import MAX_ABS, REL_L2, assert_close, errors, oracle_head, oracle_mask_only, run_library

pytestmark = pytest.mark.gpu

PREC = "i8qk_f8pv"
# low-bit output tolerance against the emulation of the same scheme
Q_MAX_ABS, Q_REL_L2 = 5e-2, 3e-2
# the scheme's own distance to the exact output (INT8 Q/K dominate it)
SCHEME_REL_L2 = 0.1


def check_codes(sla, inp, res, idxs):
    from oracle import sla_oracle as O

    import torch

    qc, kc, vc, qs, ks, vs = (x.cpu() for x in sla.get_quantized(res["params"], res["ws"]))
    vc = vc.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    qc, kc, qs, ks, vs = qc.numpy(), kc.numpy(), qs.numpy(), ks.numpy(), vs.numpy()
    N = inp.w.N
    full = len(inp.heads) == inp.w.B * inp.w.H
    for idx in idxs:
        b, h = inp.heads[idx]
        sel = (b, h) if full else (idx, 0)
        want_qc, want_qs = O.quantize_int8_blocks(O.bf16_to_f32(inp.q[sel]), N)
        want_kc, want_ks = O.quantize_int8_blocks(O.bf16_to_f32(inp.k[sel]), N)
        want_v, want_vs = O.quantize_e4m3_blocks(O.bf16_to_f32(inp.v[sel]), N)
        np.testing.assert_array_equal(qc[sel], want_qc, err_msg=f"Q codes head {idx}")
        np.testing.assert_array_equal(kc[sel], want_kc, err_msg=f"K codes head {idx}")
        np.testing.assert_array_equal(vc[sel], want_v, err_msg=f"V e4m3 values head {idx}")
        np.testing.assert_array_equal(qs[sel], want_qs, err_msg=f"Q scales head {idx}")
        np.testing.assert_array_equal(ks[sel], want_ks, err_msg=f"K scales head {idx}")
        np.testing.assert_array_equal(vs[sel], want_vs, err_msg=f"V scales head {idx}")


def check_outputs(inp, res, idxs, record=None, max_abs=MAX_ABS, rel_l2=REL_L2):
    N = inp.w.N
    full = len(inp.heads) == inp.w.B * inp.w.H
    worst = []
    for idx in idxs:
        b, h = inp.heads[idx]
        sel = (b, h) if full else (idx, 0)
        r = oracle_head(inp, idx, quantized=True)
        np.testing.assert_array_equal(res["Mc"][sel], r["Mc"], err_msg=f"mask head {idx}")
        got = res["O"][sel][:N]
        assert_close(got, r["O_q"], max_abs, rel_l2, what=f"{inp.w.name} head {idx} vs emulated low-bit branch")
        ma, rl = errors(got, r["O"])
        assert rl < SCHEME_REL_L2, f"{inp.w.name} head {idx}: rel-L2 {rl:.3e} to the exact output"
        worst.append((ma, rl))
    if record is not None:
        record("max_abs_vs_exact", max(w[0] for w in worst))
        record("rel_l2_vs_exact", max(w[1] for w in worst))


SMALL = [
    # name, B, H, N, variant, k_crit, k_neg
    ("q_sla2_ragged", 1, 2, 64 * 12 + 13, "sla2", 2, 0),
    ("q_sla_ragged", 1, 2, 64 * 12 + 13, "sla", 3, 2),
    ("q_one_partial_block", 1, 2, 37, "sla2", 1, 0),
    ("q_one_full_block", 2, 1, 64, "sla", 1, 0),
    ("q_all_critical", 1, 2, 64 * 5 + 1, "sla", 6, 0),
    ("q_no_marginal", 1, 2, 64 * 6 + 50, "sla", 3, 4),
    ("q_two_batches_many_tiles", 2, 3, 64 * 37 + 63, "sla2", 5, 0),
    ("q_window_refill", 1, 1, 64 * 80 + 7, "sla", 40, 10),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_quantized_small(cuda_lib, case, record_property):
    name, B, H, N, variant, kc, kn = case
    w = W.make_workload(name, B, H, N, 128, variant, k_crit=kc, k_neg=kn, seed=31, precision=PREC)
    inp = W.make_inputs(w)
    res = run_library(cuda_lib, inp)
    assert res["status"] == 0
    idxs = list(range(B * H))
    check_codes(cuda_lib, inp, res, idxs)
    check_outputs(inp, res, idxs, record_property)


def test_quantized_phi_elu1(cuda_lib, record_property):
    # phi = elu + 1 with the low-bit sparse branch (the linear branch stays bf16)
    w = W.make_workload("q_elu1", 1, 2, 64 * 12 + 13, 128, "sla2", k_crit=2, k_neg=0, seed=33,
                        precision=PREC, phi="elu1")
    inp = W.make_inputs(w)
    res = run_library(cuda_lib, inp)
    assert res["status"] == 0
    check_codes(cuda_lib, inp, res, [0, 1])
    check_outputs(inp, res, [0, 1], record_property)


@pytest.fixture(scope="module")
def wan14b(cuda_lib):
    """One run of the 40-head, 75,600-token SLA2 workload at 97 % sparsity and
    the oracle (with the emulated low-bit branch) of heads 5 and 31."""
    w = W.WORKLOADS["sla2_q_wan14b_b1h40n75600d128_s97"]
    inp = W.make_inputs(w)
    res = run_library(cuda_lib, inp)
    refs = {idx: oracle_head(inp, idx, quantized=True) for idx in (5, 31)}
    return inp, res, refs


@pytest.mark.slow
def test_quantized_full_size_wan14b(cuda_lib, wan14b, record_property):
    """Codes and scales of every head, the mask of eight heads, the output of
    two against the emulation of the same low-bit scheme."""
    inp, res, refs = wan14b
    w = inp.w
    assert res["status"] == 0
    check_codes(cuda_lib, inp, res, range(w.B * w.H))
    for idx in (0, 7, 13, 19, 22, 28, 33, 39):
        m = oracle_mask_only(inp, idx)
        b, h = inp.heads[idx]
        np.testing.assert_array_equal(res["Mc"][b, h], m["Mc"], err_msg=f"mask head {idx}")
    check_outputs(inp, res, [5, 31], record_property, Q_MAX_ABS, Q_REL_L2)


@pytest.mark.slow
@pytest.mark.xfail(strict=True, reason=(
    "the low-bit scheme itself misses 5e-2 / 3e-2 against the unquantised output on this "
    "workload: e4m3 P and V alone, with exact scores, already exceed it (oracle pin "
    "test_e4m3_p_and_v_alone_exceed_the_low_bit_tolerance_on_the_14b_shape); measured "
    "about 0.24 max-abs and 5 % rel-L2 for the whole scheme"))
def test_quantized_full_size_wan14b_meets_low_bit_tolerance_vs_unquantised_oracle(wan14b, record_property):
    """The stated INT8 / FP8 tolerance (max-abs 5e-2, rel-L2 3e-2) against the
    unquantised float64 output. Strict xfail: if a scheme ever meets it, this
    test reports XPASS as a failure so the expectation gets updated."""
    inp, res, refs = wan14b
    N = inp.w.N
    worst = (0.0, 0.0)
    for idx, r in refs.items():
        b, h = inp.heads[idx]
        ma, rl = errors(res["O"][b, h][:N], r["O"])
        worst = (max(worst[0], ma), max(worst[1], rl))
    record_property("max_abs_vs_unquantised", worst[0])
    record_property("rel_l2_vs_unquantised", worst[1])
    assert worst[0] <= Q_MAX_ABS and worst[1] <= Q_REL_L2, worst
