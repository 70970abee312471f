"""C-ABI checks that need no GPU: the library builds and loads, exports every
function include/sla.h declares, and rejects bad arguments on the host before
anything is enqueued (fault injection on the host: null, misaligned and
undersized buffers, bad counts)."""

import ctypes
import os
import re

import pytest

import sparse_linear_attention_pool_b200 as sla
from sparse_linear_attention_pool_b200 import build as sla_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    sla_build.build()
    return sla.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "sla.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(sla_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "sla_forward" in names and "sla_dense_forward" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(sla.EXPORTS)


def test_abi_version_and_status_strings(lib):
    assert lib.sla_abi_version() == 5
    for s in range(8):
        assert sla.status_string(s)
    assert "unknown" in sla.status_string(99)


def params(**kw):
    base = dict(B=1, H=2, N=1000, d=128, variant="sla", k_crit=2, k_neg=1)
    base.update(kw)
    B, H, N, d = base.pop("B"), base.pop("H"), base.pop("N"), base.pop("d")
    return sla.make_params(B, H, N, d, **base)


@pytest.mark.parametrize("kw,code", [
    (dict(), sla.SLA_OK),
    (dict(d=96), sla.SLA_ERR_UNSUPPORTED),
    (dict(N=0), sla.SLA_ERR_INVALID_ARG),
    (dict(B=0), sla.SLA_ERR_INVALID_ARG),
    (dict(k_crit=0), sla.SLA_ERR_INVALID_ARG),
    (dict(k_crit=16, k_neg=1), sla.SLA_ERR_INVALID_ARG),   # Nb = 16
    (dict(k_crit=17, k_neg=0), sla.SLA_ERR_INVALID_ARG),
    (dict(k_crit=16, k_neg=0), sla.SLA_OK),
    (dict(k_neg=-1), sla.SLA_ERR_INVALID_ARG),
    (dict(N=262144 + 1), sla.SLA_ERR_UNSUPPORTED),
    (dict(softmax_scale=-1.0), sla.SLA_ERR_INVALID_ARG),
    (dict(softmax_scale=float("nan")), sla.SLA_ERR_INVALID_ARG),
    (dict(variant="sla2", k_neg=0), sla.SLA_ERR_INVALID_ARG),  # SLA2 needs alpha
    (dict(phi="elu1"), sla.SLA_OK),
])
def test_validate(lib, kw, code):
    assert sla.validate(params(**kw)) == code


def test_validate_rejects_unknown_phi(lib):
    p = params()
    for bad in (2, -1, 99):
        p.phi = bad
        assert sla.validate(p) == sla.SLA_ERR_INVALID_ARG
        assert lib.sla_workspace_size(ctypes.byref(p)) == 0


def test_bad_enum_and_block_size(lib):
    p = params()
    p.variant = 7
    assert sla.validate(p) == sla.SLA_ERR_INVALID_ARG
    p = params()
    p.block_q = 128
    assert sla.validate(p) == sla.SLA_ERR_UNSUPPORTED
    p = params()
    p.alpha = 0x1000
    p.variant = 1
    p.k_neg = 0
    p.proj_q = 0x2000  # proj_q without proj_k
    assert sla.validate(p) == sla.SLA_ERR_INVALID_ARG


def test_workspace_size(lib):
    assert sla.workspace_size(params()) > 0
    assert lib.sla_workspace_size(ctypes.byref(params(k_crit=0))) == 0
    small = sla.workspace_size(params(N=64, k_crit=1, k_neg=0))
    big = sla.workspace_size(params(N=64 * 100))
    assert big > small


def call_forward(lib, p, q=0x10000, k=0x20000, v=0x30000, o=0x40000, ws=0x50000, nbytes=None):
    nbytes = sla.workspace_size(p) if nbytes is None else nbytes
    return lib.sla_forward(q, k, v, o, ctypes.byref(p), ws, nbytes, None)


def test_forward_rejects_on_host(lib):
    # Fake device addresses: every case is rejected before any CUDA call.
    p = params()
    assert call_forward(lib, p, q=None) == sla.SLA_ERR_INVALID_ARG
    assert call_forward(lib, p, v=0x30008) == sla.SLA_ERR_ALIGNMENT
    assert call_forward(lib, p, ws=None) == sla.SLA_ERR_WORKSPACE
    assert call_forward(lib, p, ws=0x50080) == sla.SLA_ERR_WORKSPACE  # not 256-aligned
    assert call_forward(lib, p, nbytes=sla.workspace_size(p) - 1) == sla.SLA_ERR_WORKSPACE
    assert call_forward(lib, params(k_crit=0), nbytes=1 << 30) == sla.SLA_ERR_INVALID_ARG
    assert call_forward(lib, params(precision="i8qk_f8pv", variant="sla2", k_neg=0, alpha=None),
                        nbytes=1 << 30) == sla.SLA_ERR_INVALID_ARG
    pw = params()
    pw.w_proj = 0x60004
    assert call_forward(lib, pw) == sla.SLA_ERR_ALIGNMENT
    assert lib.sla_dense_forward(0x10000, 0x20000, None, 0x40000, 1, 1, 64, 64, 0.0, None) == \
        sla.SLA_ERR_INVALID_ARG
    assert lib.sla_dense_forward(0x10000, 0x20000, 0x30000, 0x40000, 1, 1, 64, 80, 0.0, None) == \
        sla.SLA_ERR_UNSUPPORTED
    assert lib.sla_get_mask(ctypes.byref(p), None, None, None, None, None) == sla.SLA_ERR_WORKSPACE
    assert lib.sla_read_device_status(0x50080, None) == sla.SLA_ERR_WORKSPACE  # not 256-aligned
    # the bounded-wait self-test: a workspace of at least one 256-byte status block, a limit in range
    assert lib.sla_check_wait_timeout(None, 256, 100000, None) == sla.SLA_ERR_WORKSPACE
    assert lib.sla_check_wait_timeout(0x50080, 256, 100000, None) == sla.SLA_ERR_WORKSPACE
    assert lib.sla_check_wait_timeout(0x50000, 255, 100000, None) == sla.SLA_ERR_WORKSPACE
    assert lib.sla_check_wait_timeout(0x50000, 256, 0, None) == sla.SLA_ERR_INVALID_ARG
    assert lib.sla_check_wait_timeout(0x50000, 256, 4000000001, None) == sla.SLA_ERR_INVALID_ARG


def test_header_constants_match_the_binding():
    text = open(os.path.join(ROOT, "include", "sla.h")).read()

    def define(name):
        m = re.search(r"#define\s+" + name + r"\s+(.+?)\s*(/\*.*)?$", text, flags=re.M)
        assert m, name
        return eval(m.group(1).replace("u", ""))  # plain integer expressions such as (32u << 20)

    assert define("SLA_NOALLOC_WORKSPACE_BYTES") == sla.NOALLOC_WORKSPACE_BYTES
    assert define("SLA_NUM_STAGES") == sla.NUM_STAGES == len(sla.STAGES)
    assert define("SLA_BLOCK") == sla.BLOCK


def test_binding_fails_loudly_without_library(tmp_path):
    import importlib

    mod = importlib.import_module("sparse_linear_attention_pool_b200")
    with pytest.raises(RuntimeError, match="not built"):
        # a fresh loader pointed at a path with no library
        saved = mod._lib
        mod._lib = None
        try:
            mod.load(str(tmp_path / "missing.so"))
        finally:
            mod._lib = saved


def test_router_training_and_backward_reject_on_host(lib):
    # Fake device addresses again: every case below is rejected before any CUDA call.
    by = ctypes.byref
    p = params()
    nb = sla.workspace_size(p)
    # SoftTop-k router
    assert lib.sla_router_soft_topk(0x10000, 0x20000, by(p), 0.0, 0x60000, None, None, 0x50000, nb, None) == \
        sla.SLA_ERR_INVALID_ARG
    assert lib.sla_router_soft_topk(0x10000, 0x20000, by(p), float("inf"), 0x60000, None, None, 0x50000, nb,
                                    None) == sla.SLA_ERR_INVALID_ARG
    assert lib.sla_router_soft_topk(0x10000, 0x20000, by(p), 0.1, None, None, None, 0x50000, nb, None) == \
        sla.SLA_ERR_INVALID_ARG
    assert lib.sla_router_soft_topk(0x10008, 0x20000, by(p), 0.1, 0x60000, None, None, 0x50000, nb, None) == \
        sla.SLA_ERR_ALIGNMENT
    assert lib.sla_router_soft_topk(0x10000, 0x20000, by(p), 0.1, 0x60000, None, None, 0x50000, nb - 1, None) == \
        sla.SLA_ERR_WORKSPACE
    # training forward
    sv = sla.Saved(o_s=0x70000, o_l=0x80000, lse=0x90000, den=0xA0000)
    tf = lambda pp, s_, n=nb: lib.sla_forward_train(0x10000, 0x20000, 0x30000, 0x40000, by(pp), s_, 0x50000,  # noqa: E731
                                                    n, None)
    assert tf(p, None) == sla.SLA_ERR_INVALID_ARG
    assert tf(p, by(sla.Saved(o_s=0x70000, o_l=None, lse=0x90000, den=0xA0000))) == sla.SLA_ERR_INVALID_ARG
    assert tf(p, by(sla.Saved(o_s=0x70008, o_l=0x80000, lse=0x90000, den=0xA0000))) == sla.SLA_ERR_ALIGNMENT
    assert tf(p, by(sv), nb - 1) == sla.SLA_ERR_WORKSPACE
    pq = params(precision="i8qk_f8pv", variant="sla2", k_neg=0)
    pq.alpha = 0x1000
    assert tf(pq, by(sv), 1 << 30) == sla.SLA_ERR_UNSUPPORTED
    # backward
    bn = lib.sla_backward_workspace_size(by(p))
    assert bn > 0 and lib.sla_backward_workspace_size(by(params(k_crit=0))) == 0

    def bw(pp, dO=0xB0000, saved=sv, fb=nb, dW=None, da=None, bnb=bn):
        return lib.sla_backward(0x10000, 0x20000, 0x30000, dO, by(pp), by(saved) if saved is not None else None,
                                0x50000, fb, 0xC0000, 0xD0000, 0xE0000, dW, da, 0xF0000, bnb, None)

    assert bw(p, dO=None) == sla.SLA_ERR_INVALID_ARG
    assert bw(p, saved=None) == sla.SLA_ERR_INVALID_ARG
    assert bw(p, da=0x100000) == sla.SLA_ERR_INVALID_ARG  # dalpha is SLA2's
    assert bw(p, fb=nb - 1) == sla.SLA_ERR_WORKSPACE
    assert bw(p, bnb=bn - 1) == sla.SLA_ERR_WORKSPACE
    assert bw(p, dO=0xB0008) == sla.SLA_ERR_ALIGNMENT
    p2 = params(variant="sla2", k_neg=0)
    p2.alpha = 0x1000
    bn2 = lib.sla_backward_workspace_size(by(p2))
    assert bw(p2, dW=0x100000, bnb=bn2, fb=sla.workspace_size(p2)) == sla.SLA_ERR_INVALID_ARG  # dW is SLA's
    assert bw(pq, fb=1 << 30, bnb=1 << 30) == sla.SLA_ERR_UNSUPPORTED
