"""The C ABI without a GPU: exports, argument validation, host-only calls."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import alloc
from post_quantization_kronq_b200 import _lib
from post_quantization_kronq_b200.dist import shard_units

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = ctypes.c_void_p(4096)   # never dereferenced: every call below fails validation first


def header_functions():
    txt = open(os.path.join(ROOT, "include", "kronq.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(kronq_[a-z0-9_]+)\s*\(", txt)))


def test_every_declared_symbol_is_exported():
    names = header_functions()
    assert len(names) >= 15
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"


def test_version_and_error_strings():
    assert b"sm_100a" in _lib.lib.kronq_version()
    assert isinstance(_lib.lib.kronq_last_error(), bytes)


def _st(v):
    return int(v)


def test_pack_rejects_three_bits():
    assert _st(_lib.lib.kronq_pack(FAKE, 4, 8, 3, FAKE, None)) == _lib.ERR_INVALID_ARG
    assert b"3-bit" in _lib.lib.kronq_last_error()
    assert _st(_lib.lib.kronq_unpack(FAKE, 4, 8, 5, FAKE, None)) == _lib.ERR_INVALID_ARG
    assert _st(_lib.lib.kronq_pack(None, 4, 8, 4, FAKE, None)) == _lib.ERR_INVALID_ARG


def _qp(**kw):
    base = dict(bits=4, group=128, asym=1, damp_rel=0.01, block=128, flags=0)
    base.update(kw)
    return _lib.QuantParams(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(bits=5), _lib.ERR_INVALID_ARG),
    (dict(bits=1), _lib.ERR_INVALID_ARG),
    (dict(group=96), _lib.ERR_INVALID_ARG),
    (dict(group=0), _lib.ERR_INVALID_ARG),
    (dict(block=64), _lib.ERR_UNSUPPORTED),
    (dict(asym=2), _lib.ERR_INVALID_ARG),
    (dict(damp_rel=-1.0), _lib.ERR_INVALID_ARG),
    (dict(damp_rel=float("nan")), _lib.ERR_INVALID_ARG),
    (dict(flags=64), _lib.ERR_INVALID_ARG),
    (dict(flags=_lib.WRITE_E), _lib.ERR_INVALID_ARG),   # E is NULL below
    (dict(flags=_lib.R_FORM | _lib.U_GIVEN), _lib.ERR_INVALID_ARG),
    (dict(flags=_lib.R_FORM | _lib.ORDERED_FP32), _lib.ERR_INVALID_ARG),
    (dict(flags=_lib.R_FORM, group=256), _lib.ERR_UNSUPPORTED),
])
def test_quantize_layer_validation(kw, status):
    p = _qp(**kw)
    r = _lib.lib.kronq_quantize_layer(FAKE, FAKE, 64, 256, ctypes.byref(p), FAKE, FAKE, FAKE, None,
                                      FAKE, FAKE, 1 << 40, None)
    assert _st(r) == status


def test_quantize_layer_null_and_workspace():
    p = _qp()
    assert _st(_lib.lib.kronq_quantize_layer(FAKE, FAKE, 64, 256, None, FAKE, FAKE, FAKE, None, FAKE,
                                             FAKE, 1 << 40, None)) == _lib.ERR_INVALID_ARG
    need = _lib.lib.kronq_quantize_workspace_bytes(64, 256, ctypes.byref(p))
    assert need > 64 * 128 * 4
    r = _lib.lib.kronq_quantize_layer(FAKE, FAKE, 64, 256, ctypes.byref(p), FAKE, FAKE, FAKE, None,
                                      FAKE, FAKE, need - 1, None)
    assert _st(r) == _lib.ERR_INVALID_ARG
    r = _lib.lib.kronq_quantize_layer(FAKE, FAKE, 0, 256, ctypes.byref(p), FAKE, FAKE, FAKE, None,
                                      FAKE, FAKE, need, None)
    assert _st(r) == _lib.ERR_INVALID_ARG


def test_r_form_workspace():
    # the R form keeps a copy of W~ (m n floats) and U's 128 x 128 diagonal
    # blocks (ceil(n / 128) of them) on top
    for m, n in [(64, 256), (1000, 4500), (8192, 28672)]:
        base = _lib.lib.kronq_quantize_workspace_bytes(m, n, ctypes.byref(_qp()))
        rf = _lib.lib.kronq_quantize_workspace_bytes(m, n, ctypes.byref(_qp(flags=_lib.R_FORM)))
        extra = rf - base
        want = 4 * (m * n + 128 * 128 * (-(-n // 128)))
        assert want <= extra <= want + 512
        p = _qp(flags=_lib.R_FORM)
        r = _lib.lib.kronq_quantize_layer(FAKE, FAKE, m, n, ctypes.byref(p), FAKE, FAKE, FAKE, None,
                                          FAKE, FAKE, rf - 1, None)
        assert _st(r) == _lib.ERR_INVALID_ARG


def test_accumulate_validation():
    L = _lib.lib
    assert _st(L.kronq_accumulate_factors(FAKE, 7, 16, 8, 8, FAKE, 1, None)) == _lib.ERR_INVALID_ARG
    assert _st(L.kronq_accumulate_factors(FAKE, 0, 16, 8, 4, FAKE, 1, None)) == _lib.ERR_INVALID_ARG
    assert _st(L.kronq_accumulate_factors(FAKE, 0, -1, 8, 8, FAKE, 1, None)) == _lib.ERR_INVALID_ARG
    assert _st(L.kronq_accumulate_factors(None, 0, 16, 8, 8, FAKE, 1, None)) == _lib.ERR_INVALID_ARG
    assert _st(L.kronq_accumulate_factors(FAKE, 0, 16, 8, 8, None, 1, None)) == _lib.ERR_INVALID_ARG


def test_biip_validation():
    L = _lib.lib
    ws = L.kronq_biip_workspace_bytes(64, 128)
    assert ws >= 128 * 128 * 4
    ok_ws = ctypes.c_void_p(4096 * 256)
    # H_G required for the output-side rescale
    r = L.kronq_biip_forward(FAKE, 0, ctypes.c_void_p(8192), 64, 128, FAKE, None, 0, 0.25, 0, FAKE,
                             FAKE, ok_ws, ws, None)
    assert _st(r) == _lib.ERR_INVALID_ARG
    # odd factor 257 of n = 514 is beyond the DCT limit
    ws2 = L.kronq_biip_workspace_bytes(64, 514)
    r = L.kronq_biip_forward(FAKE, 0, ctypes.c_void_p(8192), 64, 514, FAKE, FAKE, 0, 0.25, 0, FAKE,
                             FAKE, ok_ws, ws2, None)
    assert _st(r) == _lib.ERR_UNSUPPORTED
    # bad mode, aliasing, misaligned workspace
    r = L.kronq_biip_forward(FAKE, 0, ctypes.c_void_p(8192), 64, 128, FAKE, FAKE, 0, 0.25, 9, FAKE,
                             FAKE, ok_ws, ws, None)
    assert _st(r) == _lib.ERR_INVALID_ARG
    r = L.kronq_biip_forward(FAKE, 0, FAKE, 64, 128, FAKE, FAKE, 0, 0.25, 0, FAKE, FAKE, ok_ws, ws, None)
    assert _st(r) == _lib.ERR_INVALID_ARG
    r = L.kronq_biip_forward(FAKE, 0, ctypes.c_void_p(8192), 64, 128, FAKE, FAKE, 0, 0.25, 0, FAKE,
                             FAKE, ctypes.c_void_p(4096 + 16), ws, None)
    assert _st(r) == _lib.ERR_INVALID_ARG
    r = L.kronq_biip_inverse(FAKE, 64, 128, 0, 0, FAKE, FAKE, ok_ws, ws - 256, None)
    assert _st(r) == _lib.ERR_INVALID_ARG


def test_sensitivity_and_loss_validation():
    L = _lib.lib
    out = (ctypes.c_double * 3)()
    assert _st(L.kronq_sensitivity(None, 4, FAKE, 4, out, FAKE, 16, None)) == _lib.ERR_INVALID_ARG
    assert _st(L.kronq_sensitivity(FAKE, 4, FAKE, 4, out, FAKE, 8, None)) == _lib.ERR_INVALID_ARG
    d = ctypes.c_double()
    assert _st(L.kronq_kfac_loss(FAKE, FAKE, 4, 4, ctypes.byref(d), FAKE, 0, None)) == _lib.ERR_INVALID_ARG
    assert _st(L.kronq_device_status(None, None)) == _lib.ERR_INVALID_ARG


# ------------------------------------------------------------------ host allocation
def test_budget_allocation_matches_oracle():
    from post_quantization_kronq_b200 import kronq_allocate_bits
    rng = np.random.default_rng(0)
    sizes = [4096 * 4096, 1024 * 4096, 1024 * 4096, 4096 * 4096, 14336 * 4096, 14336 * 4096,
             4096 * 14336] * 32
    for trial in range(10):
        s = list(np.exp(rng.normal(size=len(sizes)) * 3))
        assert kronq_allocate_bits(s, sizes, 2.5, 2, 4) == alloc.allocate_budget(s, sizes, 2.5, 2, 4)
    s = [1.0] * 8
    assert kronq_allocate_bits(s, [1] * 8, 2.5) == alloc.allocate_budget(s, [1] * 8, 2.5)


def test_topn_allocation_matches_oracle():
    from post_quantization_kronq_b200 import kronq_allocate_topn_types
    rng = np.random.default_rng(1)
    names = ["q", "k", "v", "o", "gate", "up", "down"]
    types = names * 32
    ids = [names.index(t) for t in types]
    for N in (0, 1, 3, 7):
        s = list(np.exp(rng.normal(size=len(types))))
        assert kronq_allocate_topn_types(s, ids, 7, 2, N) == alloc.allocate_topn_types(s, types, 2, N)


def test_allocation_validation():
    L = _lib.lib
    out = (ctypes.c_int * 2)()
    s = (ctypes.c_double * 2)(1.0, 2.0)
    z = (ctypes.c_int64 * 2)(1, 0)
    assert _st(L.kronq_allocate_bits(s, z, 2, 2.5, 2, 4, out)) == _lib.ERR_INVALID_ARG
    z = (ctypes.c_int64 * 2)(1, 1)
    assert _st(L.kronq_allocate_bits(s, z, 2, 1.5, 2, 4, out)) == _lib.ERR_INVALID_ARG
    assert _st(L.kronq_allocate_bits(s, z, 2, 2.5, 2, 4, out)) == _lib.OK


def test_shard_units_partition():
    for n in (0, 1, 7, 224):
        for w in (1, 2, 3, 8):
            got = sum((shard_units(n, r, w) for r in range(w)), [])
            assert got == list(range(n))


def test_kron_factors_validation():
    L = _lib.lib
    ws = L.kronq_kron_factors_workspace_bytes(1000, 128, 64)
    assert ws > 0 and L.kronq_kron_factors_workspace_bytes(1000, 0, 64) == 0
    ok = dict(T=1000, n=128, m=64, est=3, iters=2)

    def call(**kw):
        a = dict(ok, **kw)
        return _st(L.kronq_kron_factors(FAKE, FAKE, a["T"], a["n"], a["m"], a["est"], a["iters"], FAKE,
                                        FAKE, FAKE, ctypes.c_void_p(4096 * 256),
                                        kw.get("ws", ws), None))
    assert call(est=4) == _lib.ERR_INVALID_ARG
    assert call(n=60) == _lib.ERR_INVALID_ARG        # below 64
    assert call(m=100) == _lib.ERR_INVALID_ARG       # not a multiple of 8
    assert call(T=0) == _lib.ERR_INVALID_ARG
    assert call(iters=-1) == _lib.ERR_INVALID_ARG
    assert call(ws=ws - 1) == _lib.ERR_INVALID_ARG
    assert _st(L.kronq_kron_factors(None, FAKE, 1000, 128, 64, 3, 2, FAKE, FAKE, FAKE,
                                    ctypes.c_void_p(4096 * 256), ws, None)) == _lib.ERR_INVALID_ARG


def test_decode_matvec_validation():
    L = _lib.lib
    ws = L.kronq_decode_matvec_workspace_bytes(64, 96)
    assert ws > 0 and L.kronq_decode_matvec_workspace_bytes(0, 96) == 0
    W = ctypes.c_void_p(4096 * 256)

    def call(m=64, n=96, bits=4, group=32, mode=0, xdt=1, nbytes=ws, x=FAKE):
        return _st(L.kronq_decode_matvec(FAKE, FAKE, FAKE, m, n, bits, group, 7, mode, FAKE, FAKE, x,
                                         xdt, FAKE, W, nbytes, None))
    assert call(bits=3) == _lib.ERR_INVALID_ARG
    assert call(group=0) == _lib.ERR_INVALID_ARG
    assert call(mode=4) == _lib.ERR_INVALID_ARG
    assert call(xdt=9) == _lib.ERR_INVALID_ARG
    assert call(nbytes=ws - 1) == _lib.ERR_INVALID_ARG
    assert call(x=None) == _lib.ERR_INVALID_ARG
    assert call(n=257 * 2) == _lib.ERR_UNSUPPORTED      # odd factor 257 of a rotated dimension


def test_wait_selftest_validation():
    L = _lib.lib
    assert _st(L.kronq_wait_selftest(2, 1000000, FAKE, 16, None)) == _lib.ERR_INVALID_ARG
    assert _st(L.kronq_wait_selftest(0, 0, FAKE, 16, None)) == _lib.ERR_INVALID_ARG
    assert _st(L.kronq_wait_selftest(0, 2000000000, FAKE, 16, None)) == _lib.ERR_INVALID_ARG
    assert _st(L.kronq_wait_selftest(1, 1000000, None, 16, None)) == _lib.ERR_INVALID_ARG
    assert _st(L.kronq_wait_selftest(1, 1000000, FAKE, 8, None)) == _lib.ERR_INVALID_ARG


def test_act_order_validation():
    L = _lib.lib
    p = _lib.QuantParams(bits=2, group=128, asym=1, damp_rel=0.01, block=128, flags=_lib.U_GIVEN)
    args = [FAKE, FAKE, 8, 256, ctypes.byref(p), FAKE, FAKE, FAKE, None, FAKE, None, FAKE, FAKE, 1 << 30, None]
    assert _st(L.kronq_quantize_layer_act_order(*args)) == _lib.ERR_INVALID_ARG      # U_GIVEN
    p.flags = 0
    args[9] = None
    assert _st(L.kronq_quantize_layer_act_order(*args)) == _lib.ERR_INVALID_ARG      # no g_idx
    args[9] = FAKE
    args[13] = 16
    assert _st(L.kronq_quantize_layer_act_order(*args)) == _lib.ERR_INVALID_ARG      # workspace
    assert L.kronq_quantize_act_order_workspace_bytes(8, 256, ctypes.byref(p)) > 256 * 256 * 4


def test_two_sided_validation():
    L = _lib.lib
    p = _qp(bits=2)
    need = L.kronq_quantize_two_sided_workspace_bytes(96, 300, ctypes.byref(p))
    # two m x n float32 buffers (P = E U_X and the scaled errors) on top of
    # the factorisation scratch
    assert need >= 2 * 4 * 96 * 300
    assert L.kronq_quantize_two_sided_workspace_bytes(0, 300, ctypes.byref(p)) == 0

    def call(p, HG=FAKE, ws=need, m=96, n=300, E=None):
        return _st(L.kronq_quantize_two_sided(FAKE, FAKE, HG, m, n, ctypes.byref(p), FAKE, FAKE, FAKE, E, FAKE,
                                              FAKE, ws, None))

    assert call(p, HG=None) == _lib.ERR_INVALID_ARG
    assert call(p, ws=need - 1) == _lib.ERR_INVALID_ARG
    assert call(p, m=0) == _lib.ERR_INVALID_ARG
    assert call(p, m=(1 << 20) + 1, ws=1 << 62) == _lib.ERR_INVALID_ARG
    for flags in (_lib.R_FORM, _lib.ORDERED_FP32, _lib.WRITE_E, 64):   # WRITE_E: E is NULL
        assert call(_qp(bits=2, flags=flags)) == _lib.ERR_INVALID_ARG
    assert call(_qp(bits=5)) == _lib.ERR_INVALID_ARG
    assert call(_qp(group=96)) == _lib.ERR_INVALID_ARG
    assert call(_qp(block=64)) == _lib.ERR_UNSUPPORTED
