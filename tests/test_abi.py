"""Host-side checks of the C ABI (no GPU, no compute calls).

* the library loads and exports every function include/qlora_nf4.h declares;
* its host-computed NF4 table and thresholds equal the oracle's bit for bit
  (two independent constructions: the library bisects libm's erfc, the
  oracle uses Python's statistics.NormalDist);
* argument validation rejects bad calls before touching a device.
"""

import ctypes as C
import os
import re

import numpy as np
import pytest

import oracle
from qlora_linear_layers_b200 import _lib
from qlora_linear_layers_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "qlora_nf4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "sizeof")))


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES)
    assert lib.qlora_abi_version() == 200


def test_library_table_matches_oracle(lib):
    buf = (C.c_float * 16)()
    assert lib.nf4_code_table(buf) == 0
    got = np.frombuffer(buf, dtype=np.float32)
    want = oracle.nf4_table()
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    tb = (C.c_float * 15)()
    assert lib.nf4_code_thresholds(tb) == 0
    assert np.array_equal(np.frombuffer(tb, dtype=np.float32), oracle.thresholds(want))


@pytest.mark.parametrize("qt", [_lib.QLORA_QUANT_NF4, _lib.QLORA_QUANT_FP4])
def test_library_tables_match_oracle_per_type(lib, qt):
    """The library's tables of both 4-bit types equal the oracle's: values by
    code and the thresholds between distinct values (FP4: the E2M1 list in
    the library, the bit-field formula in the oracle)."""
    buf = (C.c_float * 16)()
    assert lib.qlora_code_table(qt, buf) == 0
    got = np.frombuffer(buf, dtype=np.float32)
    want = oracle.nf4_table() if qt == _lib.QLORA_QUANT_NF4 else oracle.fp4_table()
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    tb = (C.c_float * 15)()
    cnt = C.c_int(0)
    assert lib.qlora_code_thresholds(qt, tb, C.byref(cnt)) == 0
    T = oracle.thresholds(want)
    assert cnt.value == T.size
    assert np.array_equal(np.frombuffer(tb, dtype=np.float32)[:cnt.value], T)
    assert lib.qlora_code_table(7, buf) == _lib.QLORA_ERR_INVALID_ARG


def test_status_strings(lib):
    for code in range(9):
        assert lib.qlora_status_string(code)
    assert lib.qlora_status_string(99) == b"unknown status"


def test_workspace_sizes(lib):
    assert lib.qlora_workspace_bytes(_lib.QLORA_OP_DOUBLE_QUANT, 0, 1000, 0, 0) == 2048
    ws = lambda op, M, N, K, r: lib.qlora_workspace_bytes(op, M, N, K, r)
    for (N, K, r) in ((18944, 3584, 64), (3584, 18944, 64), (4096, 4096, 16), (200, 192, 8)):
        fwd = [ws(_lib.QLORA_OP_FWD, M, N, K, r) for M in (1, 4, 16, 17, 300, 8192)]
        # decode (M <= 16) keeps fp32 partials per token; the GEMM path per token tile
        assert all(x > 0 for x in fwd)
        assert fwd[0] <= fwd[1] <= fwd[2] and fwd[3] <= fwd[4] <= fwd[5]
        assert fwd[2] >= 16 * (N + r) * 4                      # one fp32 partial per output
        # the backward holds the transposed dequantised weight deq(W)^T in bf16
        for M in (17, 300, 8192):
            assert ws(_lib.QLORA_OP_BWD, M, N, K, r) >= 2 * N * K


def test_validation_before_any_device_call(lib):
    # Null pointers, bad shapes, misalignment: rejected synchronously.  The
    # fake addresses below are never dereferenced (validation fails first).
    fake = 1 << 20
    assert lib.nf4_quantize(None, 1, 64, 64, 64, fake, fake, None) == _lib.QLORA_ERR_INVALID_ARG
    assert lib.nf4_quantize(fake, 7, 64, 64, 64, fake, fake, None) == _lib.QLORA_ERR_INVALID_ARG
    assert lib.nf4_quantize(fake, 1, 64, 64, 32, fake, fake, None) == _lib.QLORA_ERR_UNSUPPORTED
    assert lib.nf4_quantize(fake, 1, 64, 96, 64, fake, fake, None) == _lib.QLORA_ERR_SHAPE
    assert lib.nf4_quantize(fake, 1, 0, 64, 64, fake, fake, None) == _lib.QLORA_ERR_SHAPE
    assert lib.nf4_quantize(fake + 2, 1, 64, 64, 64, fake, fake, None) == _lib.QLORA_ERR_ALIGN
    assert lib.nf4_double_quantize(fake, 100, 128, fake, fake, fake, fake, 4096, None) == \
        _lib.QLORA_ERR_UNSUPPORTED
    assert lib.nf4_double_quantize(fake, 100, 256, fake, fake, fake, None, 0, None) == \
        _lib.QLORA_ERR_WORKSPACE
    assert lib.nf4_double_quantize(fake, 100, 256, fake, fake, fake, fake, 16, None) == \
        _lib.QLORA_ERR_WORKSPACE
    w = _lib.NF4Weight(packed=fake, rows=64, cols=64, blocksize=64, double_quant=1,
                       absmax=None, qabsmax=None, dq_scale=fake, dq_mean=fake, dq_blocksize=256)
    assert lib.nf4_dequantize(C.byref(w), fake, None) == _lib.QLORA_ERR_INVALID_ARG
    w.qabsmax = fake
    w.cols = 100
    assert lib.nf4_dequantize(C.byref(w), fake, None) == _lib.QLORA_ERR_SHAPE
    w.cols = 64
    w.quant_type = 5
    assert lib.nf4_dequantize(C.byref(w), fake, None) == _lib.QLORA_ERR_INVALID_ARG
    assert lib.qlora_quantize_4bit(fake, 1, 64, 64, 64, 2, fake, fake, None, None) == \
        _lib.QLORA_ERR_INVALID_ARG
    assert lib.qlora_quantize_4bit(fake, 1, 64, 64, 64, 1, fake, fake, fake + 8, None) == \
        _lib.QLORA_ERR_ALIGN
    # the histogram pass: n_total below the local count, a missing histogram
    assert lib.nf4_double_quantize_hist(fake, 512, fake, 256, 256, fake, fake, fake, None) == \
        _lib.QLORA_ERR_SHAPE
    assert lib.nf4_double_quantize_hist(fake, 512, None, 512, 256, fake, fake, fake, None) == \
        _lib.QLORA_ERR_INVALID_ARG


def test_host_mean_from_histogram_matches_oracle(lib):
    """qlora_dq_mean_from_hist (host) equals oracle.dq_mean bit for bit on
    ordinary, extreme and degenerate absmax sets."""
    rng = np.random.default_rng(77)

    def hist_of(a):
        u = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.int64)
        e = u >> 23
        m = (u & 0x7FFFFF) | np.where(e > 0, 0x800000, 0)
        h = np.zeros(256, dtype=np.int64)
        np.add.at(h, e, m)
        return h

    cases = [
        np.abs(rng.standard_normal(100000)).astype(np.float32) * np.float32(0.05),
        np.array([1e-45, 3e-39, 1e-30, 1.0, 3e38], dtype=np.float32),      # subnormal to huge
        np.array([0.0, 0.0, 0.0], dtype=np.float32),
        np.array([0.25], dtype=np.float32),
        (np.abs(rng.standard_normal(4097)) * 10.0 ** rng.integers(-30, 30, 4097)).astype(np.float32),
    ]
    for a in cases:
        h = hist_of(a)
        mean = C.c_float(0.0)
        assert lib.qlora_dq_mean_from_hist(h.ctypes.data_as(C.POINTER(C.c_int64)), a.size,
                                           C.byref(mean)) == 0
        assert np.float32(mean.value).view(np.uint32) == np.float32(oracle.dq_mean(a)).view(np.uint32)
    h = np.zeros(256, dtype=np.int64)
    h[3] = -1
    assert lib.qlora_dq_mean_from_hist(h.ctypes.data_as(C.POINTER(C.c_int64)), 1, C.byref(mean)) == \
        _lib.QLORA_ERR_INVALID_ARG


def test_wait_limit_range_checked_on_the_host(lib):
    assert lib.qlora_set_wait_limit(1000) == _lib.QLORA_ERR_INVALID_ARG            # below 1 ms
    assert lib.qlora_set_wait_limit(61 * 10 ** 9) == _lib.QLORA_ERR_INVALID_ARG    # above 60 s
