"""Pins for the oracle's block-scaled GEMM and gates (CPU only).

GEMM: on tiny shapes the sum is done exactly in Python integers (every product
e2m1 * e2m1 * s_a * s_b is an integer multiple of 2^-20: E2M1 values are
multiples of 1/2 and E4M3 values multiples of 2^-9), then scaled by g_a * g_b;
one-hot operands reproduce single products (catches index / transpose errors).

Gates ("Anthology of the SOTA, theory-128", section "The account"): closed forms
at softplus(0) = ln 2 and sigmoid(0) = 1/2 (tests/golden), and numpy's
logaddexp / scipy's expit as independent library routines.
"""
import os

import numpy as np
import pytest
import scipy.special

from oracle import nvfp4
from oracle.gemm import gemm_bf16, gemm_fp64
from oracle.gates import gates, softplus


def _exact_int_gemm(aq, bq):
    ca = nvfp4.unpack_codes(aq["codes"]).astype(np.int64)
    cb = nvfp4.unpack_codes(bq["codes"]).astype(np.int64)
    # integer images: 2 * e2m1 value and 512 * e4m3 value are integers
    va = (nvfp4.e2m1_decode(ca) * 2).astype(np.int64)
    vb = (nvfp4.e2m1_decode(cb) * 2).astype(np.int64)
    sa = (nvfp4.e4m3_decode(aq["scales"]) * 512).astype(np.int64)
    sb = (nvfp4.e4m3_decode(bq["scales"]) * 512).astype(np.int64)
    M, K = va.shape
    N = vb.shape[0]
    out = np.empty((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0
            for kk in range(K):
                acc += int(va[m, kk]) * int(vb[n, kk]) * int(sa[m, kk // 16]) * int(sb[n, kk // 16])
            out[m, n] = float(acc) * 2.0 ** -20 * float(aq["g"]) * float(bq["g"])
    return out


@pytest.mark.parametrize("M,N,K,seed", [(3, 5, 32, 0), (8, 7, 64, 1), (4, 4, 256, 2)])
def test_gemm_matches_exact_integer_sum(M, N, K, seed):
    rng = np.random.default_rng(seed)
    a = nvfp4.round_bf16(rng.standard_normal((M, K))).astype(np.float32)
    b = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    aq, bq = nvfp4.quantize(a), nvfp4.quantize(b)
    ref = _exact_int_gemm(aq, bq)
    got = gemm_fp64(aq, bq)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-300)


def test_gemm_one_hot():
    K = 64
    a = np.zeros((3, K), np.float32)
    b = np.zeros((4, K), np.float32)
    a[1, 17] = 3.0
    b[2, 17] = -2.0      # block maxima that map exactly onto E2M1 6 * E4M3 448
    b[3, 18] = 2.0
    aq, bq = nvfp4.quantize(a), nvfp4.quantize(b)
    y = gemm_fp64(aq, bq)
    want = np.zeros((3, 4))
    want[1, 2] = -6.0
    # exact zeros everywhere else; the one product is off only by the FP32
    # rounding of the two decode scales 1/896 and 1/1344
    np.testing.assert_array_equal(y != 0, want != 0)
    np.testing.assert_allclose(y, want, rtol=2 * 2.0 ** -24)


def test_gemm_bf16_is_one_rounding():
    rng = np.random.default_rng(3)
    a = nvfp4.round_bf16(rng.standard_normal((16, 64))).astype(np.float32)
    b = (rng.standard_normal((16, 64)) * 0.02).astype(np.float32)
    aq, bq = nvfp4.quantize(a), nvfp4.quantize(b)
    y = gemm_bf16(aq, bq)
    y64 = gemm_fp64(aq, bq)
    # |y - y64| <= half a bf16 ulp (2^-8 relative)
    assert np.all(np.abs(y - y64) <= np.abs(y64) * 2.0 ** -8)


def _read_rows(path):
    rows = []
    with open(path) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append([float(t) for t in line.split()])
    return np.array(rows)


def test_gates_closed_forms(golden_dir):
    rows = _read_rows(os.path.join(golden_dir, "gates_closed_form.txt"))
    for A, x, b, alpha, beta in rows:
        la, be = gates(np.array([x]), np.array([b]), np.array([A]), np.array([0.0]))
        assert abs(np.exp(la[0]) - alpha) < 1e-15
        assert abs(be[0] - beta) < 1e-15
    # dt_bias and a enter only through their sum
    la1, _ = gates(np.array([0.3]), np.array([0.0]), np.array([0.2]), np.array([-0.1]))
    la2, _ = gates(np.array([0.0]), np.array([0.0]), np.array([0.2]), np.array([0.2]))
    assert abs(la1[0] - la2[0]) < 1e-15


def test_gates_against_library_routines():
    rng = np.random.default_rng(4)
    x = rng.standard_normal(1000) * 10
    np.testing.assert_allclose(softplus(x), np.logaddexp(0.0, x), rtol=1e-14, atol=0)
    A = rng.uniform(-2, 1, 1000)
    a = rng.standard_normal(1000)
    dt = rng.uniform(-1, 1, 1000)
    b = rng.standard_normal(1000) * 5
    la, be = gates(a, b, A, dt)
    np.testing.assert_allclose(la, -np.exp(A) * np.logaddexp(0.0, a + dt), rtol=1e-14)
    np.testing.assert_allclose(be, scipy.special.expit(b), rtol=1e-14)


def test_gates_ranges_and_monotonicity():
    x = np.linspace(-30, 30, 601)
    la, be = gates(x, x, np.zeros(1), np.zeros(1))
    assert np.all(la < 0) and np.all(np.diff(la) < 0)          # alpha in (0,1), falls with a
    assert np.all((be > 0) & (be < 1)) and np.all(np.diff(be) > 0)
    # large-|x| limits: softplus(x) -> x, softplus(-x) -> e^-x
    assert abs(softplus(np.array([40.0]))[0] - 40.0) < 1e-15
    assert abs(softplus(np.array([-40.0]))[0] / np.exp(-40.0) - 1) < 1e-12
