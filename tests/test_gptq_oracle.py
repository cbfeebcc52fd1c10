"""Pins of the FP64 GPTQ oracle ("4.3 Weight-only INT4", section 2) against facts that do not
come from the oracle itself: the page's two-column example, the least-squares optimum of one
compensation step, the inverse of the remaining submatrix, the diagonal-H case that reduces to
plain rounding, and the objective it lowers."""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import gptq
from weight_only_int4_07_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_two_column_worked_example():
    """Section 2.2: with two identical input columns, fixing w1 = 0.26 at 0.30 moves w2 by
    -0.04 (the damping keeps H invertible; as it goes to 0 the move goes to -0.04)."""
    g = _golden("gptq_two_column.json")
    x = np.linspace(-1.0, 1.0, 64)
    X = np.stack([x, x], axis=1)
    H = gptq.hessian(X)
    for damp, tol in ((1e-6, 1e-6), (1e-9, 1e-9)):
        Hd = H + damp * np.eye(2)
        W = np.array([[g["w1"]], [0.5]])
        Hinv = np.linalg.inv(Hd)
        gptq.compensate(W, Hinv, 0, np.array([g["w1_hat"]]))
        assert W[0, 0] == g["w1_hat"]
        assert abs((W[1, 0] - 0.5) - g["w2_adjustment"]) < tol
        assert abs(g["w1_hat"] - g["w1"] - g["overshoot"]) < 1e-12


def test_compensation_step_is_the_least_squares_optimum():
    """Section 2.1 objective: after channel 0 is fixed, the move of the free channels minimises
    ||X (w - w')||^2 over w' with w'_0 fixed -- checked against a least-squares solve."""
    rng = np.random.default_rng(5)
    S, K = 80, 6
    X = rng.standard_normal((S, K)) @ rng.standard_normal((K, K))   # correlated channels
    w = rng.standard_normal((K, 1))
    w0_hat = w[0, 0] + 0.137
    W = w.copy()
    Hinv = np.linalg.inv(gptq.hessian(X))
    gptq.compensate(W, Hinv, 0, np.array([w0_hat]))
    # least squares: X[:, 1:] d = X[:, 0] (w0 - w0_hat)  ->  w'_F = w_F + d
    d, *_ = np.linalg.lstsq(X[:, 1:], X[:, 0] * (w[0, 0] - w0_hat), rcond=None)
    assert np.allclose(W[1:, 0], w[1:, 0] + d, rtol=1e-9, atol=1e-12)
    assert W[0, 0] == w0_hat


def test_removal_step_gives_the_inverse_of_the_remaining_submatrix():
    rng = np.random.default_rng(6)
    K = 7
    A = rng.standard_normal((20, K))
    H = gptq.damped(gptq.hessian(A))
    Hinv = np.linalg.inv(H)
    W = rng.standard_normal((K, 3))
    for i in range(3):
        gptq.compensate(W, Hinv, i, W[i] + 0.01)
        assert np.allclose(Hinv[i + 1:, i + 1:], np.linalg.inv(H[i + 1:, i + 1:]), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("group,sym", [(128, 0), (32, 1), (64, 0)])
def test_diagonal_hessian_reduces_to_rtn(group, sym):
    """Orthogonal calibration columns make H diagonal, so no error is propagated and GPTQ gives
    exactly the RTN codes, scales and zeros of the plain quantizer."""
    K, N = 256, 64
    Wb = synthetic.weights_normal(K, N, 12)
    rng = np.random.default_rng(13)
    Q, _ = np.linalg.qr(rng.standard_normal((512, K)))
    X = Q * rng.uniform(0.5, 2.0, size=K)
    H = gptq.damped(gptq.hessian(X))
    H = np.diag(np.diag(H))   # exactly diagonal (QR leaves ~1e-16 off-diagonal terms)
    q, sb, zz, _ = gptq.gptq_values(oracle.decode16(Wb), H, group, sym)
    codes, scales, zeros = gptq.pack(q, sb, zz, sym)
    st, oc, os_, oz = oracle.quantize(Wb, group, sym)
    assert st == oracle.OK
    assert np.array_equal(codes, oc) and np.array_equal(scales, os_)
    if not sym:
        assert np.array_equal(zeros, oz)


@pytest.mark.parametrize("sym", [0, 1])
def test_gptq_lowers_the_output_error_of_rtn(sym):
    """The point of section 2: on correlated calibration inputs GPTQ's layer-output error is
    well below plain rounding's."""
    K, N, S, group = 256, 96, 512, 64
    Wb = synthetic.weights_normal(K, N, 14)
    Xb = synthetic.calibration(S, K, 15, dtype=synthetic.F16)
    X = oracle.decode16(Xb)
    codes, scales, zeros = gptq.gptq(Wb, Xb, oracle.F16, group, sym)
    W = oracle.decode16(Wb)
    e_gptq = gptq.output_error(X, W, oracle.dequant(codes, scales, zeros, K, N, group, sym))
    st, oc, os_, oz = oracle.quantize(Wb, group, sym)
    e_rtn = gptq.output_error(X, W, oracle.dequant(oc, os_, oz, K, N, group, sym))
    assert e_gptq < 0.8 * e_rtn


def test_codes_are_in_range_and_pack_round_trips():
    K, N, group = 128, 32, 32
    Wb = synthetic.weights_student_t(K, N, 16)
    Xb = synthetic.calibration(256, K, 17, dtype=synthetic.F16)
    for sym in (0, 1):
        X = oracle.decode16(Xb)
        q, sb, zz, What = gptq.gptq_values(oracle.decode16(Wb), gptq.damped(gptq.hessian(X)), group, sym)
        assert q.min() >= (-8 if sym else 0) and q.max() <= (7 if sym else 15)
        codes, scales, zeros = gptq.pack(q, sb, zz, sym)
        assert np.array_equal(oracle.unpack_codes(codes, K, sym), q)
        assert np.array_equal(oracle.dequant(codes, scales, zeros, K, N, group, sym), What)
