"""Pins of the FP64 AWQ oracle ("4.3 Weight-only INT4", section 3) against facts that do not come
from the oracle: alpha = 0 and r = 1 are plain RTN, the page's statement that scaling a channel
up while the group's tick gap stays put divides that channel's error by the factor, the clip
objective against a direct evaluation of the group's output error, constant activation
magnitudes that make every factor 1, and lower output error than RTN where a few input channels
carry large activations."""
import numpy as np
import pytest

import oracle
from oracle import awq
from weight_only_int4_07_b200 import synthetic


@pytest.mark.parametrize("group,sym", [(128, 0), (32, 1)])
def test_alpha_zero_and_no_clip_is_rtn(group, sym):
    K, N = 256, 64
    Wb = synthetic.weights_normal(K, N, 40)
    W = oracle.decode16(Wb)
    sbits, s = awq.scale_candidate(np.abs(np.random.default_rng(1).standard_normal(K)) + 0.1, 0.0)
    assert np.all(s == 1.0)
    q, sb, zz, D = awq.quantize_scaled(W, s, group, sym, 1.0)
    from oracle.gptq import pack
    codes, scales, zeros = pack(q, sb, zz, sym)
    st, oc, os_, oz = oracle.quantize(Wb, group, sym)
    assert np.array_equal(codes, oc) and np.array_equal(scales, os_)
    if not sym:
        assert np.array_equal(zeros, oz)


def test_scaling_a_channel_up_divides_its_error_when_the_tick_gap_stays():
    """Section 3.2: amplify channel j by s_j while the group's range is set elsewhere, and the
    error left on that channel after dividing back is at most half a tick over s_j."""
    g = 32
    rng = np.random.default_rng(2)
    w = rng.uniform(-0.01, 0.01, size=(g, 1))
    w[0, 0] = 1.0      # sets the range: tick = (1 - lo) / 15
    w[1, 0] = -0.3
    j = 5
    s = np.ones(g)
    for sj in (1.0, 2.0, 3.0):
        s[j] = sj
        _, ss, _, _, D = awq.rtn_clipped(w * s[:, None], 0, 1.0)
        err = abs(w[j, 0] - D[j, 0] / s[j])
        assert err <= ss[0] / (2 * sj) + 1e-15
        assert ss[0] == awq.rtn_clipped(w, 0, 1.0)[1][0]   # the tick gap did not change


def test_clip_objective_is_the_groups_output_error():
    """delta^T (X_g^T X_g) delta equals ||X_g delta||^2 evaluated directly, for every ratio."""
    K, N, S, group = 64, 8, 40, 32
    Wb = synthetic.weights_student_t(K, N, 41)
    Xb = synthetic.calibration(S, K, 42, dtype=synthetic.F16)
    W, X = oracle.decode16(Wb), oracle.decode16(Xb)
    s = awq.scale_candidate(awq.act_stats(X), 0.35)[1]
    q, sb, zz, best, errs = awq.search_clip(X, W, s, group, 0)
    for ci, r in enumerate(awq.CLIPS):
        _, _, _, D = awq.quantize_scaled(W, s, group, 0, r)
        delta = W - D / s[:, None]
        for g in range(K // group):
            rows = slice(g * group, (g + 1) * group)
            direct = np.sum((X[:, rows] @ delta[rows]) ** 2, axis=0)
            assert np.allclose(errs[ci, g], direct, rtol=1e-10, atol=0)
    assert np.all(np.min(errs, axis=0) <= errs[0])


def test_constant_activation_magnitudes_give_unit_factors():
    """|x| = 1 everywhere: a_j = 1, every candidate factor is 1, every alpha ties, the first wins."""
    K, N, S = 128, 16, 32
    rng = np.random.default_rng(3)
    X = np.where(rng.random((S, K)) < 0.5, -1.0, 1.0)
    W = oracle.decode16(synthetic.weights_normal(K, N, 43))
    ai, errs = awq.search_scale(X, W, 64, 0)
    assert ai == 0 and len(set(errs)) == 1


@pytest.mark.parametrize("sym", [0, 1])
def test_awq_lowers_the_output_error_of_rtn_on_outlier_channels(sym):
    K, N, S, group = 256, 64, 256, 64
    Wb = synthetic.weights_normal(K, N, 44)
    Xb = synthetic.calibration(S, K, 45, dtype=synthetic.F16, outlier_frac=0.02, outlier_mult=30.0)
    W, X = oracle.decode16(Wb), oracle.decode16(Xb)
    codes, scales, zeros, sbits, ai = awq.awq(Wb, Xb, synthetic.F16, group, sym)
    s = oracle.decode16(sbits)
    D = oracle.dequant(codes, scales, zeros, K, N, group, sym)
    e_awq = awq.output_error(X, W, s, D)
    st, oc, os_, oz = oracle.quantize(Wb, group, sym)
    e_rtn = awq.output_error(X, W, np.ones(K), oracle.dequant(oc, os_, oz, K, N, group, sym))
    assert ai > 0
    assert e_awq < 0.8 * e_rtn
