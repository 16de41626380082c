"""Pins for the CPU oracle against what the pages and the mathematics fix.

Each test ties the oracle to something other than itself: a worked example
printed on the pages (tests/golden, cited there), a closed form, an invariant
of round-to-nearest quantisation, or brute force on tiny inputs.  Together they
are chosen so that a plausible slip in the oracle (a dropped term, a wrong sign
or index, a transposed operand, the wrong rounding rule) fails at least one.
"""
import math

import numpy as np
import pytest

F32 = np.float32


def f32(x):
    return np.asarray(x, dtype=np.float32)


# ---------------------------------------------------------------------------
# Worked examples printed on the pages
# ---------------------------------------------------------------------------

def test_weight_rtn_worked_example(oracle, golden):
    """Per-output-channel scale max|w|/127 and round(w/scale): "Understanding
    W8A8 INT8 LLM Quantization", "Why Naive Weight Quantization Doesn't Work"."""
    g = golden("weight_rtn_example.json")
    w = f32([g["w_page_columns"]["ch0"], g["w_page_columns"]["ch1"]])  # [N=2, K=3]
    s = np.ones(3, F32)
    wq, sw = oracle.smooth_quant_weight(w, s)
    for i, ch in enumerate(("ch0", "ch1")):
        # the scales the page prints (4 significant digits)
        assert float(sw[i]) == pytest.approx(g["scales_page"][ch], rel=5e-4)
        assert wq[i].tolist() == g["q_expected"][ch]
    # every printed code except the page's arithmetic slip matches the page
    diffs = [(ch, k) for ch in ("ch0", "ch1") for k in range(3)
             if g["q_page"][ch][k] != g["q_expected"][ch][k]]
    assert diffs == [("ch1", 1)]
    # reconstruction and the page's output for x = [1, 2, 0.5]
    x = np.asarray(g["x_page"], np.float64)
    rec = wq.astype(np.float64) * sw.astype(np.float64)[:, None]
    for i, ch in enumerate(("ch0", "ch1")):
        assert rec[i] == pytest.approx(g["reconstructed_expected"][ch], abs=6e-5)
        assert float(rec[i] @ x) == pytest.approx(g["y_reconstructed_expected"][ch], abs=6e-4)
        assert float(w[i].astype(np.float64) @ x) == pytest.approx(g["y_original_page"][ch], abs=1e-6)
    # the page's own (slipped) code reproduces its printed 2.193
    q_slip = np.asarray(g["q_page"]["ch1"], np.float64) * float(sw[1])
    assert float(q_slip @ x) == pytest.approx(g["y_reconstructed_page"]["ch1"], abs=6e-4)


def test_activation_outlier_worked_example(oracle, golden):
    """One dynamic scale per token across all channels: "Why Activation
    Quantization Is Hard, and How SmoothQuant Fixes It"."""
    g = golden("activation_outlier_example.json")
    x = f32([g["x"]])
    xq, sx = oracle.quant_act(x, np.ones(4, F32))
    assert float(sx[0]) == pytest.approx(g["scale_page"], rel=5e-4)
    assert xq[0].tolist() == g["q_expected"] == g["q_page"]


def test_smoothed_activation_worked_example(oracle, golden):
    """Dividing the outlier channel by s removes the outlier: "Where the outlier
    actually comes from" (gamma of channel 3 divided by 100)."""
    g = golden("smoothed_activation_example.json")
    x = f32([g["x_before_smoothing"]])
    s = f32(g["s"])
    xq, sx = oracle.quant_act(x, s)
    assert float(sx[0]) == pytest.approx(g["scale_page"], rel=2e-2)  # page prints 0.012
    assert float(sx[0]) == float(F32(1.53) / F32(127.0))
    assert xq[0].tolist() == g["q_expected"]
    # the page's printed 63 is reproduced only by its rounded scale and half-up rounding
    assert math.floor(0.75 / g["scale_page"] + 0.5) == g["q_page"][1]


# ---------------------------------------------------------------------------
# Rounding rule, clamping, zero scales
# ---------------------------------------------------------------------------

def test_round_half_to_even_activation(oracle):
    """amax = 127 gives scale exactly 1, so exact .5 quotients expose the tie rule."""
    row = f32([[127.0, 2.5, 3.5, -2.5, 0.5, 1.5, -126.5, 126.5]])
    xq, sx = oracle.quant_act(row, np.ones(8, F32))
    assert float(sx[0]) == 1.0
    assert xq[0].tolist() == [127, 2, 4, -2, 0, 2, -126, 126]


def test_round_half_to_even_weight(oracle):
    w = f32([[-127.0, 2.5, 3.5, -0.5, 5.5, -6.5, 0.0, 1.0]])
    wq, sw = oracle.smooth_quant_weight(w, np.ones(8, F32))
    assert float(sw[0]) == 1.0
    assert wq[0].tolist() == [-127, 2, 4, 0, 6, -6, 0, 1]


def test_symmetric_range_never_minus_128(oracle):
    rng = np.random.default_rng(1)
    x = f32(rng.standard_normal((64, 96)) * 5)
    xq, _ = oracle.quant_act(x, np.ones(96, F32))
    assert xq.min() >= -127 and xq.max() <= 127
    w = f32(rng.standard_normal((64, 96)))
    wq, _ = oracle.smooth_quant_weight(w, np.ones(96, F32))
    assert wq.min() >= -127


def test_zero_rows_and_channels(oracle):
    x = np.zeros((3, 16), F32)
    x[1, 5] = -2.0
    xq, sx = oracle.quant_act(x, np.ones(16, F32))
    assert sx.tolist() == [0.0, float(F32(2.0) / F32(127.0)), 0.0]
    assert not xq[0].any() and not xq[2].any() and xq[1, 5] == -127
    w = np.zeros((2, 16), F32)
    w[0, 3] = 0.5
    wq, sw = oracle.smooth_quant_weight(w, np.ones(16, F32))
    assert sw[1] == 0.0 and not wq[1].any() and wq[0, 3] == 127
    # degenerate channels are not migrated
    s = oracle.smooth_factors(f32([0.0, 3.0, 2.0]), f32([1.0, 0.0, 2.0]), 0.5)
    assert s.tolist() == [1.0, 1.0, 1.0]


# ---------------------------------------------------------------------------
# Smoothing factor: closed forms and the alpha special cases
# ---------------------------------------------------------------------------

def test_smooth_factor_closed_forms(oracle):
    ax = f32([100.0, 4.0, 32.0, 7.25, 1e-3])
    aw = f32([1.0, 16.0, 0.5, 7.25, 0.04])
    s = oracle.smooth_factors(ax, aw, 0.5)
    assert s[0] == 10.0 and s[1] == 0.5 and s[3] == 1.0
    assert s[4] == pytest.approx(math.sqrt(1e-3 / 0.04), rel=1e-6)
    # alpha = 0.8: 32^0.8 / 0.5^0.2 = 2^4 * 2^0.2 = 2^4.2
    s8 = oracle.smooth_factors(ax, aw, 0.8)
    a = float(F32(0.8))  # the fp32 argument, widened
    assert s8[2] == F32(32.0 ** a / 0.5 ** (1.0 - a))
    assert float(s8[2]) == pytest.approx(2 ** 4.2, rel=1e-6)


def test_smooth_factor_alpha_one_is_activation_absmax(oracle):
    rng = np.random.default_rng(2)
    ax = f32(np.abs(rng.standard_normal(257)) * 30 + 0.01)
    aw = f32(np.abs(rng.standard_normal(257)) * 0.1 + 1e-4)
    s = oracle.smooth_factors(ax, aw, 1.0)
    assert np.array_equal(s, ax)


def test_smooth_factor_alpha_zero_depends_only_on_weight(oracle):
    """alpha = 0: s_j = 1 / B_j, independent of the calibration statistics."""
    rng = np.random.default_rng(3)
    aw = f32(np.abs(rng.standard_normal(300)) * 0.1 + 1e-4)
    s1 = oracle.smooth_factors(f32(np.abs(rng.standard_normal(300)) + 1), aw, 0.0)
    s2 = oracle.smooth_factors(f32(np.abs(rng.standard_normal(300)) * 50 + 1), aw, 0.0)
    assert np.array_equal(s1, s2)
    assert np.array_equal(s1, (1.0 / aw.astype(np.float64)).astype(F32))


def test_alpha_zero_unit_weight_leaves_x_unchanged(oracle):
    """The plain reading of "alpha near zero preserves the original
    distribution": with every weight input channel's absmax equal to 1 the
    factors are all 1 and X/s is X bit for bit."""
    rng = np.random.default_rng(4)
    K = 64
    w = f32(rng.uniform(-1, 1, (32, K)))
    w[0, :] = 1.0
    xcal = f32(rng.standard_normal((40, K)) * 9)
    ax, aw, s, _, _ = oracle.prepare(xcal, w, 0.0)
    assert np.all(aw == 1.0) and np.all(s == 1.0)
    x = f32(rng.standard_normal((5, K)))
    a = oracle.quant_act(x, s)
    b = oracle.quant_act(x, np.ones(K, F32))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_alpha_one_flattens_calibration_channels(oracle):
    """alpha = 1 migrates all difficulty: every calibration channel of X/s has
    absmax exactly 1 (a / a = 1 in IEEE arithmetic)."""
    rng = np.random.default_rng(5)
    K = 48
    xcal = f32(rng.standard_normal((30, K)) * rng.uniform(0.1, 80, K))
    w = f32(rng.standard_normal((16, K)) * 0.02)
    ax, aw, s, _, _ = oracle.prepare(xcal, w, 1.0)
    assert np.array_equal(s, ax)
    assert np.all(np.max(np.abs(xcal / s), axis=0) == 1.0)


def test_smooth_factor_monotone(oracle):
    """A larger calibration outlier gives a larger s (for alpha > 0); a larger
    weight range gives a smaller one (for alpha < 1)."""
    ax = f32([1.0, 2.0, 10.0, 100.0])
    s = oracle.smooth_factors(ax, f32([0.1] * 4), 0.5)
    assert np.all(np.diff(s) > 0)
    s = oracle.smooth_factors(f32([5.0] * 4), ax, 0.5)
    assert np.all(np.diff(s) < 0)


# ---------------------------------------------------------------------------
# Calibration absmax
# ---------------------------------------------------------------------------

def test_calib_absmax_bruteforce_and_merge(oracle):
    rng = np.random.default_rng(6)
    x = f32(rng.standard_normal((37, 80)) * 3)
    ax = oracle.calib_absmax(x)
    assert np.array_equal(ax, np.abs(x).max(axis=0))
    # statistics of two calibration batches merge by max
    a1 = oracle.calib_absmax(x[:20])
    a2 = oracle.calib_absmax(x[20:])
    assert np.array_equal(ax, np.maximum(a1, a2))
    # bf16 input: exact widening
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    axb = oracle.calib_absmax(xb)
    assert np.array_equal(axb, np.abs(oracle.bf16_bits_to_f32(xb)).max(axis=0))


def test_small_workload_outliers_dominate_calibration(oracle):
    from w8a8_int8_gemm_channel_b200 import workloads as wls

    wl = wls.WORKLOADS["small"]
    lin = wl.linears[0]
    xcal = wls.calibration(wl, lin).numpy()
    ax = oracle.calib_absmax(xcal)
    assert sorted(np.argsort(ax)[-4:].tolist()) == [3, 77, 150, 201]


# ---------------------------------------------------------------------------
# Smoothing: identity and direction
# ---------------------------------------------------------------------------

def _small_case(oracle):
    from w8a8_int8_gemm_channel_b200 import workloads as wls

    wl = wls.WORKLOADS["small"]
    lin = wl.linears[0]
    xcal = wls.calibration(wl, lin).numpy()
    w = wls.weight(wl, lin).numpy()
    x = wls.inputs(wl, lin, 16).numpy()
    return wl, xcal, w, x


def test_smoothing_identity_fp64(oracle):
    """(X diag(s)^-1)(W diag(s))^T = X W^T to 1e-10 relative in fp64."""
    wl, xcal, w, x = _small_case(oracle)
    _, _, s, _, _ = oracle.prepare(xcal, w, wl.alpha)
    assert s.max() > 5 * np.median(s)  # the outlier channels were migrated
    smoothed, plain = oracle.smoothing_identity_fp64(x, w, s)
    rel = np.linalg.norm(smoothed - plain) / np.linalg.norm(plain)
    assert rel < 1e-10


def test_smoothing_direction(oracle):
    """The weight's INPUT channel k is multiplied by s_k and the activation
    channel k divided by it; the dequantised operands reproduce W diag(s) and
    X diag(s)^-1 to within half a quantisation step."""
    wl, xcal, w, x = _small_case(oracle)
    _, _, s, wq, sw = oracle.prepare(xcal, w, wl.alpha)
    ws = w.astype(np.float64) * s.astype(np.float64)[None, :]
    err_w = np.abs(wq * sw.astype(np.float64)[:, None] - ws)
    assert np.all(err_w <= sw.astype(np.float64)[:, None] * (0.5 + 1e-5))
    xq, sx = oracle.quant_act(x, s)
    xs = x.astype(np.float64) / s.astype(np.float64)[None, :]
    err_x = np.abs(xq * sx.astype(np.float64)[:, None] - xs)
    assert np.all(err_x <= sx.astype(np.float64)[:, None] * (0.5 + 1e-5))
    # the max-magnitude element of every nonzero row lands on +-127
    assert np.all(np.abs(xq).max(axis=1) == 127)
    assert np.all(np.abs(wq).max(axis=1) == 127)


def test_scales_are_per_token_and_per_output_channel(oracle):
    """Scaling one token row by 2 doubles only its scale; scaling one output
    row of W by 2 doubles only its scale; the codes stay put."""
    rng = np.random.default_rng(7)
    x = f32(rng.standard_normal((6, 32)))
    s = f32(rng.uniform(0.5, 4, 32))
    xq, sx = oracle.quant_act(x, s)
    x2 = x.copy()
    x2[2] *= 2
    xq2, sx2 = oracle.quant_act(x2, s)
    assert np.array_equal(xq, xq2)
    assert sx2[2] == 2 * sx[2] and np.array_equal(np.delete(sx, 2), np.delete(sx2, 2))
    w = f32(rng.standard_normal((5, 32)))
    wq, sw = oracle.smooth_quant_weight(w, s)
    w2 = w.copy()
    w2[3] *= 2
    wq2, sw2 = oracle.smooth_quant_weight(w2, s)
    assert np.array_equal(wq, wq2)
    assert sw2[3] == 2 * sw[3] and np.array_equal(np.delete(sw, 3), np.delete(sw2, 3))


def test_quant_act_row_subset(oracle):
    rng = np.random.default_rng(8)
    x = f32(rng.standard_normal((9, 48)))
    s = f32(rng.uniform(0.5, 4, 48))
    xq, sx = oracle.quant_act(x, s)
    rows = np.array([7, 0, 3])
    xq_r, sx_r = oracle.quant_act(x, s, rows=rows)
    assert np.array_equal(xq_r, xq[rows]) and np.array_equal(sx_r, sx[rows])


def test_smoothing_reduces_quantisation_error(oracle):
    """Sanity signal, not a parity criterion: on the outlier-bearing small
    workload, W8A8 with smoothing is closer to the unquantised X W^T than
    per-token W8A8 without it."""
    wl, xcal, w, x = _small_case(oracle)
    ref = oracle.fp64_reference_linear(x, w)

    def err(alpha):
        if alpha is None:
            s = np.ones(w.shape[1], F32)
            wq, sw = oracle.smooth_quant_weight(w, s)
        else:
            _, _, s, wq, sw = oracle.prepare(xcal, w, alpha)
        y, _, _, _ = oracle.linear(x, s, wq, sw, "f32")
        return np.linalg.norm(y - ref) / np.linalg.norm(ref)

    assert err(wl.alpha) < 0.5 * err(None)


# ---------------------------------------------------------------------------
# int32 GEMM and dequantisation
# ---------------------------------------------------------------------------

def test_gemm_bruteforce_tiny(oracle):
    rng = np.random.default_rng(9)
    for M, N, K in [(1, 1, 1), (2, 3, 5), (8, 8, 8), (3, 7, 4), (5, 2, 8)]:
        xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
        wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
        acc = oracle.gemm_i32(xq, wq)
        for m in range(M):
            for n in range(N):
                ref = 0
                for k in range(K):
                    ref += int(xq[m, k]) * int(wq[n, k])
                assert int(acc[m, n]) == ref
    pairs = oracle.gemm_i32_pairs(xq, wq, [4, 0, 2], [1, 0, 1])
    assert pairs.tolist() == [int(acc[4, 1]), int(acc[0, 0]), int(acc[2, 1])]


def test_int32_accumulator_extremes():
    """|acc| <= K * 127^2 < 2^31 for every K in the workloads (K <= 28672); the bound holds up to K = 133144."""
    from oracle import oracle as o

    K = 28672
    assert K * 127 * 127 < 2 ** 31 and 133144 * 127 * 127 < 2 ** 31 <= 133145 * 127 * 127
    xq = np.full((1, K), 127, np.int8)
    wq = np.full((2, K), -127, np.int8)
    wq[1, ::2] = 127
    acc = o.gemm_i32(xq, wq)
    assert acc.tolist() == [[-K * 127 * 127, 0]]


def test_dequant_against_fp64(oracle):
    """y = (acc * sx) * sw: two correctly rounded fp32 products, so within
    2 ulp (plus the int->float rounding) of the exact product."""
    rng = np.random.default_rng(10)
    acc = rng.integers(-400_000_000, 400_000_000, (7, 9)).astype(np.int32)
    sx = f32(rng.uniform(1e-3, 3, 7))
    sw = f32(rng.uniform(1e-5, 1e-2, 9))
    y = oracle.dequant(acc, sx, sw, "f32")
    exact = acc.astype(np.float64) * sx.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :]
    assert np.all(np.abs(y - exact) <= 3 * 2.0 ** -24 * np.abs(exact))
    # order: acc times the token scale first
    assert np.array_equal(y, (acc.astype(F32) * sx[:, None]) * sw[None, :])
    yb = oracle.dequant(acc, sx, sw, "bf16")
    assert np.array_equal(yb, oracle.f32_to_bf16_bits(y))
    yp = oracle.dequant_pairs(acc[[1, 6], [2, 8]], sx[[1, 6]], sw[[2, 8]], "f32")
    assert np.array_equal(yp, y[[1, 6], [2, 8]])


def test_bf16_round_half_to_even(oracle):
    """bf16 keeps 7 fraction bits: ulp(1) = 2^-7."""
    cases = {
        1.0: 0x3F80,
        1.0 + 2 ** -8: 0x3F80,          # tie -> even (down)
        1.0 + 3 * 2 ** -8: 0x3F82,      # tie -> even (up)
        1.0 + 2 ** -8 + 2 ** -20: 0x3F81,
        -(1.0 + 2 ** -8 + 2 ** -20): 0xBF81,
        3.0e38: 0x7F62,
        0.0: 0x0000,
    }
    got = oracle.f32_to_bf16_bits(f32(list(cases)))
    assert got.tolist() == list(cases.values())
    # a value just below the largest finite fp32 rounds to +inf in bf16
    assert int(oracle.f32_to_bf16_bits(f32([3.4e38]))[0]) == 0x7F80


def test_linear_end_to_end_small(oracle):
    """The whole path on the small workload stays close to fp64 X W^T."""
    wl, xcal, w, x = _small_case(oracle)
    _, _, s, wq, sw = oracle.prepare(xcal, w, wl.alpha)
    y, xq, sx, acc = oracle.linear(x, s, wq, sw, "f32")
    ref = oracle.fp64_reference_linear(x, w)
    assert y.shape == (16, 256) and y.dtype == np.float32
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 0.05


# ---------------------------------------------------------------------------
# RMSNorm with gamma / s folded in, then per-token quantisation ("Understanding
# W8A8 INT8 LLM Quantization", section "Where the outlier actually comes from")
# ---------------------------------------------------------------------------

def test_rmsnorm_gamma_worked_example(oracle, golden):
    """The page's example: gamma = [1, 1, 1, 100] turns a balanced normalised
    vector into an outlier row that destroys three channels; dividing gamma by
    s = [1, 1, 1, 100] restores them."""
    g = golden("rmsnorm_gamma_example.json")
    h = np.array([g["normalized"]], np.float32)
    gamma = np.array(g["gamma"], np.float32)
    s = np.array(g["s"], np.float32)
    folded = oracle.fold_gamma(gamma, s)
    assert folded.tolist() == g["gamma_smoothed_page"]
    q0, _, _ = oracle.rmsnorm_quant(h, gamma, 0.0)
    q1, _, _ = oracle.rmsnorm_quant(h, folded, 0.0)
    assert q0[0].tolist() == g["q_unsmoothed_expected"]
    assert q1[0].tolist() == g["q_smoothed_expected"]


def test_rmsnorm_power_of_two_scale_invariance(oracle):
    """With eps = 0, RMSNorm is invariant to scaling a token by any positive
    number; scaling by 2^k is exact in floating point, so codes, scales and the
    normalised values agree bit for bit (a missing division by the RMS fails)."""
    rng = np.random.default_rng(41)
    h = (rng.standard_normal((6, 640)) * 3).astype(np.float32)
    g = rng.uniform(0.1, 4.0, 640).astype(np.float32)
    q, sx, r = oracle.rmsnorm_quant(h, g, 0.0)
    for k in (-20, 7, 30):
        q2, sx2, r2 = oracle.rmsnorm_quant((h * np.float32(2.0 ** k)).astype(np.float32), g, 0.0)
        assert np.array_equal(q, q2) and np.array_equal(sx, sx2)
        assert np.array_equal(r2 * np.float32(2.0 ** k), r)


def test_rmsnorm_constant_rows_and_zero_rows(oracle):
    """A constant row +-c normalises to +-1 exactly (c a power of two), so the
    smoothed activation is +-g; a zero row stays zero with or without eps."""
    K = 48
    rng = np.random.default_rng(42)
    g = rng.uniform(0.5, 2.0, K).astype(np.float32)
    signs = np.where(np.arange(K) % 3 == 0, -1.0, 1.0).astype(np.float32)
    h = np.stack([signs * 8.0, signs * 0.125, np.zeros(K), np.zeros(K)]).astype(np.float32)
    q, sx, r = oracle.rmsnorm_quant(h[:3], g, 0.0)
    assert r[0] == np.float32(0.125) and r[1] == np.float32(8.0) and r[2] == 0.0
    qa, sxa = oracle.quant_act((signs * g)[None, :].astype(np.float32), np.ones(K, np.float32))
    assert np.array_equal(q[0], qa[0]) and sx[0] == sxa[0]
    assert np.array_equal(q[1], qa[0]) and sx[1] == sxa[0]
    assert not q[2].any() and sx[2] == 0.0
    q, sx, r = oracle.rmsnorm_quant(h[2:], g, 1e-5)
    assert not q.any() and not sx.any()
    assert r[0] == np.float32(1.0 / np.sqrt(np.float64(np.float32(1e-5))))


def test_rmsnorm_against_fp64_closed_form(oracle):
    """max |a| = 127 sx against the exact max_k |h_k| g_k / sqrt(mean(h^2) + eps)
    in fp64 (three roundings), and every code against round(exact / sx) away
    from ties: a sum instead of a mean, a missing square root or eps outside
    the root all fail."""
    rng = np.random.default_rng(43)
    M, K, eps = 12, 1024, 1e-5
    h = (rng.standard_normal((M, K)) * rng.uniform(0.01, 50.0, (M, 1))).astype(np.float32)
    h[:, 17] *= 60.0
    g = rng.uniform(0.05, 3.0, K).astype(np.float32)
    q, sx, r = oracle.rmsnorm_quant(h, g, eps)
    h64 = h.astype(np.float64)
    exact = h64 / np.sqrt((h64 * h64).mean(axis=1, keepdims=True) + np.float64(np.float32(eps))) * g
    amax = np.abs(exact).max(axis=1)
    assert np.allclose(sx.astype(np.float64) * 127.0, amax, rtol=4 * 2.0 ** -24, atol=0)
    t = exact / sx[:, None].astype(np.float64)
    frac = np.abs(t - np.floor(t) - 0.5)
    safe = frac > 1e-4
    assert safe.mean() > 0.99
    assert np.array_equal(q[safe], np.clip(np.rint(t[safe]), -127, 127).astype(np.int8))


def test_rmsnorm_fold_matches_unfused_composition(oracle):
    """Folding gamma / s into the norm gives the codes of quantising
    X / s with X = RMSNorm(h) * gamma, except where the two fp32 rounding
    orders straddle a tie (a fold in the wrong direction, gamma * s, fails)."""
    rng = np.random.default_rng(44)
    M, K = 16, 512
    h = rng.standard_normal((M, K)).astype(np.float32)
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float32)
    gamma[[3, 77]] *= 60.0
    s = rng.uniform(0.5, 2.0, K).astype(np.float32)
    s[[3, 77]] *= 40.0
    q_fold, _, r = oracle.rmsnorm_quant(h, oracle.fold_gamma(gamma, s), 0.0)
    x = ((h * r[:, None]) * gamma).astype(np.float32)
    q_ref, _ = oracle.quant_act(x, s)
    d = np.abs(q_fold.astype(np.int32) - q_ref.astype(np.int32))
    assert d.max() <= 1 and (d == 0).mean() > 0.995


def test_rmsnorm_midpoint_candidate_constructed(oracle):
    """The row [4 - 2^-22, 0, ..., 0] of 16 values: its mean square is
    (1 - 2^-24)^2 exactly, so 1/RMS = 1 / (1 - 2^-24) = 1 + 2^-24 + 2^-48 + ...,
    which lies 2^-48 above the fp32 midpoint between 1 and 1 + 2^-23.  Round
    to nearest gives 1 + 2^-23; another summation order could give 1.  The
    oracle flags the token, and its alternate result is the same definition
    with 1/RMS = 1 (then a = h g exactly, so sx = RN(|h_0 g_0| / 127))."""
    K = 16
    h = np.zeros((2, K), np.float32)
    h[0, 0] = np.float32(4.0 - 2.0 ** -22)
    h[1] = np.linspace(-1.0, 2.0, K, dtype=np.float32)
    g = np.linspace(0.5, 2.0, K, dtype=np.float32)
    c = oracle.rmsnorm_quant_candidates(h, g, 0.0)
    assert c["near"].tolist() == [True, False]
    assert c["rinv"][0] == np.float32(1.0 + 2.0 ** -23)
    assert c["rinv_alt"][0] == np.float32(1.0)
    assert c["sx_alt"][0] == np.float32(np.float32(h[0, 0] * g[0]) / np.float32(127.0))
    assert c["sx"][0] == np.float32(np.float32(np.float32(h[0, 0] * c["rinv"][0]) * g[0]) / np.float32(127.0))
    assert c["xq"][0, 0] == 127 and c["xq_alt"][0, 0] == 127 and not c["xq"][0, 1:].any()
    # an unflagged token's alternate repeats its result
    assert c["rinv_alt"][1] == c["rinv"][1] and np.array_equal(c["xq_alt"][1], c["xq"][1])
    # with a window of 2^-49 the same token is not flagged: the flag follows the stated bound
    c2 = oracle.rmsnorm_quant_candidates(h, g, 0.0, window=2.0 ** -49)
    assert c2["near"].tolist() == [False, False]


def test_rmsnorm_midpoint_candidates_are_the_neighbouring_rounding(oracle):
    """With the window opened to 1 every token is flagged: the alternate 1/RMS
    is the fp32 neighbour on the side of the fp64 value, and the alternate
    codes and scale are the definition evaluated with it (numpy, element by
    element).  With the default window, random tokens are almost never
    flagged (a window that accepted both roundings everywhere would fail)."""
    rng = np.random.default_rng(45)
    M, K = 40, 384
    h = (rng.standard_normal((M, K)) * rng.uniform(0.1, 10.0, (M, 1))).astype(np.float32)
    g = rng.uniform(0.2, 3.0, K).astype(np.float32)
    c = oracle.rmsnorm_quant_candidates(h, g, 1e-5, window=1.0)
    assert c["near"].all()
    h64 = h.astype(np.float64)
    r64 = 1.0 / np.sqrt((h64 * h64).sum(axis=1) / K + np.float64(np.float32(1e-5)))
    up = c["rinv"].astype(np.float64) < r64
    want = np.where(up, np.nextafter(c["rinv"], np.float32(np.inf)), np.nextafter(c["rinv"], np.float32(0)))
    assert np.array_equal(c["rinv_alt"], want.astype(np.float32))
    for m in range(M):
        a = ((h[m] * c["rinv_alt"][m]).astype(np.float32) * g).astype(np.float32)
        sx = np.float32(np.abs(a).max() / np.float32(127.0))
        assert c["sx_alt"][m] == sx
        q = np.clip(np.rint((a / sx).astype(np.float32)), -127, 127).astype(np.int8)
        assert np.array_equal(c["xq_alt"][m], q)
    hb = rng.standard_normal((4000, 512)).astype(np.float32)
    cb = oracle.rmsnorm_quant_candidates(hb, np.ones(512, np.float32), 1e-5)
    assert cb["near"].sum() <= 2


# ---------------------------------------------------------------------------
# The gated feed-forward activation SiLU(gate) * up, quantised for the down
# projection ("Understanding W8A8 INT8 LLM Quantization", section
# "Inter-Token Latency (ITL)": the per-token quantisation is memory-bound work
# worth fusing into the op before it)
# ---------------------------------------------------------------------------

def _bf16_rne_bits(x):
    """Round-half-to-even of finite fp32 values to bf16 bit patterns (numpy)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


def _bf16_bits_f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def test_exp_f32_within_one_ulp_of_fp64(oracle):
    rng = np.random.default_rng(50)
    x = np.concatenate([np.linspace(-87.0, 88.0, 400001),
                        rng.uniform(-87.0, 88.0, 200000),
                        rng.uniform(-1e-3, 1e-3, 20000)]).astype(np.float32)
    y = oracle.exp_f32(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    ulp = np.spacing(ref.astype(np.float32)).astype(np.float64)
    assert (np.abs(y - ref) / ulp).max() <= 1.0
    e = oracle.exp_f32(f32([0.0, -0.0, 1.0, -87.5, -1e30, 88.5, 1e30]))
    assert e[0] == 1.0 and e[1] == 1.0
    assert abs(float(e[2]) - math.e) <= 2.5e-7
    assert e[3] == 0.0 and e[4] == 0.0
    assert np.isinf(e[5]) and np.isinf(e[6]) and e[5] > 0


def test_silu_closed_forms(oracle):
    """SiLU(0) = 0 with the sign of zero kept; SiLU(z) = z once 1 + e^-z rounds
    to 1 (z >= 17); -0 once e^-z overflows; SiLU(z) - SiLU(-z) = z."""
    z = f32([0.0, -0.0])
    s0 = oracle.silu_f32(z)
    assert s0[0] == 0.0 and not np.signbit(s0[0]) and s0[1] == 0.0 and np.signbit(s0[1])
    big = f32(np.concatenate([np.linspace(17.0, 87.0, 5001), [1e3, 1e20, 3e38]]))
    assert np.array_equal(oracle.silu_f32(big), big)
    neg = f32([-88.5, -1e3, -3e38])
    sn = oracle.silu_f32(neg)
    assert np.all(sn == 0.0) and np.all(np.signbit(sn))
    rng = np.random.default_rng(51)
    z = f32(rng.uniform(-10.0, 10.0, 100000))
    d = oracle.silu_f32(z).astype(np.float64) - oracle.silu_f32(-z).astype(np.float64)
    assert np.allclose(d, z.astype(np.float64), rtol=4e-7, atol=1e-6)


def test_silu_within_three_ulp_of_fp64(oracle):
    rng = np.random.default_rng(52)
    z = f32(np.concatenate([np.linspace(-80.0, 80.0, 400001), rng.standard_normal(100000) * 4.0]))
    got = oracle.silu_f32(z).astype(np.float64)
    z64 = z.astype(np.float64)
    ref = z64 / (1.0 + np.exp(-z64))
    ok = ref != 0.0
    ulp = np.spacing(np.abs(ref[ok]).astype(np.float32)).astype(np.float64)
    assert (np.abs(got[ok] - ref[ok]) / ulp).max() <= 3.0


def test_silu_mul_quant_saturated_gate_is_the_product(oracle):
    """For gate >= 17 SiLU(gate) = gate exactly, so h = RN_bf16(gate * up) and
    the codes are those of the plain quantiser on that product: pins the
    [gate | up] order, the rounding of h to bf16 and the division by s."""
    rng = np.random.default_rng(53)
    M, I = 8, 64
    g = _bf16_rne_bits(rng.uniform(17.0, 60.0, (M, I)))
    u = _bf16_rne_bits(rng.standard_normal((M, I)))
    s = f32(rng.uniform(0.5, 2.0, I))
    xq, sx, h = oracle.silu_mul_quant(np.concatenate([g, u], axis=1), s)
    prod_bits = _bf16_rne_bits(_bf16_bits_f32(g) * _bf16_bits_f32(u))  # the fp32 product is exact
    assert np.array_equal(h, _bf16_bits_f32(prod_bits))
    q_ref, sx_ref = oracle.quant_act(prod_bits, s)
    assert np.array_equal(xq, q_ref) and np.array_equal(sx, sx_ref)
    # with gate and up swapped the activation is SiLU(up) * gate, not the same codes
    xq_sw, _, _ = oracle.silu_mul_quant(np.concatenate([u, g], axis=1), s)
    assert not np.array_equal(xq_sw, xq)


def test_silu_mul_quant_against_fp64(oracle):
    """h lies within half a bf16 ulp (plus the fp32 steps) of the fp64 value
    SiLU(gate) * up, and the codes quantise exactly that h."""
    rng = np.random.default_rng(54)
    M, I = 16, 256
    g = _bf16_rne_bits(rng.standard_normal((M, I)) * 3.0)
    u = _bf16_rne_bits(rng.standard_normal((M, I)))
    s = f32(rng.uniform(0.5, 2.0, I))
    xq, sx, h = oracle.silu_mul_quant(np.concatenate([g, u], axis=1), s)
    g64 = _bf16_bits_f32(g).astype(np.float64)
    ref = g64 / (1.0 + np.exp(-g64)) * _bf16_bits_f32(u).astype(np.float64)
    assert np.all(np.abs(h - ref) <= np.abs(ref) * (2.0 ** -8) * (1.0 + 2.0 ** -18) + 1e-38)
    q_ref, sx_ref = oracle.quant_act(_bf16_rne_bits(h), s)
    assert np.array_equal(xq, q_ref) and np.array_equal(sx, sx_ref)


def test_silu_mul_quant_zero_rows_and_fp32(oracle):
    """A zero gate, or a gate whose e^-gate overflows, gives a zero row (scale 0,
    codes 0); fp32 rows keep h = SiLU(gate) * up unrounded."""
    I = 32
    s = np.ones(I, np.float32)
    gu = np.zeros((3, 2 * I), np.float32)
    gu[:, I:] = 1.5
    gu[1, :I] = -100.0
    gu[2, :I] = np.linspace(-3.0, 3.0, I, dtype=np.float32)
    xq, sx, h = oracle.silu_mul_quant(gu, s)
    assert sx[0] == 0.0 and sx[1] == 0.0 and not xq[:2].any()
    assert np.array_equal(h[2], oracle.silu_f32(gu[2, :I]) * np.float32(1.5))
    assert sx[2] == np.float32(np.abs(h[2]).max() / np.float32(127.0))


# ---------------------------------------------------------------------------
# GPTQ weight rounding ("Understanding W8A8 INT8 LLM Quantization", section
# "How GPTQ improves on naive quantization")
# ---------------------------------------------------------------------------

def _correlated_calibration(rng, T, K):
    """Calibration tokens with correlated channels (a few shared factors)."""
    f = rng.standard_normal((T, 6))
    mix = rng.standard_normal((6, K))
    return (f @ mix + 0.3 * rng.standard_normal((T, K))).astype(np.float32)


def test_gptq_hessian_is_the_gram_matrix(oracle):
    rng = np.random.default_rng(70)
    T, K = 96, 48
    x = _correlated_calibration(rng, T, K)
    s = f32(rng.uniform(0.5, 2.0, K))
    H = oracle.gptq_hessian(x, s)
    xh = (x / s).astype(np.float32).astype(np.float64)   # one fp32 division per element
    assert np.allclose(H, xh.T @ xh, rtol=1e-12, atol=1e-12)
    assert np.array_equal(H, H.T)


def test_gptq_damping_closed_forms(oracle):
    rng = np.random.default_rng(71)
    A = rng.standard_normal((20, 20))
    H = A @ A.T
    Hd = oracle.gptq_damp(H, 0.01)
    d = np.diag(Hd) - np.diag(H)
    assert np.allclose(d, 0.01 * np.trace(H) / 20, rtol=1e-14)
    assert np.array_equal(Hd - np.diag(np.diag(Hd)), H - np.diag(np.diag(H)))
    assert np.array_equal(oracle.gptq_damp(np.zeros((5, 5)), 0.01), np.eye(5))


def test_gptq_factor_is_the_cholesky_factor_of_the_inverse(oracle):
    rng = np.random.default_rng(72)
    K = 40
    x = _correlated_calibration(rng, 200, K)
    Hd = oracle.gptq_damp(oracle.gptq_hessian(x, np.ones(K, np.float32)), 0.01)
    U = oracle.gptq_factor(Hd)
    assert np.array_equal(U, np.triu(U)) and (np.diag(U) > 0).all()
    assert np.allclose(U.T @ U @ Hd, np.eye(K), atol=1e-9)
    ref = np.linalg.cholesky(np.linalg.inv(Hd)).T          # numpy / LAPACK, another route
    assert np.allclose(U, ref, rtol=1e-8, atol=1e-12)
    with pytest.raises(ValueError):
        oracle.gptq_factor(-np.eye(4))


def test_gptq_without_correlation_is_plain_rounding(oracle):
    """No calibration signal (H = 0, so U = I after the unit damping), or
    channels that never co-occur (diagonal H): no error is passed on and the
    codes are the plain per-channel rounding's."""
    rng = np.random.default_rng(73)
    N, K = 24, 32
    w = f32(rng.standard_normal((N, K)) * 0.02)
    s = f32(rng.uniform(0.5, 2.0, K))
    q_rtn, sw_rtn = oracle.smooth_quant_weight(w, s)
    for x in (np.zeros((16, K), np.float32),
              np.eye(K, dtype=np.float32) * f32(rng.uniform(0.5, 3.0, K))[:, None]):
        q, sw, U = oracle.gptq(x, w, s)
        assert np.array_equal(U, np.diag(np.diag(U)))
        assert np.array_equal(q, q_rtn) and np.array_equal(sw, sw_rtn)


@pytest.mark.parametrize("damp", [0.01, 0.0])
def test_gptq_against_brute_force_obs(oracle, damp):
    """Tiny layers against the explicit form of the method: after rounding
    weight k, spread its error over the remaining weights with the inverse of
    the Hessian restricted to them, inverted afresh by numpy at every step.
    Undamped too (64 tokens of 10 channels: H is positive definite)."""
    rng = np.random.default_rng(74)
    N, K = 12, 10
    x = _correlated_calibration(rng, 64, K)
    w = f32(rng.standard_normal((N, K)) * 0.05)
    s = np.ones(K, np.float32)
    q, sw, _ = oracle.gptq(x, w, s, damp_frac=damp)
    Hd = oracle.gptq_damp(oracle.gptq_hessian(x, s), damp)
    for n in range(N):
        r = w[n].astype(np.float64).copy()
        sc = float(np.float32(np.abs(w[n]).max() / np.float32(127.0)))
        codes = []
        for k in range(K):
            qk = float(np.clip(np.rint(r[k] / sc), -127, 127))
            codes.append(int(qk))
            Hi = np.linalg.inv(Hd[k:, k:])
            e = (r[k] - qk * sc) / Hi[0, 0]
            r[k + 1:] -= e * Hi[0, 1:]
        assert codes == q[n].tolist(), n
        assert sw[n] == np.float32(sc)


def test_gptq_reduces_output_error(oracle):
    """The point of the method: on the calibration tokens the layer's output
    error X (W' - Q)^T is smaller than plain rounding's."""
    rng = np.random.default_rng(75)
    N, K = 64, 96
    x = _correlated_calibration(rng, 512, K)
    w = f32(rng.standard_normal((N, K)) * 0.02)
    s = f32(rng.uniform(0.7, 1.5, K))
    q, sw, _ = oracle.gptq(x, w, s)
    q_rtn, sw_rtn = oracle.smooth_quant_weight(w, s)
    xh = (x / s).astype(np.float64)
    wp = (w * s).astype(np.float64)
    err = lambda qq, ss: np.linalg.norm(xh @ (wp - qq.astype(np.float64) * ss.astype(np.float64)[:, None]).T)
    assert err(q, sw) < 0.8 * err(q_rtn, sw_rtn)


def test_gptq_page_example_first_weight(oracle, golden):
    """The page's channel: the first weight is rounded exactly as plain
    rounding does (0.31 -> code 43, 0.3088 reconstructed), and with the page's
    input as the calibration token the channel's output ends closer to the
    original than plain rounding's."""
    g = golden("weight_rtn_example.json")
    w = f32([g["w_page_columns"]["ch0"], g["w_page_columns"]["ch1"]])
    x = f32([g["x_page"]])
    s = np.ones(3, F32)
    q, sw, _ = oracle.gptq(x, w, s)
    q_rtn, _ = oracle.smooth_quant_weight(w, s)
    assert q[:, 0].tolist() == q_rtn[:, 0].tolist()
    assert float(q[0, 0]) * float(sw[0]) == pytest.approx(0.3088, abs=6e-5)
    xv = np.asarray(g["x_page"], np.float64)
    for i in range(2):
        y0 = float(w[i].astype(np.float64) @ xv)
        yg = float((q[i] * np.float64(sw[i])) @ xv)
        yr = float((q_rtn[i] * np.float64(sw[i])) @ xv)
        assert abs(yg - y0) <= abs(yr - y0)
