"""Pins for the CPU oracle: each test checks it against something other than
itself (exact rational arithmetic, numpy's IEEE conversions, numpy's fp64
matmul, integer matmul, hand-worked values, closed forms), chosen so that a
dropped term, a wrong sign, a wrong group index or a transposed operand fails
at least one of them.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from gemm_w4a16_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f16(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16)


# ------------------------------------------------------------------ fp16 ----

def test_fp16_decode_every_pattern_matches_numpy():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = oracle.fp16_to_double(bits)
    ref = _f16(bits).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_fp16_encode_roundtrips_every_pattern():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = _f16(bits).astype(np.float64)
    keep = ~np.isnan(vals)
    assert np.array_equal(oracle.fp16_from_double(vals[keep]), bits[keep])


def test_fp16_encode_every_dequant_product_matches_numpy():
    """All (q - z) in [-15, 15] times every finite fp16 scale, both signs."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    s = _f16(bits).astype(np.float64)
    s = s[np.isfinite(s)]
    d = np.arange(-15, 16, dtype=np.float64)
    prod = (d[:, None] * s[None, :]).ravel()
    ours = oracle.fp16_from_double(prod)
    with np.errstate(over="ignore"):
        ref = prod.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


def test_fp16_encode_ties_subnormals_overflow_and_random():
    rng = np.random.default_rng(1)
    finite = _f16(np.arange(0x7c00, dtype=np.uint16)).astype(np.float64)
    mids = (finite[:-1] + finite[1:]) / 2          # exact ties between neighbours
    near = np.concatenate([mids, np.nextafter(mids, 0), np.nextafter(mids, 1)])
    rand = np.ldexp(rng.uniform(0.5, 1.0, 200000), rng.integers(-30, 18, 200000))
    edge = np.array([65504.0, 65519.99, 65520.0, 70000.0, 2.0**-25, 2.0**-26,
                     3 * 2.0**-26, 2.0**-14 - 2.0**-25, 1e-30, 0.0])
    x = np.concatenate([near, rand, edge])
    x = np.concatenate([x, -x])
    ours = oracle.fp16_from_double(x)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


def test_dequant_hand_worked_cases():
    rows = []
    with open(os.path.join(GOLDEN, "dequant_cases.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                q, z, s, w = line.split()
                rows.append((int(q), int(z), int(s, 16), int(w, 16)))
    assert len(rows) >= 10
    G = 128
    M = len(rows)
    q = np.zeros((M, G), np.uint8)
    zeros = np.zeros((M, 1), np.uint8)
    scales = np.zeros((M, 1), np.uint16)
    for i, (qq, zz, ss, _) in enumerate(rows):
        q[i, :] = qq
        zeros[i, 0] = zz
        scales[i, 0] = ss
    W = oracle.dequant(q, zeros, scales, G)
    for i, (_, _, _, w) in enumerate(rows):
        assert np.all(W[i] == w), (i, hex(W[i, 0]), hex(w))


# ------------------------------------------------------------- dequant ----

def test_dequant_group_indexing_against_numpy_definition():
    """Groups run along K within one row: k // G picks the scale column."""
    p = synth.make_problem(M=37, K=512, N=1, seed=3)
    W = oracle.dequant(p.q, p.zeros, p.scales, 128)
    g = np.arange(512) // 128
    d = p.q.astype(np.float64) - p.zeros[:, g].astype(np.float64)
    ref = (d * _f16(p.scales)[:, g].astype(np.float64)).astype(np.float16)
    assert np.array_equal(W, ref.view(np.uint16))


def test_dequant_other_group_sizes():
    rng = np.random.default_rng(5)
    for G in (32, 64, 256):
        q, z, s = synth.draw_weights(rng, 9, 512, G)
        W = oracle.dequant(q, z, s, G)
        g = np.arange(512) // G
        ref = ((q.astype(np.float64) - z[:, g]) * _f16(s)[:, g].astype(np.float64))
        assert np.array_equal(W, ref.astype(np.float16).view(np.uint16))


# ------------------------------------------------------------- product ----

def test_brute_force_exact_rational():
    """Exact rational sums; the fp64 oracle must sit within the recursive
    summation bound (K - 1) * 2^-53 * sum |w x| of them."""
    p = synth.make_problem(M=5, K=256, N=3, seed=11)
    y = oracle.gemm(p.q, p.zeros, p.scales, p.x, 128)
    s = _f16(p.scales).astype(np.float64)
    x = _f16(p.x).astype(np.float64)
    for m in range(p.M):
        w = []
        for k in range(p.K):
            g = k // 128
            exact = Fraction(int(p.q[m, k]) - int(p.zeros[m, g])) * Fraction(s[m, g])
            w.append(Fraction(float(np.float16(float(exact)))))   # one RNE rounding
        for n in range(p.N):
            terms = [w[k] * Fraction(x[n, k]) for k in range(p.K)]
            exact_y = sum(terms, Fraction(0))
            bound = (p.K - 1) * 2.0**-53 * float(sum(abs(t) for t in terms))
            assert abs(Fraction(y[n, m]) - exact_y) <= Fraction(bound), (m, n)


def test_matches_numpy_fp64_matmul():
    p = synth.make_problem(M=200, K=384, N=7, seed=2)
    W = oracle.dequant(p.q, p.zeros, p.scales, 128)
    ref = _f16(p.x).astype(np.float64) @ _f16(W).astype(np.float64).T
    y = oracle.gemm(p.q, p.zeros, p.scales, p.x, 128)
    assert y.shape == (7, 200)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_hand_worked_gemm():
    G, K = 128, 128
    q = np.zeros((2, K), np.uint8)
    q[0, :] = 9
    q[1, :] = np.arange(K) % 16
    zeros = np.array([[8], [0]], np.uint8)
    scales = np.array([[0x3800], [0x3C00]], np.uint16)      # 0.5, 1.0
    x = np.empty((2, K), np.float16)
    x[0, :] = 1
    x[1, :] = np.where(np.arange(K) % 2 == 0, 1, -1)
    y = oracle.gemm(q, zeros, scales, x.view(np.uint16), G)
    with open(os.path.join(GOLDEN, "gemm_closed_form.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                n, m, v = line.split()
                assert y[int(n), int(m)] == float(v)


def test_q_equal_z_gives_exact_zero():
    p = synth.make_problem(M=64, K=512, N=4, seed=4)
    g = np.arange(512) // 128
    q = np.ascontiguousarray(p.zeros[:, g])
    y = oracle.gemm(q, p.zeros, p.scales, p.x, 128)
    assert np.all(y == 0.0)


def test_unit_scale_zero_eight_integer_inputs_exact():
    """s = 1, z = 8, x in {-1, 0, 1}: the result is an integer matmul."""
    rng = np.random.default_rng(6)
    M, K, N = 96, 256, 5
    q = rng.integers(0, 16, (M, K), dtype=np.uint8)
    zeros = np.full((M, K // 128), 8, np.uint8)
    scales = np.full((M, K // 128), 0x3C00, np.uint16)
    xi = rng.integers(-1, 2, (N, K))
    y = oracle.gemm(q, zeros, scales, xi.astype(np.float16).view(np.uint16), 128)
    ref = xi.astype(np.int64) @ (q.astype(np.int64) - 8).T
    assert np.array_equal(y, ref.astype(np.float64))


def test_scale_enters_per_group_and_sign():
    """Flipping z and q around 8 negates every output; doubling one group's
    scale changes only that group's share."""
    p = synth.make_problem(M=16, K=256, N=2, seed=8)
    y = oracle.gemm(p.q, p.zeros, p.scales, p.x, 128)
    y_neg = oracle.gemm((15 - p.q).astype(np.uint8), (15 - p.zeros).astype(np.uint8),
                        p.scales, p.x, 128)
    assert np.array_equal(y_neg, -y)
    s2 = p.scales.copy()
    s2[:, 1] = (_f16(p.scales[:, 1]).astype(np.float64) * 2).astype(np.float16).view(np.uint16)
    y2 = oracle.gemm(p.q, p.zeros, s2, p.x, 128)
    W = _f16(oracle.dequant(p.q, p.zeros, p.scales, 128)).astype(np.float64)
    xs = _f16(p.x).astype(np.float64)
    second = xs[:, 128:] @ W[:, 128:].T
    np.testing.assert_allclose(y2 - y, second, rtol=1e-12, atol=1e-12)


def test_gemv_equals_column_of_gemm():
    p = synth.make_problem(M=130, K=256, N=9, seed=9)
    y = oracle.gemm(p.q, p.zeros, p.scales, p.x, 128)
    for j in range(p.N):
        yj = oracle.gemm(p.q, p.zeros, p.scales, p.x[j:j + 1], 128)
        assert np.array_equal(yj[0], y[j])


def test_rows_subset_matches_full():
    p = synth.make_problem(M=300, K=256, N=3, seed=10)
    y = oracle.gemm(p.q, p.zeros, p.scales, p.x, 128)
    rows = np.array([0, 7, 299, 150, 7])
    ys = oracle.gemm_rows(p.q, p.zeros, p.scales, p.x, rows, 128)
    assert np.array_equal(ys, y[:, rows])


def test_thread_count_does_not_change_result():
    p = synth.make_problem(M=257, K=512, N=3, seed=12)
    old = oracle.get_threads()
    try:
        oracle.set_threads(1)
        y1 = oracle.gemm(p.q, p.zeros, p.scales, p.x, 128)
        oracle.set_threads(max(2, os.cpu_count() or 2))
        y2 = oracle.gemm(p.q, p.zeros, p.scales, p.x, 128)
    finally:
        oracle.set_threads(old)
    assert np.array_equal(y1, y2)


def test_rejects_bad_shapes():
    p = synth.make_problem(M=4, K=256, N=1, seed=0)
    with pytest.raises(ValueError):
        oracle.gemm(p.q[:, :200], p.zeros, p.scales, p.x[:, :200], 128)
    with pytest.raises(ValueError):
        oracle.gemm(p.q, p.zeros, p.scales, p.x[:, :128], 128)


# --------------------------------------------------------- synth inputs ----

def test_synthetic_distributions():
    p = synth.make_problem(M=512, K=4096, N=4, seed=0, outlier_frac=0.01)
    assert p.q.min() == 0 and p.q.max() == 15
    assert p.zeros.min() == 0 and p.zeros.max() == 15
    s = _f16(p.scales).astype(np.float64)
    assert s.min() >= 0.001 - 1e-6 and s.max() <= 0.02 + 1e-5
    assert len(p.outliers) == 41 and len(set(p.outliers.tolist())) == 41
    x = np.abs(_f16(p.x).astype(np.float64))
    others = np.setdiff1d(np.arange(4096), p.outliers)
    assert x[:, p.outliers].mean() > 10 * x[:, others].mean()
    again = synth.make_problem(M=512, K=4096, N=4, seed=0, outlier_frac=0.01)
    assert np.array_equal(again.q, p.q) and np.array_equal(again.x, p.x)


# ------------------------------------------------------------ quantiser ----

def _quantize_golden():
    cases = []
    for line in open(os.path.join(GOLDEN, "quantize_cases.txt")):
        line = line.strip()
        if not line.startswith("case "):
            continue
        f = dict(kv.split("=") for kv in line[5:].split())
        runs = [(int(c), int(h, 16)) for c, h in (r.split("x") for r in f["runs"].split(","))]
        codes = [int(v) for v in f["q"].split(",")]
        cases.append((runs, codes, int(f["s"], 16), int(f["z"])))
    return cases


def test_quantize_hand_worked_cases():
    """Hand-derived groups (tests/golden/quantize_cases.txt)."""
    cases = _quantize_golden()
    assert len(cases) == 4
    for runs, codes, s, z in cases:
        w = np.concatenate([np.full(c, h, dtype=np.uint16) for c, h in runs])[None, :]
        q, sc, ze = oracle.quantize(w)
        assert sc[0, 0] == s and ze[0, 0] == z
        got = np.split(q[0], np.cumsum([c for c, _ in runs])[:-1])
        for part, code in zip(got, codes):
            assert np.all(part == code)


@pytest.mark.parametrize("group", [64, 128])
def test_quantize_recovers_values_on_its_grid(group):
    """Weights already on a grid (k - z) s with s a power of two and both
    k = 0 and k = 15 present: the quantiser returns exactly (k, s, z)."""
    rng = np.random.default_rng(11)
    M, K = 6, 4 * group
    q0 = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    q0[:, ::group] = 0
    q0[:, 1::group] = 15
    z0 = rng.integers(0, 16, size=(M, K // group)).astype(np.uint8)
    e = rng.integers(-9, -2, size=(M, K // group))
    s0 = np.ldexp(1.0, e)                                   # exact in fp16
    zf = np.repeat(z0, group, axis=1).astype(np.float64)
    sf = np.repeat(s0, group, axis=1)
    w = ((q0.astype(np.float64) - zf) * sf).astype(np.float16).view(np.uint16)
    q, s, z = oracle.quantize(w, group)
    assert np.array_equal(q, q0)
    assert np.array_equal(z, z0)
    assert np.array_equal(oracle.fp16_to_double(s), s0)


def test_quantize_error_bound_and_ranges():
    """Codes and zeros stay in 0..15, and every weight is reproduced by
    (q - z) s within half a step plus the scale's own fp16 rounding at the
    range ends: |w - (q - z) s| <= s / 2 + |r - 15 s|."""
    rng = np.random.default_rng(12)
    M, K = 32, 1024
    wd = rng.normal(0.0, 0.05, size=(M, K))
    wd[:, ::7] = rng.normal(0.3, 0.1, size=(M, K // 7 + 1))[:, : wd[:, ::7].shape[1]]
    w = wd.astype(np.float16).view(np.uint16)
    q, s, z = oracle.quantize(w)
    assert q.max() <= 15 and z.max() <= 15
    wv = oracle.fp16_to_double(w).reshape(M, K // 128, 128)
    sv = oracle.fp16_to_double(s)[..., None]
    deq = (q.reshape(M, K // 128, 128).astype(np.float64) - z[..., None]) * sv
    lo = np.minimum(wv.min(axis=2, keepdims=True), 0.0)
    hi = np.maximum(wv.max(axis=2, keepdims=True), 0.0)
    bound = 0.5 * sv + np.abs((hi - lo) - 15.0 * sv) + 1e-9
    assert np.all(np.abs(deq - wv) <= bound)


def test_quantize_sign_symmetry_and_scale_invariance():
    """Negating a group mirrors its codes (q -> 15 - q with z -> 15 - z up to
    ties), and multiplying it by a power of two scales s and keeps q, z."""
    rng = np.random.default_rng(13)
    w = rng.normal(0.0, 0.1, size=(4, 256)).astype(np.float16)
    q, s, z = oracle.quantize(w.view(np.uint16))
    q2, s2, z2 = oracle.quantize((w * np.float16(4)).view(np.uint16))
    assert np.array_equal(q, q2) and np.array_equal(z, z2)
    assert np.array_equal(oracle.fp16_to_double(s2), 4 * oracle.fp16_to_double(s))
    qn, sn, zn = oracle.quantize((-w).view(np.uint16))
    assert np.array_equal(sn, s)
    deq = lambda qq, ss, zz: (qq.reshape(4, 2, 128).astype(np.float64) - zz[..., None]) * \
        oracle.fp16_to_double(ss)[..., None]
    assert np.allclose(deq(qn, sn, zn), -deq(q, s, z), atol=float(oracle.fp16_to_double(s).max()))


# ------------------------------------------------ residual add + RMS norm ----

def _bits(vals):
    return np.asarray(vals, dtype=np.float16).view(np.uint16)


def test_add_rmsnorm_closed_form_3_4():
    """r = (1 + 2, 4 + 0) = (3, 4): the mean of squares is 12.5, so
    x = (3, 4) / sqrt(12.5) = (3 sqrt2 / 5, 4 sqrt2 / 5); gamma = (2, 1/2)
    scales channel by channel (swapped channels would give other values)."""
    h, d = _bits([[1.0, 4.0]]), _bits([[2.0, 0.0]])
    r, x = oracle.add_rmsnorm(h, _bits([1.0, 1.0]), 0.0, d=d)
    assert r.tolist() == _bits([[3.0, 4.0]]).tolist()
    s2 = np.sqrt(2.0)
    np.testing.assert_allclose(x[0], [3 * s2 / 5, 4 * s2 / 5], rtol=1e-15, atol=0)
    _, x = oracle.add_rmsnorm(h, _bits([2.0, 0.5]), 0.0, d=d)
    np.testing.assert_allclose(x[0], [6 * s2 / 5, 2 * s2 / 5], rtol=1e-15, atol=0)


def test_add_rmsnorm_residual_rounds_to_nearest_even():
    """In [2048, 4096) fp16 values are 2 apart.  2048 + 1 = 2049 is halfway
    between 2048 and 2050 and goes to the even significand, 2048; 2048 + 3 =
    2051 goes to 2052; 2048 + 0.5 to 2048; -2048 - 1 to -2048.  Without d the
    residual is h bit for bit, a negative zero and a subnormal included."""
    h, d = _bits([[2048, 2048, 2048, -2048]]), _bits([[1, 3, 0.5, -1]])
    r, _ = oracle.add_rmsnorm(h, _bits([1] * 4), 0.0, d=d)
    assert r[0].tolist() == [0x6800, 0x6802, 0x6800, 0xE800]
    h2 = np.array([[0x8000, 0x3C00, 0x0001, 0x7BFF]], dtype=np.uint16)
    r2, _ = oracle.add_rmsnorm(h2, _bits([1] * 4), 0.0)
    assert np.array_equal(r2, h2)


def test_add_rmsnorm_normalises_the_rounded_residual():
    """h = (2048, 1), d = (1, 0): r = (2048, 1) after rounding (not the exact
    2049), so x0 = 2048 / sqrt((2048^2 + 1) / 2); the unrounded sum would be
    off by about 5e-4 relative."""
    _, x = oracle.add_rmsnorm(_bits([[2048, 1]]), _bits([1, 1]), 0.0, d=_bits([[1, 0]]))
    rms = np.sqrt((2048.0 ** 2 + 1.0) / 2.0)
    np.testing.assert_allclose(x[0], [2048.0 / rms, 1.0 / rms], rtol=1e-14, atol=0)


@pytest.mark.parametrize("K", [1, 7, 4096])
def test_add_rmsnorm_constant_row_is_sign_times_gamma(K):
    """A row holding one value c has mean(r^2) = c^2, so with eps = 0,
    x = gamma * c / |c| for every K (a sum in place of the mean would give
    gamma / sqrt(K))."""
    rng = np.random.default_rng(K)
    gamma = rng.normal(1, 0.2, K).astype(np.float16)
    for c in (0.75, -3.0, 2.0 ** -10):
        h = np.full((1, K), c, dtype=np.float16).view(np.uint16)
        _, x = oracle.add_rmsnorm(h, gamma.view(np.uint16), 0.0)
        np.testing.assert_allclose(x[0], np.sign(c) * gamma.astype(np.float64), rtol=1e-15, atol=0)


def test_add_rmsnorm_eps_inside_the_root():
    """c = 2^-10 and eps = 3 * 2^-20: sqrt(c^2 + eps) = sqrt(4 * 2^-20) = 2^-9,
    so x = gamma / 2 exactly; a zero row with eps > 0 gives x = 0."""
    K = 16
    gamma = _bits(np.linspace(0.5, 2.0, K))
    h = np.full((1, K), 2.0 ** -10, dtype=np.float16).view(np.uint16)
    _, x = oracle.add_rmsnorm(h, gamma, 3 * 2.0 ** -20)
    np.testing.assert_array_equal(x[0], _f16(gamma).astype(np.float64) / 2)
    _, x0 = oracle.add_rmsnorm(np.zeros((2, K), np.uint16), gamma, 2.0 ** -20)
    assert np.all(x0 == 0)


def test_add_rmsnorm_scale_invariance_and_row_independence():
    """With eps = 0, scaling h and d by 8 scales r by 8 exactly (fp16 values
    are multiples of 2^-24, so no sum rounds in the subnormal range) and
    leaves x unchanged; a row's result does not depend on the other rows."""
    rng = np.random.default_rng(3)
    N, K = 4, 4096
    h = rng.normal(0, 1, (N, K)).astype(np.float16)
    d = rng.normal(0, 1, (N, K)).astype(np.float16)
    gamma = rng.normal(1, 0.1, K).astype(np.float16).view(np.uint16)
    r, x = oracle.add_rmsnorm(h.view(np.uint16), gamma, 0.0, d=d.view(np.uint16))
    r8, x8 = oracle.add_rmsnorm((h * np.float16(8)).view(np.uint16), gamma, 0.0,
                                d=(d * np.float16(8)).view(np.uint16))
    assert np.array_equal(r8, (_f16(r) * np.float16(8)).view(np.uint16))
    np.testing.assert_allclose(x8, x, rtol=1e-13, atol=0)
    h2 = h.copy()
    h2[0] = rng.normal(0, 5, K).astype(np.float16)
    r2, x2 = oracle.add_rmsnorm(h2.view(np.uint16), gamma, 0.0, d=d.view(np.uint16))
    assert np.array_equal(r2[1:], r[1:]) and np.array_equal(x2[1:], x[1:])
    assert not np.array_equal(x2[0], x[0])


# ------------------------------------------------ gate/up: SiLU(gate) * up ----

# The logistic function at 1, 2 and -1: e/(1+e), e^2/(1+e^2), 1/(1+e).
SIGMA_1 = 0.7310585786300049
SIGMA_2 = 0.8807970779778823
SIGMA_M1 = 0.2689414213699951


def _one_hot_problem(g_vals, u_vals, K=128):
    """s = 1, z = 8 and X = e_0, so the product's row m is q[m][0] - 8 exactly:
    the gate rows hold g_vals, the up rows u_vals."""
    Mi = len(g_vals)
    q = np.full((2 * Mi, K), 8, dtype=np.uint8)
    q[:Mi, 0] = 8 + np.asarray(g_vals)
    q[Mi:, 0] = 8 + np.asarray(u_vals)
    zeros = np.full((2 * Mi, K // 128), 8, dtype=np.uint8)
    scales = np.full((2 * Mi, K // 128), 0x3C00, dtype=np.uint16)       # 1.0
    x = np.zeros((1, K), dtype=np.float16)
    x[0, 0] = 1.0
    return q, zeros, scales, x.view(np.uint16), Mi


def test_gate_up_textbook_logistic_values():
    """silu(g) = g * sigma(g): g = 0, 1, 2, -1 against the logistic function's
    textbook values, each times its own u (row i pairs with row Mi + i)."""
    g, u = [0, 1, 2, -1], [3, 2, 1, 5]
    q, z, s, x, Mi = _one_hot_problem(g, u)
    h = oracle.gate_up(q, z, s, x, Mi)
    expect = [0.0, 1 * SIGMA_1 * 2, 2 * SIGMA_2 * 1, -1 * SIGMA_M1 * 5]
    np.testing.assert_allclose(h[0], expect, rtol=1e-15, atol=0)


def test_gate_up_order_of_gate_and_up_matters():
    """(g, u) = (1, 2) gives 2 sigma(1) = 1.462...; the swapped reading
    silu(u) * g would give 2 sigma(2) = 1.761..."""
    q, z, s, x, Mi = _one_hot_problem([1], [2])
    h = oracle.gate_up(q, z, s, x, Mi)[0, 0]
    assert abs(h - 2 * SIGMA_1) < 1e-15
    assert abs(h - 2 * SIGMA_2) > 0.2


def test_gate_up_odd_symmetry_and_extremes():
    """silu(g) - silu(-g) = g (sigma(g) + sigma(-g) = 1) for every g; far
    negative g gives 0 (exp overflows to infinity, no NaN), far positive g
    gives g."""
    rng = np.random.default_rng(21)
    g = rng.normal(0, 4, 64)
    y = np.concatenate([np.stack([g, -g]), np.ones((2, 64))], axis=1)
    h = oracle.silu_mul(y, 64)
    np.testing.assert_allclose(h[0] - h[1], g, rtol=0, atol=1e-13)
    ext = oracle.silu_mul(np.array([[-1024.0, 40.0, 3.0, 2.0]]), 2)
    assert np.all(np.isfinite(ext)) and ext[0, 0] == 0.0
    assert ext[0, 1] == 80.0                 # 40 * (1 + e^-40)^-1 rounds to 40 in fp64


def test_gate_up_large_negative_accumulator_through_the_product():
    """All gate codes 0 (w = -8) and X = 1 in every channel: g = -1024 exactly,
    so SiLU(g) * u underflows to zero without a NaN."""
    K = 128
    q = np.zeros((2, K), dtype=np.uint8)
    q[1] = 9                                                            # u = K * 1
    zeros = np.full((2, 1), 8, dtype=np.uint8)
    scales = np.full((2, 1), 0x3C00, dtype=np.uint16)
    x = np.ones((1, K), dtype=np.float16).view(np.uint16)
    y = oracle.gemm(q, zeros, scales, x)
    assert y[0, 0] == -1024.0 and y[0, 1] == 128.0
    h = oracle.gate_up(q, zeros, scales, x, 1)
    assert h.shape == (1, 1) and h[0, 0] == 0.0


def test_gate_up_rejects_bad_shapes():
    with pytest.raises(ValueError):
        oracle.silu_mul(np.zeros((1, 5)), 2)
    q, z, s, x, Mi = _one_hot_problem([1, 2], [3, 4])
    with pytest.raises(ValueError):
        oracle.gate_up(q, z, s, x, 3)
