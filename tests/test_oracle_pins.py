"""Pins for the fp64 oracle: each test ties one oracle routine to something other
than itself -- a hand-worked example, a closed form, an invariant, brute force
with Python complex numbers, or exact rational arithmetic.  CPU only."""
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
from conftest import read_golden


# ---------------------------------------------------------------------------
# Phase rule
# ---------------------------------------------------------------------------
def _grid_points():
    """fp32 grid: integer lattice -4..4, diagonal neighbours at many magnitudes,
    subnormals and signed zeros (as float64 arrays of fp32 values)."""
    pts = []
    ints = np.arange(-4, 5, dtype=np.float32)
    for a in ints:
        for b in ints:
            pts.append((a, b))
    mags = np.array([1.4e-45, 1e-40, 1.17549435e-38, 1e-30, 1e-3, 0.02, 1.0, 3.7, 1e20, 3e38], np.float32)
    for m in mags:
        up = np.nextafter(m, np.float32(np.inf))
        dn = np.nextafter(m, np.float32(0))
        for s1 in (1, -1):
            for s2 in (1, -1):
                for (u, v) in ((m, m), (m, up), (up, m), (m, dn), (dn, m)):
                    pts.append((np.float32(s1 * u), np.float32(s2 * v)))
    for z1 in (0.0, -0.0):
        for z2 in (0.0, -0.0, 1.0, -1.0, 1e-45, -1e-45):
            pts.append((np.float32(z1), np.float32(z2)))
            pts.append((np.float32(z2), np.float32(z1)))
    a = np.array([p[0] for p in pts], np.float32).astype(np.float64)
    b = np.array([p[1] for p in pts], np.float32).astype(np.float64)
    return a, b


def test_phase_rule_exact_form_matches_atan2_form_on_fp32_grid():
    a, b = _grid_points()
    assert a.size > 300
    np.testing.assert_array_equal(O.phase_code(a, b), O.phase_code_atan2(a, b))


def test_phase_rule_exact_form_matches_atan2_form_on_random_fp32():
    rng = np.random.default_rng(123)
    a = rng.standard_normal(200000).astype(np.float32).astype(np.float64)
    b = rng.standard_normal(200000).astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(O.phase_code(a, b), O.phase_code_atan2(a, b))


def test_phase_rule_hand_sector_table():
    rows = read_golden("phase_rule_sectors.txt")
    a = np.array([float(r[0]) for r in rows])
    b = np.array([float(r[1]) for r in rows])
    want = np.array([int(r[2]) for r in rows], np.uint8)
    np.testing.assert_array_equal(O.phase_code(a, b), want)
    np.testing.assert_array_equal(O.phase_code_atan2(a, b), want)


def test_phase_rule_matches_nearest_codeword_off_ties():
    """Away from ties the rule picks the codeword nearest to w/|w| (brute force over 4 entries)."""
    rng = np.random.default_rng(7)
    w = rng.standard_normal(5000) + 1j * rng.standard_normal(5000)
    u = w / np.abs(w)
    dist = np.abs(u[:, None] - np.array(O.CODEBOOK)[None, :])
    want = np.argmin(dist, axis=1).astype(np.uint8)
    np.testing.assert_array_equal(O.phase_code(w.real, w.imag), want)


def test_phase_rule_rotation_equivariance():
    """k(i w) = k(w) + 1 and k(-w) = k(w) + 2 (mod 4) for w != 0; i w = -b + i a is exact."""
    a, b = _grid_points()
    rng = np.random.default_rng(11)
    a = np.concatenate([a, rng.standard_normal(5000)])
    b = np.concatenate([b, rng.standard_normal(5000)])
    nz = ~((a == 0) & (b == 0))
    a, b = a[nz], b[nz]
    k = O.phase_code(a, b).astype(np.int64)
    np.testing.assert_array_equal(O.phase_code(-b, a), (k + 1) % 4)
    np.testing.assert_array_equal(O.phase_code(-a, -b), (k + 2) % 4)


def test_times_i_is_swap_and_negate():
    """("iFairy talk notes" §2.3.1) i (a + ib) = -b + ia for every bf16 pair tried."""
    rng = np.random.default_rng(5)
    xr = O.bf16_round(rng.standard_normal(1000).astype(np.float32)).astype(np.float64)
    xi = O.bf16_round(rng.standard_normal(1000).astype(np.float32)).astype(np.float64)
    for r, i in zip(xr, xi):
        z = 1j * complex(r, i)
        assert z.real == -i and z.imag == r


def test_codebook_br_bi():
    br, bi = O.code_to_br_bi(np.arange(4, dtype=np.uint8))
    for k in range(4):
        assert complex(int(br[k]), int(bi[k])) == O.CODEBOOK[k]
    # exactly one of Re, Im is zero for every codeword ("iFairy article" §二.1)
    assert np.all((br == 0) ^ (bi == 0))


# ---------------------------------------------------------------------------
# Scales and residual stages
# ---------------------------------------------------------------------------
def test_two_stage_hand_example():
    g = {r[0]: r[1:] for r in read_golden("two_stage_example.txt")}
    w_re = np.array([float(v) for v in g["w_re"]], np.float32)[None, :]
    w_im = np.array([float(v) for v in g["w_im"]], np.float32)[None, :]
    packed, scales, _ = O.quantize_tensor(w_re, w_im, 2)
    k = O.unpack_codes(packed[:, 0])
    np.testing.assert_array_equal(k[0], [int(v) for v in g["k1"]])
    np.testing.assert_array_equal(k[1], [int(v) for v in g["k2"]])
    assert scales[0, 0] == np.float32(float(g["s1"][0]))
    assert scales[0, 1] == np.float32(float(g["s1"][1]))
    assert scales[1, 0] == np.float32(Fraction(17, 12))   # 4.25 / 3
    assert scales[1, 1] == np.float32(float(g["s2"][1]))
    assert list(packed[0, 0]) == [int(v, 16) for v in g["bytes1"]]
    assert list(packed[1, 0]) == [int(v, 16) for v in g["bytes2"]]


def _stage_python_loop(a, b):
    """Element-by-element stage with Python floats and the atan2 form (independent route)."""
    S = [0.0, 0.0]
    C = [0, 0]
    ks = []
    for x, y in zip(a.ravel().tolist(), b.ravel().tolist()):
        k = int(O.phase_code_atan2(np.array([x]), np.array([y]))[0])
        ks.append(k)
        if k % 2 == 0:
            S[0] += abs(x)
            C[0] += 1
        else:
            S[1] += abs(y)
            C[1] += 1
    return np.array(ks, np.uint8).reshape(a.shape), S, C


def test_quantize_stage_matches_python_loop():
    rng = np.random.default_rng(3)
    a = (0.02 * rng.standard_normal((6, 16))).astype(np.float32).astype(np.float64)
    b = (0.02 * rng.standard_normal((6, 16))).astype(np.float32).astype(np.float64)
    k, (s_re, s_im), sums = O.quantize_stage(a, b)
    k2, S, C = _stage_python_loop(a, b)
    np.testing.assert_array_equal(k, k2)
    assert sums[1] == C[0] and sums[3] == C[1]
    assert abs(sums[0] - S[0]) <= 1e-15 * S[0] and abs(sums[2] - S[1]) <= 1e-15 * S[1]
    assert s_re == np.float32(S[0] / C[0]) and s_im == np.float32(S[1] / C[1])


def test_energy_identity_and_least_squares():
    """||r_{t+1}||^2 = ||r_t||^2 - C_re s_re^2 - C_im s_im^2 when s is the class mean
    (codes carry sign(Re r) on +-1 entries, sign(Im r) on +-i entries); any other scale is worse."""
    rng = np.random.default_rng(9)
    a = (0.02 * rng.standard_normal((64, 96))).astype(np.float32).astype(np.float64)
    b = (0.02 * rng.standard_normal((64, 96))).astype(np.float32).astype(np.float64)
    for _stage in range(3):
        k, _, (S_re, C_re, S_im, C_im) = O.quantize_stage(a, b)
        s_re, s_im = S_re / C_re, S_im / C_im
        br, bi = O.code_to_br_bi(k)

        def energy(sr, si):
            return float(np.sum((a - sr * br) ** 2 + (b - si * bi) ** 2))

        e0 = float(np.sum(a * a + b * b))
        e1 = energy(s_re, s_im)
        want = e0 - C_re * s_re ** 2 - C_im * s_im ** 2
        assert abs(e1 - want) <= 1e-12 * e0
        for eps in (1e-3, -1e-3):
            assert energy(s_re * (1 + eps), s_im) > e1
            assert energy(s_re, s_im * (1 + eps)) > e1
        a, b = a - s_re * br, b - s_im * bi


def test_real_only_weights_reduce_to_sign_binarisation():
    """Im w = 0: codes are +-1 by sign(Re w), s_re = mean |w| (binary-weight rule), s_im = 0."""
    rng = np.random.default_rng(4)
    w = (0.02 * rng.standard_normal((8, 32))).astype(np.float32)
    packed, scales, _ = O.quantize_tensor(w, np.zeros_like(w), 1)
    k = O.unpack_codes(packed[0])
    np.testing.assert_array_equal(k, np.where(w >= 0, 0, 2))
    assert scales[0, 0] == np.float32(np.mean(np.abs(w.astype(np.float64))))
    assert scales[0, 1] == 0.0


def test_scales_swap_under_multiplication_by_i():
    rng = np.random.default_rng(6)
    a = (0.02 * rng.standard_normal((16, 64))).astype(np.float32)
    b = (0.03 * rng.standard_normal((16, 64))).astype(np.float32)
    p1, s1, _ = O.quantize_tensor(a, b, 2)
    p2, s2, _ = O.quantize_tensor(-b, a, 2)     # i w
    assert s1[0, 0] == s2[0, 1] and s1[0, 1] == s2[0, 0]
    k1 = O.unpack_codes(p1[0]).astype(int)
    k2 = O.unpack_codes(p2[0]).astype(int)
    np.testing.assert_array_equal(k2, (k1 + 1) % 4)


def test_isotropic_gaussian_codes_are_uniform():
    """Isotropic weights use the four codewords equally (cf. "iFairy article" §四), within 5 sigma."""
    rng = np.random.default_rng(0)
    n = 400000
    k = O.phase_code(rng.standard_normal(n), rng.standard_normal(n))
    counts = np.bincount(k, minlength=4)
    sigma = np.sqrt(n * 0.25 * 0.75)
    assert np.all(np.abs(counts - n / 4) < 5 * sigma)


def test_second_stage_is_rule_on_complex_residual():
    """Stage 2 codes equal the rule applied to w - w_hat_1 formed with complex arithmetic."""
    rng = np.random.default_rng(8)
    wr = (0.02 * rng.standard_normal((12, 40))).astype(np.float32)
    wi = (0.02 * rng.standard_normal((12, 40))).astype(np.float32)
    packed, scales, _ = O.quantize_tensor(wr, wi, 2)
    w_hat1 = O.dequantize(packed[:1], scales[:1])
    r = (wr.astype(np.float64) + 1j * wi.astype(np.float64)) - w_hat1
    np.testing.assert_array_equal(O.unpack_codes(packed[1]), O.phase_code(r.real, r.imag))


def test_chunked_quantizer_matches_whole_tensor():
    rng = np.random.default_rng(10)
    wr = (0.02 * rng.standard_normal((37, 24))).astype(np.float32)
    wi = (0.02 * rng.standard_normal((37, 24))).astype(np.float32)
    p1, s1, _ = O.quantize_tensor(wr, wi, 3)
    p2, s2, _ = O.quantize_tensor(wr, wi, 3, row_chunk=5)
    np.testing.assert_array_equal(p1, p2)
    np.testing.assert_allclose(s1, s2, rtol=1e-7)


def test_nonfinite_weight_is_taken_as_zero():
    wr = np.array([[np.nan, 1.0, -2.0, 0.5]], np.float32)
    wi = np.array([[0.0, np.inf, 0.1, 3.0]], np.float32)
    packed, scales, sums = O.quantize_tensor(wr, wi, 1)
    k = O.unpack_codes(packed[0])[0]
    assert list(k) == [0, 0, 2, 1]
    S_re, C_re, S_im, C_im = sums[0]
    assert (S_re, C_re, S_im, C_im) == (2.0, 3, 3.0, 1)


def test_empty_class_gives_zero_scale():
    wr = np.ones((2, 4), np.float32)
    wi = np.zeros((2, 4), np.float32)
    _, scales, _ = O.quantize_tensor(wr, wi, 2)
    assert scales[0, 0] == 1.0 and scales[0, 1] == 0.0
    # stage 2 residual is exactly zero everywhere -> all code 0, mean 0
    assert scales[1, 0] == 0.0 and scales[1, 1] == 0.0


def test_near_boundary_mask():
    a = np.array([1.0, 1.0, 1.0, 1e-9, 0.5])
    b = np.array([1.0, 1.0 + 1e-7, 0.9, 0.0, 0.1])
    m = O.near_boundary_mask(a, b, prev_scale_sum=1.0)
    assert list(m) == [True, True, False, True, False]


# ---------------------------------------------------------------------------
# Packing
# ---------------------------------------------------------------------------
def test_pack_hand_byte_and_round_trip():
    assert O.pack_codes(np.array([0, 1, 2, 3], np.uint8))[0] == 0xE4   # 0b11_10_01_00
    rng = np.random.default_rng(2)
    k = rng.integers(0, 4, size=(5, 64), dtype=np.uint8)
    np.testing.assert_array_equal(O.unpack_codes(O.pack_codes(k)), k)


def test_storage_is_two_bits_per_weight():
    """2 bits per complex weight: N K / 4 bytes per stage and branch; 1.3e9 weights ~ 325 MB
    ("iFairy talk notes" Q&A quotes about 300 MB; "iFairy article" §一 quotes 1/8 of FP16)."""
    k = np.zeros((48, 128), np.uint8)
    assert O.pack_codes(k).nbytes == 48 * 128 // 4
    assert 1.3e9 * 2 / 8 / 1e6 == pytest.approx(325.0)
    assert 2 / 16 == 1 / 8


# ---------------------------------------------------------------------------
# Widely-linear transform
# ---------------------------------------------------------------------------
def test_widely_linear_hand_example():
    g = {r[0]: r[1:] for r in read_golden("widely_linear_2x2.txt")}
    R = np.array([float(v) for v in g["R"]]).reshape(2, 2)
    U, W = O.widely_linear_from_real(R)
    assert U[0, 0] == complex(*[float(v) for v in g["U"]])
    assert W[0, 0] == complex(*[float(v) for v in g["W"]])


def test_widely_linear_identity_fp64():
    """R [x_re; x_im] = U x + W conj(x), to 1e-12 relative, on random shapes."""
    rng = np.random.default_rng(12)
    for (n, m) in ((3, 5), (16, 8), (40, 64)):
        R = rng.standard_normal((2 * n, 2 * m))
        U, W = O.widely_linear_from_real(R)
        xr, xi = rng.standard_normal(m), rng.standard_normal(m)
        y_real = R @ np.concatenate([xr, xi])
        x = xr + 1j * xi
        y = U @ x + W @ np.conj(x)
        scale = np.abs(R) @ np.concatenate([np.abs(xr), np.abs(xi)])
        assert np.max(np.abs(y.real - y_real[:n]) / scale[:n]) <= 1e-12
        assert np.max(np.abs(y.imag - y_real[n:]) / scale[n:]) <= 1e-12


def test_widely_linear_fp32_planes_are_exactly_rounded():
    """Each fp32 plane entry is the exact rational (R_ab +- R_cd)/2 rounded to nearest-even."""
    rng = np.random.default_rng(13)
    R = (0.02 * rng.standard_normal((6, 8))).astype(np.float32)
    ur, ui, wr, wi = O.widely_linear_planes_fp32(R)
    n, m = 3, 4
    for i in range(n):
        for j in range(m):
            r11, r12 = Fraction(float(R[i, j])), Fraction(float(R[i, j + m]))
            r21, r22 = Fraction(float(R[i + n, j])), Fraction(float(R[i + n, j + m]))
            for got, exact in ((ur, (r11 + r22) / 2), (ui, (r21 - r12) / 2),
                               (wr, (r11 - r22) / 2), (wi, (r12 + r21) / 2)):
                # nearest fp32 to the exact rational: compare with both neighbours
                g = Fraction(float(got[i, j]))
                up = Fraction(float(np.nextafter(got[i, j], np.float32(np.inf))))
                dn = Fraction(float(np.nextafter(got[i, j], np.float32(-np.inf))))
                assert abs(g - exact) <= abs(up - exact) and abs(g - exact) <= abs(dn - exact)


def test_widely_linear_rounded_planes_meet_page_bound():
    """With fp32-rounded U, W the identity still holds far inside the 1e-6 conversion bound
    ("Fairy2i write-up" §5.2)."""
    rng = np.random.default_rng(14)
    R = (0.02 * rng.standard_normal((64, 96))).astype(np.float32)
    ur, ui, wr, wi = (p.astype(np.float64) for p in O.widely_linear_planes_fp32(R))
    xr, xi = rng.standard_normal(48), rng.standard_normal(48)
    x = xr + 1j * xi
    y = (ur + 1j * ui) @ x + (wr + 1j * wi) @ np.conj(x)
    y_real = R.astype(np.float64) @ np.concatenate([xr, xi])
    rel = np.max(np.abs(np.concatenate([y.real, y.imag]) - y_real)) / np.max(np.abs(y_real))
    assert rel < 1e-6


# ---------------------------------------------------------------------------
# Product
# ---------------------------------------------------------------------------
def test_product_hand_example():
    g = {r[0]: r[1:] for r in read_golden("product_example.txt")}
    cu = O.pack_codes(np.array([[int(v) for v in g["u_codes"]]], np.uint8))[None]
    cw = O.pack_codes(np.array([[int(v) for v in g["w_codes"]]], np.uint8))[None]
    su = np.array([[float(v) for v in g["u_scales"]]], np.float32)
    sw = np.array([[float(v) for v in g["w_scales"]]], np.float32)
    xr = np.array([[float(v) for v in g["x_re"]]])
    xi = np.array([[float(v) for v in g["x_im"]]])
    yu = O.product(cu, su, None, None, xr, xi)
    y = O.product(cu, su, cw, sw, xr, xi)
    assert yu[0, 0] == complex(*[float(v) for v in g["y_u"]])
    assert y[0, 0] == complex(*[float(v) for v in g["y"]])


def test_product_brute_force_all_code_rows():
    """K = 4: all 256 code rows, against direct multiplication by codebook values as Python complex."""
    rng = np.random.default_rng(15)
    rows = np.array([[(r >> (2 * q)) & 3 for q in range(4)] for r in range(256)], np.uint8)
    T = 2
    codes = [rows, rows[::-1].copy()]
    scales = np.array([[0.7, 1.3], [0.11, 0.05]], np.float32)
    wcodes = [rows[rng.permutation(256)], rows[rng.permutation(256)]]
    wscales = np.array([[0.3, 0.9], [0.02, 0.08]], np.float32)
    xr = O.bf16_round(rng.standard_normal((3, 4)).astype(np.float32))
    xi = O.bf16_round(rng.standard_normal((3, 4)).astype(np.float32))
    y = O.product(np.stack([O.pack_codes(c) for c in codes]), scales,
                  np.stack([O.pack_codes(c) for c in wcodes]), wscales, xr, xi)
    for bb in range(3):
        x = [complex(float(xr[bb, j]), float(xi[bb, j])) for j in range(4)]
        for n in range(256):
            acc = 0j
            for t in range(T):
                for j in range(4):
                    cu = O.CODEBOOK[codes[t][n, j]]
                    cw = O.CODEBOOK[wcodes[t][n, j]]
                    wu = complex(float(scales[t, 0]) * cu.real, float(scales[t, 1]) * cu.imag)
                    ww = complex(float(wscales[t, 0]) * cw.real, float(wscales[t, 1]) * cw.imag)
                    acc += wu * x[j] + ww * x[j].conjugate()
            assert abs(y[bb, n] - acc) <= 1e-12 * (1 + abs(acc))


def test_product_one_hot_and_all_ones():
    rng = np.random.default_rng(16)
    k = rng.integers(0, 4, size=(8, 12), dtype=np.uint8)
    packed = O.pack_codes(k)[None]
    sc = np.array([[0.5, 0.25]], np.float32)
    W_hat = O.dequantize(packed, sc)
    for j in range(12):
        xr = np.zeros((1, 12))
        xr[0, j] = 1.0
        y = O.product(packed, sc, None, None, xr, np.zeros((1, 12)))
        np.testing.assert_array_equal(y[0], W_hat[:, j])
    ones = O.pack_codes(np.zeros((3, 12), np.uint8))[None]
    xr = O.bf16_round(rng.standard_normal((1, 12)).astype(np.float32))
    xi = O.bf16_round(rng.standard_normal((1, 12)).astype(np.float32))
    y = O.product(ones, sc, None, None, xr, xi)
    want = 0.5 * (np.sum(xr.astype(np.float64)) + 1j * np.sum(xi.astype(np.float64)))
    assert np.allclose(y[0], want, rtol=1e-14, atol=0)


def test_product_rows_subset_matches_full():
    rng = np.random.default_rng(17)
    k = rng.integers(0, 4, size=(2, 20, 16), dtype=np.uint8)
    packed = np.stack([O.pack_codes(k[0]), O.pack_codes(k[1])])
    sc = np.array([[0.5, 0.25], [0.1, 0.2]], np.float32)
    xr = rng.standard_normal((2, 16))
    xi = rng.standard_normal((2, 16))
    full = O.product(packed, sc, packed, sc[::-1], xr, xi)
    rows = np.array([3, 0, 19])
    sub = O.product_rows(packed, sc, packed, sc[::-1], xr, xi, rows)
    np.testing.assert_allclose(sub, full[:, rows], rtol=1e-14)


def test_tolerance_bound_formula():
    su = np.array([[1.0, 2.0]], np.float32)
    sw = np.array([[0.5, 0.5]], np.float32)
    xr = np.array([[1.0, -2.0]])
    xi = np.array([[0.0, 3.0]])
    assert O.tolerance_bound(su, sw, xr, xi)[0] == pytest.approx(1e-5 * 4.0 * 6.0)
    assert O.tolerance_bound(su, None, xr, xi)[0] == pytest.approx(1e-5 * 3.0 * 6.0)


# ---------------------------------------------------------------------------
# The plain-C restatement of a stage (used for full-size runs) against the above
# ---------------------------------------------------------------------------
def test_c_stage_matches_hand_example():
    from oracle import cref
    g = {r[0]: r[1:] for r in read_golden("two_stage_example.txt")}
    w_re = np.array([float(v) for v in g["w_re"]], np.float32)[None, :]
    w_im = np.array([float(v) for v in g["w_im"]], np.float32)[None, :]
    codes, scales = cref.quantize_tensor(w_re, w_im, 2)
    assert list(codes[0, 0]) == [int(v, 16) for v in g["bytes1"]]
    assert list(codes[1, 0]) == [int(v, 16) for v in g["bytes2"]]
    assert scales[1, 0] == np.float32(Fraction(17, 12)) and scales[1, 1] == np.float32(1.7)


def test_c_stage_matches_numpy_oracle():
    from oracle import cref
    rng = np.random.default_rng(21)
    for (N, K, T) in ((7, 12, 1), (33, 64, 3), (64, 256, 4)):
        wr = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
        wi = (0.03 * rng.standard_normal((N, K))).astype(np.float32)
        wr[0, :3] = [np.nan, np.inf, 0.0]
        wi[1, :2] = [1e-3, 1e-3]
        wr[1, :2] = [1e-3, -1e-3]
        c1, s1 = cref.quantize_tensor(wr, wi, T)
        c2, s2, _ = O.quantize_tensor(wr, wi, T)
        np.testing.assert_array_equal(c1, c2)
        np.testing.assert_allclose(s1, s2, rtol=1e-7, atol=0)


def test_c_near_boundary_flags_match_numpy():
    from oracle import cref
    rng = np.random.default_rng(22)
    wr = (0.02 * rng.standard_normal((16, 64))).astype(np.float32)
    wi = wr.copy()
    wi[:, ::2] = (0.02 * rng.standard_normal((16, 32))).astype(np.float32)
    codes, scales = cref.quantize_tensor(wr, wi, 2)
    _, _, near = cref.stage(wr, wi, 1, codes[:1].reshape(1, -1), scales[:1], want_near=True)
    a, b = O.residual_after(wr, wi, [O.unpack_codes(codes[0])], [tuple(scales[0])])
    want = O.near_boundary_mask(a, b, float(np.sum(scales[0].astype(np.float64))))
    np.testing.assert_array_equal(near.reshape(16, 64).astype(bool), want)


# ---------------------------------------------------------------- rotation and score
def test_rotation_by_i_is_swap_and_negate():
    """x i = (-Im x) + i Re x exactly ("iFairy talk notes" §2.3.1), element by element."""
    rng = np.random.default_rng(21)
    y = rng.standard_normal((3, 17)) + 1j * rng.standard_normal((3, 17))
    got = O.rotate_outputs(y, np.zeros((3, 17)), np.ones((3, 17)))
    np.testing.assert_array_equal(got.real, -y.imag)
    np.testing.assert_array_equal(got.imag, y.real)
    np.testing.assert_array_equal(O.rotate_outputs(y, np.ones((3, 17)), np.zeros((3, 17))), y)


def test_rotation_keeps_modulus_and_inverts():
    rng = np.random.default_rng(22)
    y = rng.standard_normal((4, 33)) + 1j * rng.standard_normal((4, 33))
    th = rng.uniform(-np.pi, np.pi, (4, 33))
    z = O.rotate_outputs(y, np.cos(th), np.sin(th))
    np.testing.assert_allclose(np.abs(z), np.abs(y), rtol=1e-14)
    back = O.rotate_outputs(z, np.cos(-th), np.sin(-th))
    np.testing.assert_allclose(back, y, rtol=1e-13, atol=1e-13)
    # the phase advances by theta: arg(z) - arg(y) = theta (mod 2 pi)
    d = np.angle(z) - np.angle(y) - th
    np.testing.assert_allclose(np.angle(np.exp(1j * d)), 0.0, atol=1e-12)


def test_score_is_polar_form_and_real_special_case():
    """Re(q^T conj(k)) = sum |q||k| cos(arg q - arg k); for real vectors the ordinary dot product;
    symmetric in q and k."""
    rng = np.random.default_rng(23)
    q = rng.standard_normal(64) + 1j * rng.standard_normal(64)
    k = rng.standard_normal(64) + 1j * rng.standard_normal(64)
    polar = float(np.sum(np.abs(q) * np.abs(k) * np.cos(np.angle(q) - np.angle(k))))
    assert abs(O.score(q, k) - polar) <= 1e-12 * float(np.sum(np.abs(q) * np.abs(k)))
    assert O.score(q, k) == pytest.approx(O.score(k, q), rel=1e-15, abs=1e-15)
    a, b = rng.standard_normal(50), rng.standard_normal(50)
    assert O.score(a + 0j, b + 0j) == pytest.approx(float(sum(float(u) * float(v) for u, v in zip(a, b))),
                                                   rel=1e-12)


def test_score_of_rotated_pair_depends_on_position_difference_only():
    """Rotating q by theta_q and k by theta_k per dimension, with theta = position * omega, leaves a
    score that depends on the positions only through their difference (the point of the rotary code)."""
    rng = np.random.default_rng(24)
    d = 32
    omega = 10000.0 ** (-np.arange(d) / d)
    q = rng.standard_normal(d) + 1j * rng.standard_normal(d)
    k = rng.standard_normal(d) + 1j * rng.standard_normal(d)

    def rot(v, pos):
        return O.rotate_outputs(v, np.cos(pos * omega), np.sin(pos * omega))
    s1 = O.score(rot(q, 7), rot(k, 3))
    s2 = O.score(rot(q, 104), rot(k, 100))
    assert s1 == pytest.approx(s2, rel=1e-10, abs=1e-10)
    assert O.score(rot(q, 5), rot(k, 5)) == pytest.approx(O.score(q, k), rel=1e-12, abs=1e-12)


# ---------------------------------------------------------------- dequantized training weights
def test_dequantize_bf16_single_stage_is_the_rounded_codeword():
    """T = 1: each entry is s_re * (+-1) or i s_im * (+-1) rounded to bf16, with the other part zero
    (one of real and imaginary part is always zero: "iFairy article" §二.1)."""
    rng = np.random.default_rng(41)
    k = rng.integers(0, 4, (1, 5, 64))
    packed = O.pack_codes(k)
    sc = np.array([[0.0123456, 0.0345678]], np.float32)
    re, im = O.dequantize_bf16(packed, sc)
    exact = O.dequantize(packed, sc)
    np.testing.assert_array_equal(re, O.bf16_round(exact.real.astype(np.float32)))
    np.testing.assert_array_equal(im, O.bf16_round(exact.imag.astype(np.float32)))
    assert np.all((re == 0) | (im == 0))
    vals = {float(v) for v in np.abs(re[re != 0])} | {float(v) for v in np.abs(im[im != 0])}
    assert vals == {float(O.bf16_round(np.float32(0.0123456))), float(O.bf16_round(np.float32(0.0345678)))}


def test_dequantize_bf16_is_within_rounding_of_the_exact_sum():
    rng = np.random.default_rng(42)
    for T in (2, 3, 8):
        k = rng.integers(0, 4, (T, 7, 32))
        packed = O.pack_codes(k)
        sc = (rng.uniform(0.001, 0.05, (T, 2))).astype(np.float32)
        re, im = O.dequantize_bf16(packed, sc)
        exact = O.dequantize(packed, sc)
        tot = float(np.sum(sc, dtype=np.float64))
        for got, want in ((re, exact.real), (im, exact.imag)):
            assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 2.0 ** -20 * tot)


# ---------------------------------------------------------------- bf16 rounding and decoding
def _rne(q, p, emin):
    """Exact rational q rounded to the nearest binary floating-point value with p significant bits,
    ties to the even significand, with subnormals below 2^emin on the fixed quantum 2^(emin - p + 1).
    Written from the definition of round-to-nearest-even; no overflow handling (returns a Fraction)."""
    q = Fraction(q)
    if q == 0:
        return Fraction(0)
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    quantum = Fraction(2) ** (max(e, emin) - p + 1)
    n = a / quantum
    f = n.numerator // n.denominator
    rest = n - f
    if rest > Fraction(1, 2) or (rest == Fraction(1, 2) and f % 2 == 1):
        f += 1
    return (1 if q > 0 else -1) * f * quantum


def _bf16_by_definition(x32):
    """bf16 RNE of one finite float32 value, through exact arithmetic; +-inf past the largest finite."""
    r = _rne(Fraction(float(x32)), 8, -126)
    if abs(r) >= Fraction(2) ** 128:
        return float("inf") if r > 0 else float("-inf")
    return float(r)


# (float32 bits, expected bf16 bits): worked by hand from round-to-nearest-even on the upper 16 bits
BF16_HAND = [
    (0x3F800000, 0x3F80),  # 1.0 is exact
    (0x3F808000, 0x3F80),  # exact tie, kept LSB 0 (even): down
    (0x3F818000, 0x3F82),  # exact tie, kept LSB 1 (odd): up
    (0x3F808001, 0x3F81),  # just above the tie: up
    (0x3F807FFF, 0x3F80),  # just below the tie: down
    (0xBF818000, 0xBF82),  # negative tie, odd: magnitude up, sign kept
    (0xBF808000, 0xBF80),  # negative tie, even: down
    (0x3FFF8000, 0x4000),  # tie with odd LSB carries into the exponent: 2.0
    (0x7F7F7FFF, 0x7F7F),  # largest finite bf16 from below
    (0x7F7F8000, 0x7F80),  # tie at the largest finite, odd: rounds to +inf
    (0x00008000, 0x0000),  # subnormal tie, even: +0
    (0x00018000, 0x0002),  # subnormal tie, odd: up
    (0x0000FFFF, 0x0001),  # rounds up to the smallest bf16 subnormal
    (0x00010001, 0x0001),  # just above the smallest subnormal: down
    (0x80000000, 0x8000),  # -0 stays -0
    (0x80008000, 0x8000),  # negative subnormal tie, even: -0
]


def test_bf16_round_hand_worked_bit_patterns():
    bits = np.array([b for b, _ in BF16_HAND], np.uint32)
    want = np.array([w for _, w in BF16_HAND], np.uint32) << 16
    got = O.bf16_round(bits.view(np.float32)).view(np.uint32)
    np.testing.assert_array_equal(got, want)


def test_bf16_round_equals_exact_round_to_nearest_even():
    """Random finite float32 values across the whole exponent range, plus values placed exactly on,
    one ulp below and one ulp above bf16 rounding ties, against the exact-arithmetic rounding."""
    rng = np.random.default_rng(51)
    u = rng.integers(0, 2 ** 32, 4000, dtype=np.uint64).astype(np.uint32)
    u = u[((u >> 23) & 0xFF) != 0xFF]                             # finite only
    ties = (rng.integers(0, 2 ** 16, 1000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    ties = ties[((ties >> 23) & 0xFF) != 0xFF]
    x = np.concatenate([u, ties, ties - 1, ties + 1]).view(np.float32)
    got = O.bf16_round(x)
    want = np.array([_bf16_by_definition(v) for v in x], np.float64)
    np.testing.assert_array_equal(got.astype(np.float64), want)
    # sign of zero results follows the input's sign
    zero = got == 0
    np.testing.assert_array_equal(np.signbit(got[zero]), np.signbit(x[zero]))


def test_bf16_round_agrees_with_torch_on_a_wide_sweep():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(52)
    u = rng.integers(0, 2 ** 32, 300000, dtype=np.uint64).astype(np.uint32)
    x = u[((u >> 23) & 0xFF) != 0xFF].view(np.float32)
    t = torch.from_numpy(x.copy()).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(O.bf16_round(x).view(np.uint32), t.view(np.uint32))


def test_bf16_bits_to_f64_decodes_every_pattern():
    """All 65536 bf16 patterns against sign * (1 + m/128) * 2^(e - 127) (normal), sign * m/128 * 2^-126
    (subnormal), +-inf and NaN."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        got = O.bf16_bits_to_f64(bits)
    for b in range(65536):
        s, e, m = b >> 15, (b >> 7) & 0xFF, b & 0x7F
        sign = -1.0 if s else 1.0
        if e == 0xFF:
            if m == 0:
                assert got[b] == sign * float("inf")
            else:
                assert np.isnan(got[b])
            continue
        mag = Fraction(m, 128) * Fraction(2) ** -126 if e == 0 else (1 + Fraction(m, 128)) * Fraction(2) ** (e - 127)
        assert got[b] == sign * float(mag), hex(b)
        if mag == 0:
            assert bool(np.signbit(got[b])) == bool(s)


def _dequant_entry_by_definition(codes_tn, scales, part):
    """One entry of the training weights: stage terms added in float32 (each partial sum rounded to
    nearest-even float32) in stage order from 0, then rounded once to bf16.  part 0: real, 1: imag."""
    acc = Fraction(0)
    for t, k in enumerate(codes_tn):
        if (k & 1) != part:
            continue                              # this stage's code lies on the other axis
        term = Fraction(float(scales[t][part])) * (-1 if k >> 1 else 1)
        acc = _rne(acc + term, 24, -126)
    return float(_rne(acc, 8, -126))


@pytest.mark.parametrize("T", [2, 3])
def test_dequantize_bf16_multi_stage_equals_exact_stage_order_sum(T):
    rng = np.random.default_rng(60 + T)
    k = rng.integers(0, 4, (T, 6, 40))
    packed = O.pack_codes(k)
    sc = rng.uniform(0.001, 0.05, (T, 2)).astype(np.float32)
    re, im = O.dequantize_bf16(packed, sc)
    for n in range(k.shape[1]):
        for j in range(k.shape[2]):
            col = [int(k[t, n, j]) for t in range(T)]
            assert re[n, j] == _dequant_entry_by_definition(col, sc, 0), (n, j)
            assert im[n, j] == _dequant_entry_by_definition(col, sc, 1), (n, j)


def test_dequantize_bf16_rounds_each_stage_sum_in_float32():
    """Hand-worked: real-axis codes with scales 1 + 2^-8, 2^-25, 2^-25.  In float32 each 2^-25 added
    to 1 + 2^-8 is a tie that rounds back to the even 1 + 2^-8, whose bf16 rounding is again a tie,
    to 1.0.  The exact sum 1 + 2^-8 + 2^-24 would round to 1 + 2^-7 instead."""
    sc = np.array([[1 + 2.0 ** -8, 0.5], [2.0 ** -25, 0.5], [2.0 ** -25, 0.5]], np.float32)
    packed = O.pack_codes(np.zeros((3, 1, 4), np.uint8))       # code 0 (+1) at every stage
    re, im = O.dequantize_bf16(packed, sc)
    np.testing.assert_array_equal(re, np.ones((1, 4), np.float32))
    np.testing.assert_array_equal(im, np.zeros((1, 4), np.float32))
    assert float(_rne(Fraction(1) + Fraction(1, 256) + Fraction(1, 2 ** 24), 8, -126)) == 1 + 2.0 ** -7
