"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test ties one oracle function to a closed form, a published table or
value, a library routine on the special case it reduces to, or brute force,
chosen so that a plausible mistake (a dropped term, a wrong sign, an
off-by-one index, a transposed operand) fails at least one of them.
"""
import math
from pathlib import Path

import numpy as np
import pytest
from scipy import integrate
from scipy.stats import norm

from oracle import turboquant_oracle as o


GOLDEN = Path(__file__).parent / "golden"


def _records(name):
    """Non-comment lines of a golden fixture, split on whitespace."""
    return [ln.split() for ln in (GOLDEN / name).read_text().splitlines() if ln.strip() and not ln.startswith("#")]


# ---------------------------------------------------------------- codebook
# Max's 1960 table of the optimal Gaussian quantizer (golden fixture, with its
# citation): mean squared error of the 2/4/8/16-level quantizer of N(0,1) and
# the positive halves of its levels and thresholds.  The table's 16-level
# error is 0.04% below the exact optimum (0.0095010, found here by closed form
# and by quadrature), so the distortion tolerance is the printed precision of
# the table (5e-4 relative).
_MAX = _records("max1960_gaussian_quantizer.txt")
DISTORTION = {int(r[0]): float(r[2]) for r in _MAX if r[1] == "distortion"}
MAX_CENTROIDS = {int(r[0]): [float(v) for v in r[2:]] for r in _MAX if r[1] == "centroids"}
MAX_THRESHOLDS = {int(r[0]): [float(v) for v in r[2:]] for r in _MAX if r[1] == "thresholds"}


def test_golden_max_table_is_complete():
    assert sorted(DISTORTION) == [1, 2, 3, 4]
    for bits in (2, 3, 4):
        assert len(MAX_CENTROIDS[bits]) == len(MAX_THRESHOLDS[bits]) == 2 ** (bits - 1)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_lloyd_max_distortion_matches_published(bits):
    c = o.lloyd_max_normal(bits)
    d = o.lloyd_max_distortion(c)
    assert abs(d - DISTORTION[bits]) / DISTORTION[bits] < 5e-4


def test_one_bit_closed_form():
    c = o.lloyd_max_normal(1)
    assert np.allclose(c, [-math.sqrt(2 / math.pi), math.sqrt(2 / math.pi)], atol=1e-13)
    assert abs(o.lloyd_max_distortion(c) - (1 - 2 / math.pi)) < 1e-13


def _table_tol(v):
    """1.5 units of the last of four printed significant digits (half a unit
    of rounding plus one unit of error in the 1960 hand computation)."""
    v = abs(v)
    return 1e-12 if v == 0 else 1.5 * 10.0 ** (math.floor(math.log10(v)) - 3)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_lloyd_max_matches_max_1960_table(bits):
    c = o.lloyd_max_normal(bits)
    t = o.thresholds_of(c)
    for got, want in zip(c[len(c) // 2:], MAX_CENTROIDS[bits]):
        assert abs(got - want) <= _table_tol(want)
    for got, want in zip(t[len(t) // 2:], MAX_THRESHOLDS[bits]):
        assert abs(got - want) <= _table_tol(want)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_centroid_and_nearest_neighbour_conditions_by_quadrature(bits):
    """Each centroid is its cell's conditional mean (checked by numerical
    integration, not by the closed form the iteration uses), the codebook is
    antisymmetric, and the closed-form distortion equals the integral."""
    c = o.lloyd_max_normal(bits)
    assert np.array_equal(c, -c[::-1])
    t = o.thresholds_of(c)
    edges = np.concatenate(([-np.inf], t, [np.inf]))
    total = 0.0
    for j, cj in enumerate(c):
        mass = integrate.quad(norm.pdf, edges[j], edges[j + 1], epsabs=1e-15)[0]
        mean = integrate.quad(lambda x: x * norm.pdf(x), edges[j], edges[j + 1], epsabs=1e-15)[0] / mass
        assert abs(mean - cj) < 1e-10
        total += integrate.quad(lambda x: (x - cj) ** 2 * norm.pdf(x), edges[j], edges[j + 1],
                                epsabs=1e-15, epsrel=1e-13)[0]
    assert abs(total - o.lloyd_max_distortion(c)) < 1e-12


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_distortion_monte_carlo(bits):
    rng = np.random.default_rng(7 + bits)
    x = rng.standard_normal(1_000_000)
    c = o.lloyd_max_normal(bits)
    t = o.thresholds_of(c)
    err = (x - c[np.sum(x[:, None] > t[None, :], axis=1)]) ** 2
    d = o.lloyd_max_distortion(c)
    assert abs(err.mean() - d) < 5 * err.std() / math.sqrt(x.size)


def test_codebook_fp16_scaling():
    d = 128
    for bits in (2, 3, 4):
        c, t = o.codebook(bits, d)
        assert np.array_equal(c, c.astype(np.float16).astype(np.float64))     # fp16 centroids
        assert np.array_equal(t, t.astype(np.float32).astype(np.float64))     # midpoints fit fp32
        assert np.array_equal(2 * t, c[:-1] + c[1:])
        assert np.allclose(c * math.sqrt(d), o.lloyd_max_normal(bits), rtol=2 ** -11)
        assert np.all(np.diff(c) > 0) and np.all((t > c[:-1]) & (t < c[1:]))
        assert t[len(t) // 2] == 0.0 and np.array_equal(c, -c[::-1])
        # rounding the centroids to fp16 moves the N(0,1) distortion by < 1e-5 relative
        dist = o.lloyd_max_distortion(c * math.sqrt(d))
        assert abs(dist / o.lloyd_max_distortion(o.lloyd_max_normal(bits)) - 1) < 1e-5


# ------------------------------------------- codebook for the exact law (sphere)
# One coordinate of a uniform unit vector in R^d has the density
# (1 - x^2)^((d-3)/2) / B(1/2, (d-1)/2) on (-1, 1).  The pins below use plain
# quadrature of that density, closed forms of special cases, the large-d
# limit and sampled unit vectors: none of them uses the incomplete beta
# function the oracle's iteration uses.
def _sphere_pdf(d):
    from scipy.special import gammaln
    logc = gammaln(0.5 * d) - gammaln(0.5) - gammaln(0.5 * (d - 1))   # 1 / B(1/2, (d-1)/2)
    return lambda x: math.exp(logc + 0.5 * (d - 3) * math.log1p(-x * x)) if abs(x) < 1 else 0.0


def test_sphere_density_normalised_and_d3_is_uniform():
    for d in (3, 16, 128):
        f = _sphere_pdf(d)
        assert abs(integrate.quad(f, -1, 1, epsabs=1e-14, points=[0.0])[0] - 1) < 1e-10
    # d = 3: the coordinate is uniform on [-1, 1] (Archimedes), so the optimal
    # L-level quantizer has equal cells: c_j = -1 + (2 j + 1) / L and MSE 1 / (3 L^2)
    for bits in (1, 2, 3, 4):
        levels = 1 << bits
        c = o.lloyd_max_sphere(bits, 3)
        assert np.allclose(c, -1 + (2 * np.arange(levels) + 1) / levels, atol=1e-12)
        assert abs(o.sphere_distortion(c, 3) - 1 / (3 * levels ** 2)) < 1e-12


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_sphere_centroid_and_nearest_neighbour_conditions_by_quadrature(bits):
    d = 128
    f = _sphere_pdf(d)
    c = o.lloyd_max_sphere(bits, d)
    assert np.array_equal(c, -c[::-1]) and np.all(np.diff(c) > 0)
    t = o.thresholds_of(c)
    edges = np.concatenate(([-1.0], t, [1.0]))
    total = 0.0
    for j, cj in enumerate(c):
        lo, hi = edges[j], edges[j + 1]
        mass = integrate.quad(f, lo, hi, epsabs=1e-15, epsrel=1e-13, limit=200)[0]
        mean = integrate.quad(lambda x: x * f(x), lo, hi, epsabs=1e-15, epsrel=1e-13, limit=200)[0] / mass
        assert abs(mean - cj) < 1e-11
        total += integrate.quad(lambda x: (x - cj) ** 2 * f(x), lo, hi, epsabs=1e-16, epsrel=1e-12, limit=200)[0]
    assert abs(total - o.sphere_distortion(c, d)) < 1e-13


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_sphere_codebook_tends_to_the_gaussian_one(bits):
    """N(0, 1/d) is the large-d limit of the coordinate law: sqrt(d) times the
    exact-law centroids approach the N(0,1) ones at rate 1/d."""
    g = o.lloyd_max_normal(bits)
    gaps = [np.max(np.abs(o.lloyd_max_sphere(bits, d) * math.sqrt(d) - g)) for d in (128, 1024)]
    assert gaps[1] < 0.01
    assert 6 < gaps[0] / gaps[1] < 10   # about 1024 / 128 = 8


def test_sphere_codebook_on_sampled_unit_vectors():
    """On the coordinates of sampled unit vectors, the closed-form MSE of a
    codebook under the exact law matches the sampled MSE (checked for the
    exact-law codebook and for the N(0, 1/d) one), and the exact-law codebook
    has the lower closed-form MSE (it is the optimum for that law)."""
    d, bits = 128, 3
    rng = np.random.default_rng(2024)
    x = rng.standard_normal((20000, d))
    y = (x / np.linalg.norm(x, axis=1, keepdims=True)).ravel()
    cs = o.lloyd_max_sphere(bits, d)
    cg = o.lloyd_max_normal(bits) / math.sqrt(d)
    for c in (cs, cg):
        t = o.thresholds_of(c)
        e = (y - c[np.searchsorted(t, y, side="left")]) ** 2
        assert abs(e.mean() - o.sphere_distortion(c, d)) < 5 * e.std() / math.sqrt(y.size)
    assert o.sphere_distortion(cs, d) < o.sphere_distortion(cg, d)


def test_codebook_laws():
    for bits in (2, 3, 4):
        c, t = o.codebook(bits, 128, o.LAW_SPHERE)
        assert np.array_equal(c, c.astype(np.float16).astype(np.float64))
        assert np.array_equal(2 * t, c[:-1] + c[1:])
        assert np.allclose(c, o.lloyd_max_sphere(bits, 128), rtol=2 ** -11)
    with pytest.raises(ValueError):
        o.codebook(3, 128, "cauchy")


# ------------------------------------------------------------------- random
def test_splitmix64_published_values():
    # First outputs of the reference SplitMix64 (golden fixture, with its citation).
    rec = _records("splitmix64_outputs.txt")
    assert len(rec) == 4
    for seed, n, want in rec:
        assert o.splitmix64_output(int(seed), int(n)) == int(want)


def test_splitmix64_counter_form_equals_sequential_generator():
    seed = 987654321
    state = seed
    for n in range(1, 200):
        state = (state + o.SPLITMIX_GAMMA) & ((1 << 64) - 1)
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & ((1 << 64) - 1)
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & ((1 << 64) - 1)
        assert o.splitmix64_output(seed, n) == z ^ (z >> 31)


def test_gaussian_stream_moments_and_independence():
    g0 = o.gaussian_stream(42, o.STREAM_PI, 200_000)
    g1 = o.gaussian_stream(42, o.STREAM_S, 200_000)
    for g in (g0, g1):
        assert abs(g.mean()) < 5 / math.sqrt(g.size)
        assert abs(g.var() - 1) < 5 * math.sqrt(2 / g.size)
        assert abs(np.mean(g ** 4) - 3) < 0.05
    assert abs(np.corrcoef(g0, g1)[0, 1]) < 5 / math.sqrt(g0.size)
    assert abs(np.corrcoef(g0[:-1], g0[1:])[0, 1]) < 5 / math.sqrt(g0.size)
    assert np.array_equal(g0[:10], o.gaussian_stream(42, o.STREAM_PI, 10))


# ----------------------------------------------------------------- rounding
def test_bf16_rounding_matches_torch_on_fp32_values():
    import torch
    rng = np.random.default_rng(3)
    x = rng.standard_normal(100_000).astype(np.float32).astype(np.float64) * 0.1
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(o.round_to_bf16(x), ref)
    # exact ties go to the even neighbour
    assert o.round_to_bf16(1 + 2 ** -8) == 1.0
    assert o.round_to_bf16(1 + 3 * 2 ** -8) == 1 + 2 ** -6


def test_fp16_rounding_matches_numpy_and_saturates():
    rng = np.random.default_rng(4)
    x = np.exp(rng.uniform(-20, 11, 100_000)).astype(np.float32).astype(np.float64)
    x = x[x < 65504]
    ref = x.astype(np.float32).astype(np.float16).astype(np.float64)
    assert np.array_equal(o.round_to_fp16_sat(x), ref)
    assert o.round_to_fp16_sat(1 + 2 ** -11) == 1.0
    assert o.round_to_fp16_sat(1 + 3 * 2 ** -11) == 1 + 2 ** -9
    assert o.round_to_fp16_sat(70000.0) == 65504.0
    assert o.round_to_fp16_sat(1e9) == 65504.0
    assert o.round_to_fp16_sat(2 ** -25) == 0.0            # tie below the smallest subnormal
    assert o.round_to_fp16_sat(3 * 2 ** -25) == 2 ** -23


# ---------------------------------------------------------------- rotation
@pytest.mark.parametrize("d,seed", [(128, 42), (64, 7), (16, 1)])
def test_rotation_is_signed_qr_of_the_seeded_gaussian(d, seed):
    q = o.rotation_exact(d, seed)
    g = o.gaussian_stream(seed, o.STREAM_PI, d * d).reshape(d, d)
    assert np.abs(q.T @ q - np.eye(d)).max() < 1e-12
    r = q.T @ g                                   # must be R of G = Q R
    assert np.abs(np.tril(r, -1)).max() < 1e-10
    assert np.all(np.diag(r) > 0)
    x = np.random.default_rng(seed).standard_normal((10, d))
    assert np.allclose(np.linalg.norm(x @ q.T, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)


def test_rotation_bf16_is_near_orthogonal():
    pi = o.rotation_bf16(128, 42)
    assert np.array_equal(pi, o.round_to_bf16(pi))
    err = np.abs(pi.T @ pi - np.eye(128)).max()
    assert 0 < err < 3e-3


def test_rotation_haar_statistics():
    # Entries of a Haar orthogonal matrix have mean 0 and variance 1/d.
    d = 64
    vals = np.concatenate([o.rotation_exact(d, s).ravel() for s in range(1, 6)])
    assert abs(vals.mean()) < 5 / math.sqrt(vals.size) / math.sqrt(d)
    assert abs(vals.var() * d - 1) < 0.02


def test_qjl_matrix_is_fp32_gaussian():
    s = o.qjl_matrix(128, 42)
    assert np.array_equal(s, s.astype(np.float32).astype(np.float64))
    assert abs(s.mean()) < 0.03 and abs(s.var() - 1) < 0.03
    assert not np.allclose(s, o.gaussian_stream(42, o.STREAM_PI, 128 * 128).reshape(128, 128))


# ---------------------------------------------------------------- quantize
def _random_bf16_rows(n, d, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return o.round_to_bf16(rng.standard_normal((n, d)) * scale)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quantize_picks_nearest_centroid(bits):
    d = 128
    pi = o.rotation_bf16(d, 42)
    c, t = o.codebook(bits, d)
    x = _random_bf16_rows(2000, d, bits)
    qz = o.quantize(x, pi, c, t)
    # brute force: y from an independent formula, nearest centroid by argmin
    y = (pi @ x.T).T / np.linalg.norm(x, axis=1)[:, None]
    assert np.allclose(y, qz.y, atol=1e-13)
    nearest = np.argmin(np.abs(y[:, :, None] - c[None, None, :]), axis=2)
    # ties are impossible to hit except within fp32 rounding of a midpoint
    gap = np.min(np.abs(y[:, :, None] - t[None, None, :]), axis=2)
    ok = (nearest == qz.codes) | (gap < 1e-7)
    assert ok.all()
    assert np.array_equal(qz.norm, o.round_to_fp16_sat(np.linalg.norm(x, axis=1)))


def test_quantize_zero_vector_and_threshold_tie():
    d = 128
    pi = o.rotation_bf16(d, 42)
    for bits in (2, 3, 4):
        c, t = o.codebook(bits, d)
        qz = o.quantize(np.zeros((1, d)), pi, c, t, s_matrix=o.qjl_matrix(d, 42))
        assert np.all(qz.codes == (1 << (bits - 1)) - 1)
        assert qz.norm[0] == 0.0
    # a coordinate exactly on a threshold goes to the lower cell
    # (x = e_0 has norm exactly 1 and diag(t_5, 1, 1, 1) puts y_0 exactly on t_5)
    c, t = o.codebook(3, 4)
    qz = o.quantize(np.array([[1.0, 0.0, 0.0, 0.0]]), np.diag([t[5], 1.0, 1.0, 1.0]), c, t)
    assert qz.y[0, 0] == t[5] and qz.codes[0, 0] == 5
    qz = o.quantize(np.array([[1.0, 0.0, 0.0, 0.0]]), np.diag([np.nextafter(t[5], 1), 1.0, 1.0, 1.0]), c, t)
    assert qz.codes[0, 0] == 6


def test_quantize_codes_are_scale_invariant_until_the_stored_norm_vanishes():
    """y = (Pi x)/||x|| does not depend on the scale of x, so exact power-of-two
    scalings of x keep every code and QJL sign while the fp16 norm is nonzero
    (fp16 subnormals reach down to 2^-24); once ||x|| <= 2^-25 the stored norm
    is 0 and the vector is stored as the zero vector."""
    d = 128
    pi = o.rotation_bf16(d, 42)
    s = o.qjl_matrix(d, 42)
    rng = np.random.default_rng(5)
    x = rng.standard_normal((64, d))
    x /= np.linalg.norm(x, axis=1)[:, None]
    for bits in (2, 3, 4):
        c, t = o.codebook(bits, d)
        ref = o.quantize(x, pi, c, t, s_matrix=s)
        for e in (-24, -10, 0, 10):            # stored norm 2^e > 0
            q = o.quantize(x * 2.0 ** e, pi, c, t, s_matrix=s)
            assert np.array_equal(q.codes, ref.codes) and np.array_equal(q.qjl_signs, ref.qjl_signs)
            assert np.all(q.norm == 2.0 ** e)
        for e in (-26, -40):                   # stored norm rounds to 0
            q = o.quantize(x * 2.0 ** e, pi, c, t, s_matrix=s)
            zero = o.quantize(np.zeros((1, d)), pi, c, t, s_matrix=s)
            assert np.all(q.norm == 0.0)
            assert np.all(q.codes == (1 << (bits - 1)) - 1)
            assert np.array_equal(q.qjl_signs, np.repeat(zero.qjl_signs, len(x), axis=0))


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quantize_distortion_on_unit_vectors(bits):
    """E||u - Pi^T c[code]||^2 over random unit vectors ~= D_b (Gaussian law
    approximation of the rotated coordinates; a few percent at d = 128)."""
    d = 128
    pi = o.rotation_bf16(d, 11)
    c, t = o.codebook(bits, d)
    rng = np.random.default_rng(bits)
    u = rng.standard_normal((20000, d))
    u /= np.linalg.norm(u, axis=1)[:, None]
    qz = o.quantize(u, pi, c, t)
    recon = c[qz.codes] @ pi
    mse = np.mean(np.sum((u - recon) ** 2, axis=1))
    assert abs(mse / DISTORTION[bits] - 1) < 0.04


# ----------------------------------------------------------------- packing
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pack_roundtrip_and_size(bits):
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 1 << bits, size=(500, 128))
    packed = o.pack_codes(codes, bits)
    assert packed.shape == (500, 128 * bits // 8)
    assert np.array_equal(o.unpack_codes(packed, bits, 128), codes)
    pos = o.code_bit_position(bits, 128)
    assert np.array_equal(np.sort(pos.ravel()), np.arange(128 * bits))


def test_pack_bit_positions_worked_examples():
    # 2 bits, LSB first: code 3 at coordinate 5 sets bits 10,11 -> byte 1 = 0b00001100
    codes = np.zeros((1, 128), dtype=np.int64)
    codes[0, 5] = 3
    assert o.pack_codes(codes, 2)[0, 1] == 0b00001100
    # 4 bits: code 9 at coordinate 3 -> byte 1 high nibble = 9
    codes = np.zeros((1, 128), dtype=np.int64)
    codes[0, 3] = 9
    assert o.pack_codes(codes, 4)[0, 1] == 0x90
    # 3 bits: coordinate 10 (word 1, nibble 2) code 5 -> word 1 = 0x500 -> byte 5 = 0x05
    codes = np.zeros((1, 128), dtype=np.int64)
    codes[0, 10] = 5
    p = o.pack_codes(codes, 3)[0]
    assert p[5] == 0x05 and p.sum() == 5
    # 3 bits: coordinate 25 (spare column 1) code 0b101 -> bit 7 of words 0 and 2
    codes = np.zeros((1, 128), dtype=np.int64)
    codes[0, 25] = 0b101
    p = o.pack_codes(codes, 3)[0]
    assert p[0] == 0x80 and p[8] == 0x80 and p.sum() == 0x100
    # 3 bits, second group starts at byte 12
    codes = np.zeros((1, 128), dtype=np.int64)
    codes[0, 33] = 7
    p = o.pack_codes(codes, 3)[0]
    assert p[12] == 0x70 and p.sum() == 0x70
    # QJL signs: bit m at position m
    s = np.zeros((1, 128), dtype=np.int64)
    s[0, 9] = 1
    assert o.pack_signs(s)[0, 1] == 0x02


# --------------------------------------------------------------------- QJL
def test_qjl_estimator_is_unbiased_with_predicted_variance():
    """Over independent Gaussian S, the mean of the estimate equals <q, r>
    and its variance equals ((pi/2)|q|^2|r|^2 - <q,r>^2)/d."""
    d = 128
    rng = np.random.default_rng(5)
    q = rng.standard_normal(d)
    r = 0.3 * q / np.linalg.norm(q) + rng.standard_normal(d) * 0.02
    trials = 12000
    est = np.empty(trials)
    for b0 in range(0, trials, 1000):
        s = rng.standard_normal((1000, d, d))
        qt = s @ q
        sg = (s @ r >= 0).astype(np.int64)
        for k in range(1000):
            est[b0 + k] = o.qjl_inner_product(qt[k][None, :], sg[k][None, :],
                                              np.array([np.linalg.norm(r)]), d)[0, 0]
    exact = q @ r
    var_pred = ((math.pi / 2) * (q @ q) * (r @ r) - exact ** 2) / d
    assert abs(est.mean() - exact) < 4 * math.sqrt(var_pred / trials)
    assert abs(est.var() / var_pred - 1) < 0.05


def test_qjl_sign_of_zero_projection_is_plus():
    # reading: (S r)_m == 0 stores bit 1 (+1); an all-zero S makes every projection 0
    p = o.Params(128, 3, 3, False, 42)
    qz = o.quantize(_random_bf16_rows(5, 128, 1), p.pi, p.ck, p.tk, s_matrix=np.zeros((128, 128)))
    assert np.all(qz.qjl_signs == 1)


def test_qjl_quantize_fields():
    d = 128
    p = o.Params(d, 2, 2, True, 42)
    x = _random_bf16_rows(300, d, 9)
    qz = o.quantize(x, p.pi, p.ck, p.tk, s_matrix=p.s)
    r = qz.y - p.ck[qz.codes]
    assert np.allclose(qz.qjl_proj, r @ p.s.T)
    assert np.array_equal(qz.qjl_signs, (r @ p.s.T >= 0).astype(np.int64))
    assert np.array_equal(qz.qjl_gamma, o.round_to_fp16_sat(np.linalg.norm(r, axis=1)))


# ------------------------------------------------------------------ decode
def _decode_case(d, t_len, g, bits_k, bits_v, qjl, seed):
    p = o.Params(d, bits_k, bits_v, qjl, seed)
    rng = np.random.default_rng(seed)
    k = o.round_to_bf16(rng.standard_normal((t_len, d)) * rng.lognormal(0, 0.5, (t_len, 1)))
    v = o.round_to_bf16(rng.standard_normal((t_len, d)))
    q = rng.standard_normal((g, d))
    qk = o.quantize(k, p.pi, p.ck, p.tk, s_matrix=p.s)
    qv = o.quantize(v, p.pi, p.cv, p.tv)
    return p, q, k, v, qk, qv


@pytest.mark.parametrize("qjl", [False, True])
@pytest.mark.parametrize("bits", [(2, 2), (3, 3), (4, 2)])
def test_decode_equals_attention_over_explicit_dequantization(bits, qjl):
    """The rotated-space decode equals plain attention over the vectors
    reconstructed in the original space: k~ = n Pi^T (c[code] + QJL residual
    estimate), v~ = n Pi^T c[code] (identity <Pi q, c> = <q, Pi^T c>)."""
    d = 64
    p, q, k, v, qk, qv = _decode_case(d, 37, 3, bits[0], bits[1], qjl, 3)
    scale = 1 / math.sqrt(d)
    o_dec, lse_dec, _ = o.decode_attention(
        q, p.pi, p.ck, qk.codes, qk.norm, p.cv, qv.codes, qv.norm, scale,
        s_matrix=p.s, qjl_signs=qk.qjl_signs, qjl_gamma=qk.qjl_gamma)
    k_rec = o.dequantize(p.pi, p.ck, qk.codes, qk.norm)
    if qjl:
        pm = 2.0 * qk.qjl_signs - 1.0
        resid_rot = math.sqrt(math.pi / 2) / d * qk.qjl_gamma[:, None] * (pm @ p.s)
        k_rec = k_rec + qk.norm[:, None] * (resid_rot @ p.pi)
    v_rec = o.dequantize(p.pi, p.cv, qv.codes, qv.norm)
    o_ref, lse_ref = o.exact_attention(q, k_rec, v_rec, scale)
    assert np.allclose(o_dec, o_ref, rtol=1e-11, atol=1e-12)
    assert np.allclose(lse_dec, lse_ref, rtol=1e-12)


def test_decode_single_token_and_equal_scores():
    d = 32
    p, q, k, v, qk, qv = _decode_case(d, 1, 2, 3, 3, False, 4)
    o1, _, _ = o.decode_attention(q, p.pi, p.ck, qk.codes, qk.norm, p.cv, qv.codes, qv.norm, 0.1)
    assert np.allclose(o1, np.repeat(o.dequantize(p.pi, p.cv, qv.codes, qv.norm), 2, axis=0))
    # all keys zero -> uniform weights -> mean of the reconstructed values
    p, q, k, v, qk, qv = _decode_case(d, 9, 2, 3, 3, False, 5)
    zeros = o.quantize(np.zeros((9, d)), p.pi, p.ck, p.tk)
    o2, lse, _ = o.decode_attention(q, p.pi, p.ck, zeros.codes, zeros.norm, p.cv, qv.codes, qv.norm, 0.1)
    assert np.allclose(o2, o.dequantize(p.pi, p.cv, qv.codes, qv.norm).mean(axis=0)[None, :])
    assert np.allclose(lse, math.log(9))


def test_compressed_attention_converges_to_exact_with_bits():
    """More bits -> attention over the compressed cache approaches attention
    over the original vectors; error falls roughly as 2^-b."""
    d = 64
    rng = np.random.default_rng(8)
    k = o.round_to_bf16(rng.standard_normal((200, d)))
    v = o.round_to_bf16(rng.standard_normal((200, d)))
    q = rng.standard_normal((4, d)) * 2
    pi = o.rotation_bf16(d, 42)
    o_ex, _ = o.exact_attention(q, k, v, 1 / math.sqrt(d))
    errs = []
    for bits in (2, 3, 4, 5, 6):
        c, t = o.codebook(bits, d)
        qk = o.quantize(k, pi, c, t)
        qv = o.quantize(v, pi, c, t)
        ob, _, _ = o.decode_attention(q, pi, c, qk.codes, qk.norm, c, qv.codes, qv.norm, 1 / math.sqrt(d))
        errs.append(np.abs(ob - o_ex).max() / np.abs(o_ex).max())
    assert all(a > b for a, b in zip(errs, errs[1:]))
    assert errs[-1] < 0.05 and errs[0] / errs[-1] > 6


def test_exact_attention_definition():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((3, 8))
    k = rng.standard_normal((5, 8))
    v = rng.standard_normal((5, 8))
    o_ref, lse = o.exact_attention(q, k, v, 0.5)
    for g in range(3):
        s = [0.5 * sum(q[g, i] * k[j, i] for i in range(8)) for j in range(5)]
        w = [math.exp(x) for x in s]
        for i in range(8):
            assert abs(o_ref[g, i] - sum(w[j] * v[j, i] for j in range(5)) / sum(w)) < 1e-12
        assert abs(lse[g] - math.log(sum(w))) < 1e-12


def test_cosine_similarity():
    assert o.cosine_similarity([1, 0], [2, 0]) == pytest.approx(1.0)
    assert o.cosine_similarity([1, 0], [0, 3]) == pytest.approx(0.0)


# ----------------------------------------------------------------- prefill
@pytest.mark.parametrize("qjl", [False, True])
def test_prefill_is_causal_attention_over_explicit_dequantization(qjl):
    """Every query of a prefill chunk equals plain causal softmax attention
    over the vectors reconstructed in the original space (QJL residual
    included), with the mask written out as a full score matrix: query t at
    position p sees keys 0..p and nothing after."""
    d, t_len, g = 32, 29, 2
    p, _, k, v, qk, qv = _decode_case(d, t_len, g, 3, 2, qjl, 8)
    rng = np.random.default_rng(81)
    q_pos = np.array([3, 10, 11, 20, 28])                    # a chunk of positions inside the cache
    q = rng.standard_normal((len(q_pos), g, d))
    scale = 1 / math.sqrt(d)
    o_pre, lse_pre, _ = o.prefill_attention(q, q_pos, p.pi, p.ck, qk.codes, qk.norm, p.cv, qv.codes, qv.norm, scale,
                                         s_matrix=p.s, qjl_signs=qk.qjl_signs, qjl_gamma=qk.qjl_gamma)
    k_rec = o.dequantize(p.pi, p.ck, qk.codes, qk.norm)
    if qjl:
        pm = 2.0 * qk.qjl_signs - 1.0
        k_rec = k_rec + qk.norm[:, None] * ((math.sqrt(math.pi / 2) / d * qk.qjl_gamma[:, None] * (pm @ p.s)) @ p.pi)
    v_rec = o.dequantize(p.pi, p.cv, qv.codes, qv.norm)
    for t, pos in enumerate(q_pos):
        s_full = scale * q[t] @ k_rec.T                      # [g, t_len]
        s_full[:, np.arange(t_len) > pos] = -np.inf           # causal mask
        w = np.exp(s_full - s_full.max(axis=1, keepdims=True))
        o_ref = (w @ v_rec) / w.sum(axis=1, keepdims=True)
        lse_ref = s_full.max(axis=1) + np.log(w.sum(axis=1))
        assert np.allclose(o_pre[t], o_ref, rtol=1e-11, atol=1e-12)
        assert np.allclose(lse_pre[t], lse_ref, rtol=1e-12)


def test_prefill_ignores_tokens_after_each_query():
    """Causality: changing the cached tokens after a query's position leaves
    that query's output unchanged, and the first position attends to itself
    alone."""
    d = 32
    p, _, k, v, qk, qv = _decode_case(d, 16, 3, 2, 4, False, 9)
    q = np.random.default_rng(4).standard_normal((3, 3, d))
    q_pos = np.array([0, 7, 15])
    args = (p.pi, p.ck, qk.codes, qk.norm, p.cv, qv.codes, qv.norm, 0.2)
    o1, l1, _ = o.prefill_attention(q, q_pos, *args)
    codes_k2, codes_v2 = qk.codes.copy(), qv.codes.copy()
    codes_k2[8:] = (codes_k2[8:] + 1) % 4
    codes_v2[8:] = (codes_v2[8:] + 5) % 16
    o2, l2, _ = o.prefill_attention(q, q_pos, p.pi, p.ck, codes_k2, qk.norm, p.cv, codes_v2, qv.norm, 0.2)
    assert np.array_equal(o1[:2], o2[:2]) and np.array_equal(l1[:2], l2[:2])
    assert not np.allclose(o1[2], o2[2])
    assert np.allclose(o1[0], np.repeat(o.dequantize(p.pi, p.cv, qv.codes[:1], qv.norm[:1]), 3, axis=0))


# ----------------------------------------------------------------- weights
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_weight_gemm_equals_matmul_with_explicit_reconstruction(bits):
    """y = W~ x computed in rotated space equals x times the rows rebuilt
    block by block in the original space (n_b Pi^T c[codes_b]); every block
    of a row is quantized like a KV vector of its own."""
    d, n_out, n_in = 32, 7, 96
    p = o.Params(d, bits, bits, False, 3)
    rng = np.random.default_rng(bits)
    w = o.round_to_bf16(rng.standard_normal((n_out, n_in)) * rng.lognormal(0, 0.5, (n_out, 1)))
    x = rng.standard_normal((5, n_in))
    qz = o.weight_quantize(w, d, p.pi, p.ck, p.tk)
    assert qz.codes.shape == (n_out, n_in // d, d) and qz.norm.shape == (n_out, n_in // d)
    blk = o.quantize(w[3, 32:64][None], p.pi, p.ck, p.tk)        # row 3, block 1 on its own
    assert np.array_equal(blk.codes[0], qz.codes[3, 1]) and blk.norm[0] == qz.norm[3, 1]
    w_rec = np.concatenate([o.dequantize(p.pi, p.ck, qz.codes[:, b], qz.norm[:, b]) for b in range(n_in // d)],
                           axis=1)
    y = o.weight_gemm(x, p.pi, p.ck, qz.codes, qz.norm)
    assert np.allclose(y, x @ w_rec.T, rtol=1e-12, atol=1e-12)


def test_weight_reconstruction_error_matches_distortion():
    """Relative squared error of the rebuilt rows ~ the codebook's
    distortion per coordinate (the blocks are independent unit directions
    after rotation); zero rows give zero outputs."""
    d = 128
    p = o.Params(d, 4, 4, False, 42)
    rng = np.random.default_rng(0)
    w = o.round_to_bf16(rng.standard_normal((64, 512)))
    w[5] = 0.0
    qz = o.weight_quantize(w, d, p.pi, p.ck, p.tk)
    w_rec = np.concatenate([o.dequantize(p.pi, p.ck, qz.codes[:, b], qz.norm[:, b]) for b in range(4)], axis=1)
    live = np.arange(64) != 5
    rel = ((w_rec - w) ** 2).sum(axis=1)[live] / (w ** 2).sum(axis=1)[live]
    assert abs(rel.mean() / 0.009497 - 1) < 0.1
    y = o.weight_gemm(rng.standard_normal((3, 512)), p.pi, p.ck, qz.codes, qz.norm)
    assert np.all(y[:, 5] == 0)
