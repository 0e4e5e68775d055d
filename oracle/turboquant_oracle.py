"""TurboQuant KV-cache compression: plain CPU oracle (TEST INFRASTRUCTURE ONLY).

This module is the slow, obviously-correct statement of what the hot path
computes, in float64 unless the method fixes a narrower precision.  It exists
so that the CUDA library can be checked against something that shares no code
with it.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import it.  It imports nothing from the library, and the
library never imports it.

Sources (pages are cited by site, title and section; none prints a formula,
so every formula below is the plainest reading of the prose, listed as such):

* ai-accelerate.xyz TurboQuant explainer (2026-04-04), section
  "TurboQuantの仕組み", "ステップ1: PolarQuant": multiply each KV vector by a
  random orthogonal matrix so every coordinate follows a predictable,
  near-Gaussian law; quantize each coordinate on its own with the optimal
  (Lloyd-Max) scalar quantizer; keep no per-block scales or centroids.
* same page, "ステップ2: QJL": one sign bit per projected coordinate of the
  stage-1 residual corrects inner products and makes their estimate unbiased.
* same page, "ローカルLLMユーザーにとっての意味": separate K and V cache types,
  2/3/4 bits per value (turbo2/turbo3/turbo4); K and V may use different
  widths.
* qxai.app, "Tether QVACのTurboQuant実装", third paragraph: random rotation,
  scalar quantization, 1-bit quantized JL transform on the residual.

Readings where the pages are silent (each also listed in the design notes):

* coordinate law N(0, 1/d); codebook = Lloyd-Max centroids of N(0,1) / sqrt(d),
  rounded to fp16 (the precision of the stored norms; it changes the
  distortion by < 1e-5 relative); thresholds = exact midpoints of adjacent
  centroids (representable in fp32); code = #{j : t_j < y}  (a value equal to
  a threshold goes to the lower cell).
* every head vector x (bf16) is split into n = ||x||_2 and direction x/n;
  y = (Pi x)/n with Pi the bf16-rounded rotation; a vector whose stored fp16
  norm is zero (n <= 2^-25) gives y = 0, as n = 0 does.
* n is stored as fp16 (round to nearest even, saturating at 65504).
* QJL (K only, optional): r = y - c[code] in rotated, unit-direction units,
  gamma = ||r|| stored as fp16, sign bit s_m = [(S r)_m >= 0] for the d rows
  of a d x d Gaussian S; inner-product estimate
  <q_hat, r> ~= sqrt(pi/2)/d * gamma * sum_m (S q_hat)_m (2 s_m - 1).
* Pi: QR of a seeded d x d Gaussian, columns signed so diag(R) > 0, rounded to
  bf16.  S: a second seeded d x d Gaussian, rounded to fp32.  The Gaussians
  come from SplitMix64 (Steele, Lea & Flood, OOPSLA 2014) used as a
  counter-based generator and the Box-Muller transform.
* decode: q_hat = Pi q, q_tilde = S q_hat, score
  s_j = scale * n_j * (q_hat . c_K[code_j] + QJL term), softmax over j,
  o_tilde = sum_j p_j nV_j c_V[codeV_j] in rotated space, o = Pi^T o_tilde.
* weights (ai-accelerate.xyz explainer, "重みの量子化にも応用できる": the same
  algorithm applied to the weights of a linear layer): every row of W is cut
  into blocks of d coordinates, each block quantized as one vector (norm,
  rotation, codes); y = W~ x is evaluated in rotated space,
  y_i = sum_b n_ib (Pi x_b) . c[code_ib].
* prefill (prompt processing, whose cost over a compressed cache qxai.app's
  "Tether QVACのTurboQuant実装", fifth paragraph, singles out): the chunk's
  tokens are quantized into the cache first, then the query at position p
  attends over the cached positions [0, p] (causal), each query exactly as
  the decode above over that prefix.

Parity pins: every function here is checked in ``tests/test_oracle_pins.py``
against closed forms, textbook values and brute force (no function is
"parity unpinned").
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import ndtr

# --------------------------------------------------------------------------
# Counter-based random numbers (SplitMix64, Steele/Lea/Flood 2014)
# --------------------------------------------------------------------------
_MASK64 = (1 << 64) - 1
SPLITMIX_GAMMA = 0x9E3779B97F4A7C15
# The rotation Pi draws from counters 1.. ; the QJL matrix S from 2^32 + 1 ..
STREAM_PI = 0
STREAM_S = 1


def splitmix64_output(seed: int, counter: int) -> int:
    """Output number ``counter`` (1-based) of SplitMix64 started from ``seed``.

    SplitMix64 advances its state by the golden-ratio constant and returns the
    state passed through the variant-13 finaliser; the n-th output therefore
    depends only on seed + n * gamma, i.e. it is counter-based.
    """
    z = (seed + counter * SPLITMIX_GAMMA) & _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def gaussian_stream(seed: int, stream: int, count: int) -> np.ndarray:
    """``count`` standard normals of one stream, Box-Muller on 53-bit uniforms.

    Pair k uses outputs at counters base+2k+1 (u1 in (0,1]) and base+2k+2
    (u2 in [0,1)); the pair is (r cos 2 pi u2, r sin 2 pi u2) with
    r = sqrt(-2 ln u1).  Element e of the stream is component e % 2 of pair e // 2.
    """
    base = stream << 32
    out = np.empty(count, dtype=np.float64)
    two_pi = 2.0 * math.pi
    for k in range((count + 1) // 2):
        x1 = splitmix64_output(seed, base + 2 * k + 1)
        x2 = splitmix64_output(seed, base + 2 * k + 2)
        u1 = ((x1 >> 11) + 1) * (1.0 / 9007199254740992.0)
        u2 = (x2 >> 11) * (1.0 / 9007199254740992.0)
        r = math.sqrt(-2.0 * math.log(u1))
        theta = two_pi * u2
        out[2 * k] = r * math.cos(theta)
        if 2 * k + 1 < count:
            out[2 * k + 1] = r * math.sin(theta)
    return out


# --------------------------------------------------------------------------
# Roundings the method fixes
# --------------------------------------------------------------------------
def round_to_bf16(x) -> np.ndarray:
    """Round float64 values to bfloat16 (8 significant bits), ties to even.

    Valid in bf16's normal range, which covers every value the method rounds.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0), e - 8)


def round_to_fp16_sat(x) -> np.ndarray:
    """Round float64 values to IEEE fp16, ties to even, saturating at +-65504."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e = np.frexp(a)                      # leading bit has weight 2**(e-1)
    q = np.maximum(e - 11, -24)             # quantum: 11 significant bits, subnormal step 2^-24
    r = np.ldexp(np.rint(np.ldexp(a, -q)), q)
    r = np.minimum(r, 65504.0)
    return np.copysign(r, x)


def round_to_fp32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# Rotation Pi and QJL projection S
# --------------------------------------------------------------------------
def rotation_exact(d: int, seed: int) -> np.ndarray:
    """Haar-random orthogonal Q (float64) from the QR of a seeded Gaussian.

    G (d x d, row-major from the Pi stream) = Q R; the columns of Q are
    multiplied by sign(R_jj) so that R has a positive diagonal, which makes
    the factorisation unique.
    """
    g = gaussian_stream(seed, STREAM_PI, d * d).reshape(d, d)
    q, r = np.linalg.qr(g)
    sign = np.where(np.diag(r) < 0.0, -1.0, 1.0)
    return q * sign[None, :]


def rotation_bf16(d: int, seed: int) -> np.ndarray:
    """The method's Pi: the exact rotation rounded entrywise to bf16 (as float64)."""
    return round_to_bf16(rotation_exact(d, seed))


def qjl_matrix(d: int, seed: int) -> np.ndarray:
    """The QJL projection S: d x d standard normals from the S stream, in fp32."""
    return round_to_fp32(gaussian_stream(seed, STREAM_S, d * d).reshape(d, d))


# --------------------------------------------------------------------------
# Lloyd-Max scalar quantizer for N(0,1)
# --------------------------------------------------------------------------
def _phi(x):
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore"):
        return np.where(np.isinf(x), 0.0, np.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi))


def _cell_mass(a, b):
    """P(a < X <= b) for X ~ N(0,1), taking the tail that avoids cancellation."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    upper = ndtr(-a) - ndtr(-b)
    lower = ndtr(b) - ndtr(a)
    return np.where(a >= 0.0, upper, lower)


def lloyd_max_normal(bits: int, tol: float = 1e-14, max_iter: int = 200000):
    """Lloyd-Max centroids (ascending, float64) of N(0,1) for 2**bits levels.

    Lloyd's iteration: thresholds are midpoints of neighbouring centroids
    (nearest-neighbour condition) and each centroid is the conditional mean
    of its cell, (phi(a) - phi(b)) / (Phi(b) - Phi(a))  (centroid condition).
    Starts from equiprobable cells; stops when no centroid moves by more than
    ``tol``.  The result is symmetrised exactly (c_j = -c_{L-1-j}).
    """
    levels = 1 << bits
    from scipy.special import ndtri
    t = ndtri(np.arange(1, levels) / levels)
    c = None
    for _ in range(max_iter):
        a = np.concatenate(([-np.inf], t))
        b = np.concatenate((t, [np.inf]))
        c_new = (_phi(a) - _phi(b)) / _cell_mass(a, b)
        t = 0.5 * (c_new[:-1] + c_new[1:])
        if c is not None and np.max(np.abs(c_new - c)) < tol:
            c = c_new
            break
        c = c_new
    return 0.5 * (c - c[::-1])


def thresholds_of(centroids) -> np.ndarray:
    c = np.asarray(centroids, dtype=np.float64)
    return 0.5 * (c[:-1] + c[1:])


def lloyd_max_distortion(centroids) -> float:
    """Mean squared error of the quantizer on N(0,1), in closed form.

    Per cell (a, b] with centroid c:  int (x - c)^2 phi
      = P - (b phi(b) - a phi(a)) - 2 c (phi(a) - phi(b)) + c^2 P,
    from  int x^2 phi = Phi - x phi  and  int x phi = -phi.
    """
    c = np.asarray(centroids, dtype=np.float64)
    t = thresholds_of(c)
    a = np.concatenate(([-np.inf], t))
    b = np.concatenate((t, [np.inf]))
    mass = _cell_mass(a, b)
    bphi = np.where(np.isinf(b), 0.0, np.where(np.isinf(b), 0.0, b) * _phi(b))
    aphi = np.where(np.isinf(a), 0.0, np.where(np.isinf(a), 0.0, a) * _phi(a))
    per_cell = mass - (bphi - aphi) - 2.0 * c * (_phi(a) - _phi(b)) + c * c * mass
    return float(np.sum(per_cell))


# --------------------------------------------------------------------------
# Lloyd-Max scalar quantizer for the exact coordinate law of a unit vector
# --------------------------------------------------------------------------
# A coordinate X of a uniformly distributed unit vector in R^d has the density
# f(x) = (1 - x^2)^((d-3)/2) / B(1/2, (d-1)/2) on (-1, 1), i.e. (X + 1)/2 is
# Beta(a, a) with a = (d-1)/2; N(0, 1/d) is its large-d limit.  This is the
# law the rotation makes every coordinate follow exactly (the pages call it
# close to Gaussian); quantizing against it is the exact-law variant of the
# codebook.
def _sphere_mass(lo, hi, d: int):
    """P(lo < X <= hi) for the coordinate law, taking the tail that avoids
    cancellation."""
    from scipy.special import betainc
    a = 0.5 * (d - 1)
    lo = np.asarray(lo, dtype=np.float64)
    hi = np.asarray(hi, dtype=np.float64)
    upper = betainc(a, a, 0.5 * (1.0 - lo)) - betainc(a, a, 0.5 * (1.0 - hi))
    lower = betainc(a, a, 0.5 * (1.0 + hi)) - betainc(a, a, 0.5 * (1.0 + lo))
    return np.where(lo >= 0.0, upper, lower)


def _sphere_first_moment(lo, hi, d: int):
    """int_lo^hi x f(x) dx = ((1 - lo^2)^a - (1 - hi^2)^a) / (2 a B(1/2, a)),
    a = (d-1)/2, since d/dx (1 - x^2)^a = -2 a x (1 - x^2)^(a-1)."""
    from scipy.special import beta
    a = 0.5 * (d - 1)
    lo = np.asarray(lo, dtype=np.float64)
    hi = np.asarray(hi, dtype=np.float64)
    return ((1.0 - lo * lo) ** a - (1.0 - hi * hi) ** a) / (2.0 * a * beta(0.5, a))


def lloyd_max_sphere(bits: int, d: int, tol: float = 1e-15, max_iter: int = 2000000):
    """Lloyd-Max centroids (ascending, float64) of the coordinate law of a
    uniform unit vector in R^d, for 2**bits levels.

    The same two optimality conditions as for N(0,1): thresholds at midpoints,
    centroids at the conditional means int x f / int f of their cells.  Starts
    from equiprobable cells; stops when no centroid moves by more than
    ``tol``; symmetrised exactly.
    """
    from scipy.special import betaincinv
    levels = 1 << bits
    a = 0.5 * (d - 1)
    t = 2.0 * betaincinv(a, a, np.arange(1, levels) / levels) - 1.0
    c = None
    for _ in range(max_iter):
        lo = np.concatenate(([-1.0], t))
        hi = np.concatenate((t, [1.0]))
        c_new = _sphere_first_moment(lo, hi, d) / _sphere_mass(lo, hi, d)
        t = 0.5 * (c_new[:-1] + c_new[1:])
        if c is not None and np.max(np.abs(c_new - c)) <= tol:
            c = c_new
            break
        c = c_new
    return 0.5 * (c - c[::-1])


def sphere_distortion(centroids, d: int) -> float:
    """Mean squared error of the quantizer on the coordinate law, in closed
    form: per cell, int (x - c)^2 f = M2 - 2 c M1 + c^2 P, where the second
    moment uses x^2 (1 - x^2)^(a-1) = (1 - x^2)^(a-1) - (1 - x^2)^a, i.e.
    M2 = P_d - (d-1)/d P_(d+2) with P_d the cell's mass under dimension d."""
    c = np.asarray(centroids, dtype=np.float64)
    t = thresholds_of(c)
    lo = np.concatenate(([-1.0], t))
    hi = np.concatenate((t, [1.0]))
    mass = _sphere_mass(lo, hi, d)
    m1 = _sphere_first_moment(lo, hi, d)
    m2 = mass - (d - 1) / d * _sphere_mass(lo, hi, d + 2)
    return float(np.sum(m2 - 2.0 * c * m1 + c * c * mass))


LAW_GAUSSIAN, LAW_SPHERE = "gaussian", "sphere"


def codebook(bits: int, d: int, law: str = LAW_GAUSSIAN):
    """The method's codebook: (centroids, thresholds) as float64.

    law "gaussian" (the reading the build defaults to): the N(0,1) Lloyd-Max
    centroids divided by sqrt(d), for the N(0, 1/d) law.  law "sphere": the
    Lloyd-Max centroids of the exact coordinate law of a unit vector in R^d.
    Centroids are rounded to fp16; thresholds are the exact midpoints of
    adjacent centroids."""
    if law == LAW_GAUSSIAN:
        c = round_to_fp16_sat(lloyd_max_normal(bits) / math.sqrt(d))
    elif law == LAW_SPHERE:
        c = round_to_fp16_sat(lloyd_max_sphere(bits, d))
    else:
        raise ValueError(f"unknown codebook law {law!r}")
    t = 0.5 * (c[:-1] + c[1:])
    return c, t


# --------------------------------------------------------------------------
# Bit layouts of one packed vector
# --------------------------------------------------------------------------
def code_bit_position(bits: int, d: int) -> np.ndarray:
    """Table pos[i, k]: bit index (within the vector's little-endian byte
    string) of bit k of coordinate i's code.

    * 2 and 4 bits: plain LSB-first stream, bit k of code i at i*bits + k.
    * 3 bits: groups of 32 coordinates in 12 bytes (three little-endian 32-bit
      words w0..w2).  Local coordinate l < 24 keeps its three bits in nibble
      l % 8 of word l // 8 (bits 4*(l%8) .. 4*(l%8)+2); for l >= 24, bit k of
      the code is bit 4*(l-24)+3 of word k.  Every code therefore sits in the
      low three bits of a nibble or in the spare top bits of one nibble
      column, which the decode kernel turns into byte-permute selectors
      cheaply.
    """
    pos = np.zeros((d, bits), dtype=np.int64)
    if bits in (1, 2, 4, 8) or bits > 4:
        for i in range(d):
            for k in range(bits):
                pos[i, k] = i * bits + k
        return pos
    assert bits == 3 and d % 32 == 0
    for i in range(d):
        g, l = divmod(i, 32)
        base = 96 * g
        for k in range(3):
            if l < 24:
                word, nib = divmod(l, 8)
                pos[i, k] = base + 32 * word + 4 * nib + k
            else:
                pos[i, k] = base + 32 * k + 4 * (l - 24) + 3
    return pos


def pack_codes(codes, bits: int) -> np.ndarray:
    """codes [N, d] ints in [0, 2**bits) -> bytes [N, d*bits/8] (uint8)."""
    codes = np.asarray(codes, dtype=np.int64)
    n, d = codes.shape
    pos = code_bit_position(bits, d)
    nbits = d * bits
    stream = np.zeros((n, nbits), dtype=np.uint8)
    for k in range(bits):
        stream[:, pos[:, k]] = ((codes >> k) & 1).astype(np.uint8)
    return np.packbits(stream, axis=1, bitorder="little")


def unpack_codes(packed, bits: int, d: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    stream = np.unpackbits(packed, axis=1, bitorder="little").astype(np.int64)
    pos = code_bit_position(bits, d)
    codes = np.zeros((packed.shape[0], d), dtype=np.int64)
    for k in range(bits):
        codes |= stream[:, pos[:, k]] << k
    return codes


def pack_signs(bits01) -> np.ndarray:
    """QJL sign bits [N, d] in {0,1} -> [N, d/8] bytes, bit m at position m."""
    return np.packbits(np.asarray(bits01, dtype=np.uint8), axis=1, bitorder="little")


def unpack_signs(packed, d: int) -> np.ndarray:
    return np.unpackbits(np.asarray(packed, dtype=np.uint8), axis=1,
                         bitorder="little")[:, :d].astype(np.int64)


# --------------------------------------------------------------------------
# Quantize-on-append (stage 1 rotation + Lloyd-Max, optional stage 2 QJL)
# --------------------------------------------------------------------------
class Quantized:
    """Result of quantizing N head vectors (all fields numpy arrays)."""

    def __init__(self, codes, norm, y, qjl_signs=None, qjl_gamma=None, qjl_proj=None):
        self.codes = codes          # [N, d] int code = index of the centroid
        self.norm = norm            # [N] fp16 values (float64)
        self.y = y                  # [N, d] rotated unit-direction coordinates (float64)
        self.qjl_signs = qjl_signs  # [N, d] {0,1} or None
        self.qjl_gamma = qjl_gamma  # [N] fp16 values or None
        self.qjl_proj = qjl_proj    # [N, d] float64 S r or None


def quantize(x, pi, centroids, thresholds, s_matrix=None, chunk: int = 8192) -> Quantized:
    """Quantize rows of x ([N, d], the exact bf16 values as float64).

    n = ||x||;  y = (Pi x) / n;  code_i = #{j : t_j < y_i};  stored norm =
    fp16(n).  A vector whose stored norm is zero (n <= 2^-25, below half the
    smallest fp16 subnormal) is stored as the zero vector: y = 0 (codes
    2^(b-1) - 1), since its reconstruction fp16(n) Pi^T c[code] is zero
    whatever the codes.  With ``s_matrix``: r = y - c[code], gamma = ||r||
    (stored as fp16), sign bit m = [(S r)_m >= 0].
    """
    x = np.asarray(x, dtype=np.float64)
    c = np.asarray(centroids, dtype=np.float64)
    t = np.asarray(thresholds, dtype=np.float64)
    n_rows = x.shape[0]
    codes = np.empty(x.shape, dtype=np.int64)
    ys = np.empty(x.shape, dtype=np.float64)
    norms = np.sqrt(np.sum(x * x, axis=1))
    stored = round_to_fp16_sat(norms)
    for s0 in range(0, n_rows, chunk):
        xb = x[s0:s0 + chunk]
        nb = norms[s0:s0 + chunk]
        live = stored[s0:s0 + chunk] > 0.0
        z = xb @ pi.T
        safe = np.where(live, nb, 1.0)
        y = np.where(live[:, None], z / safe[:, None], 0.0)
        ys[s0:s0 + chunk] = y
        # code = number of thresholds strictly below y
        codes[s0:s0 + chunk] = np.sum(y[:, :, None] > t[None, None, :], axis=2)
    out = Quantized(codes, stored, ys)
    if s_matrix is not None:
        r = ys - c[codes]
        gamma = np.sqrt(np.sum(r * r, axis=1))
        proj = r @ np.asarray(s_matrix, dtype=np.float64).T
        out.qjl_signs = (proj >= 0.0).astype(np.int64)
        out.qjl_gamma = round_to_fp16_sat(gamma)
        out.qjl_proj = proj
    return out


def qjl_inner_product(q_tilde, signs, gamma, d: int):
    """QJL estimate of <q_hat, r>: sqrt(pi/2)/d * gamma * sum_m q_tilde_m (2 s_m - 1).

    q_tilde [..., d] = S q_hat; signs [T, d] in {0,1}; gamma [T].  Returns
    [..., T].  The constant follows from E[<s,q> sign(<s,r>)] =
    sqrt(2/pi) <q,r>/||r|| for a standard normal row s.
    """
    pm = 2.0 * np.asarray(signs, dtype=np.float64) - 1.0
    return math.sqrt(math.pi / 2.0) / d * np.asarray(gamma)[None, :] * (np.asarray(q_tilde) @ pm.T)


# --------------------------------------------------------------------------
# Decode attention read from the packed representation
# --------------------------------------------------------------------------
def decode_attention(q, pi, centroids_k, codes_k, norm_k, centroids_v, codes_v, norm_v,
                     scale, s_matrix=None, qjl_signs=None, qjl_gamma=None):
    """Attention of G query heads over T cached tokens of one (sequence, KV head).

    q [G, d] float64; codes_* [T, d]; norm_* [T] (stored fp16 values).
    q_hat = Pi q, q_tilde = S q_hat;
    s_gj = scale * nK_j * (q_hat_g . cK[code_j] + QJL term);
    p = softmax_j(s);  o_tilde_g = sum_j p_gj nV_j cV[codeV_j];  o_g = Pi^T o_tilde_g.
    Returns (o [G, d], lse [G], scores [G, T]).
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[-1]
    q_hat = q @ pi.T
    dots = q_hat @ np.asarray(centroids_k)[codes_k].T
    if s_matrix is not None:
        q_tilde = q_hat @ np.asarray(s_matrix, dtype=np.float64).T
        dots = dots + qjl_inner_product(q_tilde, qjl_signs, qjl_gamma, d)
    scores = scale * np.asarray(norm_k)[None, :] * dots
    m = np.max(scores, axis=1)
    p = np.exp(scores - m[:, None])
    l = np.sum(p, axis=1)
    o_tilde = (p * np.asarray(norm_v)[None, :]) @ np.asarray(centroids_v)[codes_v]
    o = (o_tilde / l[:, None]) @ pi          # row form of Pi^T o_tilde
    return o, m + np.log(l), scores


def prefill_attention(q, q_pos, pi, centroids_k, codes_k, norm_k, centroids_v, codes_v, norm_v, scale,
                      s_matrix=None, qjl_signs=None, qjl_gamma=None):
    """Causal attention of a chunk of queries over one (sequence, KV head)'s
    packed cache: the query at position q_pos[t] attends over the cached
    positions [0, q_pos[t]], exactly as decode_attention over that prefix.

    q [n, G, d] float64; q_pos [n] (each below the cached length); codes_*,
    norm_*, qjl_* as decode_attention, over the whole cached sequence.
    Returns (o [n, G, d], lse [n, G], max_abs_score [n, G]), the last being
    max_j |s_j| over each query's prefix.
    """
    q = np.asarray(q, dtype=np.float64)
    o = np.empty(q.shape)
    lse = np.empty(q.shape[:2])
    smax = np.empty(q.shape[:2])
    for t, p in enumerate(np.asarray(q_pos, dtype=np.int64)):
        n = int(p) + 1
        o[t], lse[t], sc = decode_attention(
            q[t], pi, centroids_k, codes_k[:n], norm_k[:n], centroids_v, codes_v[:n], norm_v[:n], scale,
            s_matrix=s_matrix, qjl_signs=None if qjl_signs is None else qjl_signs[:n],
            qjl_gamma=None if qjl_gamma is None else qjl_gamma[:n])
        smax[t] = np.abs(sc).max(axis=1)
    return o, lse, smax


def weight_quantize(w, d, pi, centroids, thresholds) -> Quantized:
    """Rows of W [n_out, n_in] (n_in a multiple of d) cut into n_in / d blocks of
    d coordinates, every block quantized as one vector.  Returns the Quantized
    fields with shapes [n_out, n_in / d, ...] (codes [n_out, n_blocks, d], norm
    [n_out, n_blocks])."""
    w = np.asarray(w, dtype=np.float64)
    n_out, n_in = w.shape
    qz = quantize(w.reshape(n_out * (n_in // d), d), pi, centroids, thresholds)
    nb = n_in // d
    return Quantized(qz.codes.reshape(n_out, nb, d), qz.norm.reshape(n_out, nb), qz.y.reshape(n_out, nb, d))


def weight_gemm(x, pi, centroids, codes, norm):
    """y = W~ x for the block-quantized rows, in rotated space:
    y[t, i] = sum_b norm[i, b] (Pi x[t, b]) . c[codes[i, b]].
    x [n_tok, n_in] float64; codes [n_out, n_blocks, d]; norm [n_out, n_blocks].
    Returns y [n_tok, n_out]."""
    x = np.asarray(x, dtype=np.float64)
    n_out, nb, d = codes.shape
    xb = x.reshape(x.shape[0], nb, d)
    x_hat = np.einsum("ij,tbj->tbi", pi, xb)                 # Pi x_tb
    c = np.asarray(centroids)[codes]                          # [n_out, nb, d]
    return np.einsum("tbk,obk,ob->to", x_hat, c, np.asarray(norm, dtype=np.float64))


def exact_attention(q, k, v, scale):
    """Plain softmax attention in float64: (o [G, d], lse [G])."""
    s = scale * (np.asarray(q, dtype=np.float64) @ np.asarray(k, dtype=np.float64).T)
    m = np.max(s, axis=1)
    p = np.exp(s - m[:, None])
    l = np.sum(p, axis=1)
    return (p @ np.asarray(v, dtype=np.float64)) / l[:, None], m + np.log(l)


def dequantize(pi, centroids, codes, norm):
    """Explicit reconstruction in the original space: n * Pi^T c[code] (rows)."""
    return np.asarray(norm)[:, None] * (np.asarray(centroids)[codes] @ pi)


def cosine_similarity(a, b) -> float:
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


class Params:
    """Everything tq_create(d, bits_k, bits_v, qjl, seed) fixes, computed here
    independently of the library."""

    def __init__(self, d: int, bits_k: int, bits_v: int, qjl: bool, seed: int, law: str = LAW_GAUSSIAN):
        self.d, self.bits_k, self.bits_v, self.qjl, self.seed = d, bits_k, bits_v, bool(qjl), seed
        self.law = law
        self.pi = rotation_bf16(d, seed)
        self.ck, self.tk = codebook(bits_k, d, law)
        self.cv, self.tv = codebook(bits_v, d, law)
        self.s = qjl_matrix(d, seed) if qjl else None
