"""CPU oracle for the rotated W4A4 linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module.  The product path (the CUDA library and its Python
binding) never imports, links or calls it, and this module imports nothing from
the product: the two share only the seeded input generators.

What it computes, in plain numpy, step by step as the pages state it:

* the randomized permuted block-Hadamard (RPBH) rotation R = BlockDiag(H_b/sqrt b) P D
  (OrbitQuant abstract: random signs, a permutation and block Hadamard
  transforms, the RPBH rotation;
  TR-DQ section 3.2, Eq. 8: block-diagonal rotation with K = C_in / 2^n blocks;
  TR-DQ section 3.2: a permutation is itself orthogonal);
* folding the rotation into the weights, W' = W R^T, so that it cancels inside
  the layer (OrbitQuant abstract; TR-DQ Eq. 9);
* per-token normalisation and 4-bit quantization of the rotated row with
  - a symmetric uniform INT4 grid (TR-DQ section 3.1, Eq. 1-3, symmetric form),
  - a Lloyd-Max codebook for the known marginal of a rotated, normalised
    coordinate (OrbitQuant abstract),
  - NVFP4: e2m1 elements with 16-element e4m3 block scales (DiRotQ abstract:
    NVFP4 on Blackwell);
* the DiRotQ low-rank branch: r PCA coefficients kept in BF16 and the residual
  quantized (DiRotQ abstract);
* DiRotQ's full PCA rotation y = x V, its first r coordinates in BF16 and the
  rest quantized (DiRotQ abstract);
* TR-DQ's zigzag permutation and double block rotation (section 3.2, Eq. 9),
  asymmetric per-token INT4 (section 3.1, Eq. 1-3) and the 8-bit per-token /
  per-channel quantizer of the W4A8 and W8A8 settings (section 3.1, Tables 1-5);
* the FP64 reference GEMM over the dequantized values.

Readings taken where the pages are silent:
FP32 arithmetic with round-to-nearest-even and no fused multiply-add except
where a product is exact; butterfly stages in ascending stride; a perfect
pairwise sum of squares inside each block and a sequential sum over blocks;
the PCA coefficients summed per 128-channel chunk in k order, chunks added in
order, the residual subtracted in order of j; signs applied before the
permutation; SplitMix64 for the rotation's random draws.

Parity status of each function is stated in its docstring ("pinned by ...").
"""
from __future__ import annotations

import math

import numpy as np

INT4, LM16, NVFP4, LM4, INT4A, INT8 = 1, 2, 3, 4, 5, 6

MASK64 = (1 << 64) - 1
F32 = np.float32


# ----------------------------------------------------------------------------
# Random draws: SplitMix64 (Steele, Lea & Flood 2014, "Fast splittable
# pseudorandom number generators"; the 64-bit finaliser constants are the
# published ones of that generator).
# ----------------------------------------------------------------------------
class SplitMix64:
    """SplitMix64: state += 0x9E3779B97F4A7C15, output = mix(state).

    Pinned by: tests/test_oracle_rotation.py (bijective permutations, sign
    balance, uniformity of the Fisher-Yates draw on tiny K) and by the stored
    first outputs in tests/golden/splitmix64.txt."""

    GAMMA = 0x9E3779B97F4A7C15

    def __init__(self, seed: int):
        self.state = seed & MASK64

    def next(self) -> int:
        self.state = (self.state + self.GAMMA) & MASK64
        z = self.state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        return z ^ (z >> 31)

    def below(self, n: int) -> int:
        """Uniform integer in [0, n) by rejection: drop draws at or above the
        largest multiple of n that fits in 2^64, then reduce modulo n."""
        limit = (1 << 64) - ((1 << 64) % n)
        while True:
            z = self.next()
            if z < limit:
                return z % n


def make_rotation(K: int, block: int, seed: int):
    """RPBH rotation parameters: signs D (int8 +-1, length K) and the fixed
    permutation P (int32, length K).

    OrbitQuant abstract ("randomized permuted block-Hadamard"): a random sign per
    channel, one fixed random permutation of all K channels, then a Hadamard
    transform per block of ``block`` channels (TR-DQ section 3.2, Eq. 8).
    Reading: signs are drawn first (sign k is negative when bit 63 of draw k is
    set), then the permutation by a Fisher-Yates shuffle of 0..K-1 from the top
    index down, each swap partner drawn uniformly with ``SplitMix64.below``.

    Pinned by: tests/test_oracle_rotation.py (perm is a bijection, R is
    orthogonal, Fisher-Yates uniformity on K=4)."""
    if block < 2 or block & (block - 1) or K % block:
        raise ValueError("block must be a power of two dividing K")
    g = SplitMix64(seed)
    sign = np.empty(K, dtype=np.int8)
    for k in range(K):
        sign[k] = -1 if (g.next() >> 63) else 1
    perm = list(range(K))
    for i in range(K - 1, 0, -1):
        j = g.below(i + 1)
        perm[i], perm[j] = perm[j], perm[i]
    return sign, np.asarray(perm, dtype=np.int32)


# ----------------------------------------------------------------------------
# Rotation
# ----------------------------------------------------------------------------
def fwht_blocks(v: np.ndarray, block: int) -> np.ndarray:
    """Unnormalised Walsh-Hadamard transform of every ``block``-wide block of
    each row (Sylvester natural order): stages h = 1, 2, 4, ..., block/2; in each
    stage every pair (i, i+h) with bit h of i clear becomes (v_i + v_{i+h},
    v_i - v_{i+h}).  Works in the dtype of ``v`` (float32 for the contract,
    float64 for the exact checks).

    Pinned by: brute-force dense H_b (Sylvester recursion) at b in {2,4,8,16}
    and H_b H_b^T = b I (tests/test_oracle_rotation.py)."""
    rows, K = v.shape
    assert K % block == 0
    v = v.copy()
    h = 1
    while h < block:
        t = v.reshape(rows, K // (2 * h), 2, h)
        a = t[:, :, 0, :].copy()
        b = t[:, :, 1, :].copy()
        t[:, :, 0, :] = a + b
        t[:, :, 1, :] = a - b
        h *= 2
    return v


def permute_sign(x: np.ndarray, sign: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """(P D x)_i = sign[perm[i]] * x[perm[i]] for every row (exact)."""
    return x[:, perm] * sign[perm].astype(x.dtype)


def rotate(x: np.ndarray, sign, perm, block: int) -> np.ndarray:
    """y = R x for every row: signs, permutation, block FWHT, then one multiply by
    the FP32 (or FP64) value of 1/sqrt(block).  float32 input follows the FP32
    contract; float64 input gives the exact rotation for the checks."""
    dt = x.dtype
    v = fwht_blocks(permute_sign(x, sign, perm), block)
    return v * dt.type(1.0 / math.sqrt(block))


def rotation_matrix(K: int, sign, perm, block: int) -> np.ndarray:
    """Dense R (FP64), column k = R e_k; for the orthogonality checks only."""
    return rotate(np.eye(K, dtype=np.float64), sign, perm, block).T


# ----------------------------------------------------------------------------
# TR-DQ: zigzag permutation and double block rotation (section 3.2, Eq. 9)
# ----------------------------------------------------------------------------
def zigzag_permutation(channel_mag, block: int) -> np.ndarray:
    """The zigzag permutation P of TR-DQ section 3.2: channels ranked by
    activation magnitude, largest first (equal magnitudes: lower channel index
    first), are dealt to the K/block blocks back and forth -- the first
    K/block to blocks 0, 1, ..., K/block - 1, the next K/block to blocks
    K/block - 1, ..., 0, and so on -- and inside a block they keep the order in
    which they were dealt.  Returns perm with output position i reading channel
    perm[i] (a permutation matrix, orthogonal as the paper notes).

    Pinned by: tests/test_oracle_trdq.py (a hand-dealt K = 8 example, the
    bijection, and the rank balance between blocks)."""
    mag = np.asarray(channel_mag, dtype=np.float64)
    K = mag.size
    if block < 1 or K % block:
        raise ValueError("block must divide K")
    nblk = K // block
    order = np.lexsort((np.arange(K), -mag))        # magnitude descending, then index
    perm = np.empty(K, dtype=np.int32)
    for t, c in enumerate(order):
        rnd, i = divmod(t, nblk)
        blk = i if rnd % 2 == 0 else nblk - 1 - i
        perm[blk * block + rnd] = c
    return perm


def zigzag_from_calibration(calib_f32: np.ndarray, sign, block: int) -> np.ndarray:
    """Zigzag permutation from calibration tokens (TR-DQ section 3.2): the
    channel magnitudes are max over tokens of |(x R1)_j|, R1 the first block
    rotation (signs, no permutation, block FWHT, FP32 contract)."""
    K = calib_f32.shape[1]
    y1 = rotate(np.asarray(calib_f32, dtype=F32), sign, np.arange(K, dtype=np.int32), block)
    return zigzag_permutation(np.max(np.abs(y1), axis=0), block)


def rotate_double(x: np.ndarray, sign, zz_perm, block: int) -> np.ndarray:
    """TR-DQ Eq. 9, activation side: y = R2 P R1 x with R1 the first block
    rotation (random signs on the natural channel order, orthonormal FWHT per
    block), P the zigzag permutation and R2 a second orthonormal FWHT per block.
    Each rotation follows the FP32 contract of ``rotate`` (reading: the two
    block rotations are RPBH rotations of their own -- signs only on the first,
    the zigzag as the permutation of the second).  The weight side folds the
    same R into W (``rotate_quantize(..., double=...)``).

    Pinned by: tests/test_oracle_trdq.py (equal to the product of the dense
    matrices; orthogonal; cancels inside the layer in FP64)."""
    K = x.shape[1]
    y1 = rotate(x, sign, np.arange(K, dtype=np.int32), block)
    return rotate(y1, np.ones(K, dtype=np.int8), zz_perm, block)


# ----------------------------------------------------------------------------
# Number formats (OCP Microscaling Formats specification v1.0: FP8 E4M3 and
# FP4 E2M1 element encodings; NVFP4 uses E4M3 as an unsigned block scale)
# ----------------------------------------------------------------------------
def _grid_round(a: np.ndarray, values: np.ndarray) -> np.ndarray:
    """Index of the nearest entry of the ascending non-negative grid ``values``
    for every |a|, ties to the even index (= even mantissa bit), saturating at
    the last entry.  Exact in FP64 for FP32 inputs."""
    a = np.abs(a.astype(np.float64))
    idx = np.searchsorted(values, a, side="right") - 1          # values[idx] <= a
    idx = np.clip(idx, 0, len(values) - 1)
    hi = np.minimum(idx + 1, len(values) - 1)
    lo_v = values[idx]
    hi_v = values[hi]
    d_lo = a - lo_v
    d_hi = hi_v - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (idx % 2 == 1))
    take_hi &= hi != idx
    return np.where(take_hi, hi, idx)


def _e4m3_grid() -> np.ndarray:
    """All non-negative finite E4M3 values by code 0x00..0x7E (bias 7; exponent
    field 0 is subnormal m/8 * 2^-6; code 0x7F is NaN, so 448 is the largest)."""
    vals = []
    for code in range(0x7F):
        e, m = code >> 3, code & 7
        vals.append((m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7))
    return np.asarray(vals, dtype=np.float64)


E4M3_GRID = _e4m3_grid()
E2M1_GRID = np.asarray([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e4m3_encode(a: np.ndarray) -> np.ndarray:
    """FP32 -> E4M3 byte, round to nearest even, saturating to +-448 (satfinite).
    The sign bit is kept for negative inputs, -0.0 included.

    Pinned by: grid facts of the OCP definition (max 448, min subnormal 2^-9,
    ties to even mantissa) and torch's float8_e4m3fn cast in
    tests/test_oracle_formats.py, and by the GPU's cvt.rn.satfinite.e4m3x2.f32
    over FP32 patterns spanning the format's range, every midpoint +-1 ulp and
    the saturation edges (tests/test_gpu_formats.py)."""
    a = np.asarray(a, dtype=np.float32)
    code = _grid_round(a, E4M3_GRID).astype(np.uint8)
    return code | np.where(np.signbit(a), np.uint8(0x80), np.uint8(0))


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8)
    mag = E4M3_GRID[np.minimum(code & 0x7F, 0x7E)]
    return np.where(code & 0x80, -mag, mag)


def e2m1_encode(a: np.ndarray) -> np.ndarray:
    """FP32 -> E2M1 nibble (sign in bit 3), round to nearest even, saturating to
    +-6.  Pinned by the grid, tie and saturation cases and a brute-force
    nearest-value search in tests/test_oracle_formats.py, and by the GPU's
    cvt.rn.satfinite.e2m1x2.f32 (tests/test_gpu_formats.py)."""
    a = np.asarray(a, dtype=np.float32)
    code = _grid_round(a, E2M1_GRID).astype(np.uint8)
    return code | np.where(np.signbit(a), np.uint8(8), np.uint8(0))


def e2m1_decode(code: np.ndarray) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8)
    mag = E2M1_GRID[code & 7]
    return np.where(code & 8, -mag, mag)


# ----------------------------------------------------------------------------
# Lloyd-Max codebook for the marginal of a rotated, normalised coordinate
# ----------------------------------------------------------------------------
def _log_gamma_ratio_half(twice_q: int) -> float:
    """log(Gamma(q + 1/2) / Gamma(q)) for q = twice_q / 2, by the exact product
    over the Gamma recurrence (accurate to ~1e-15 where library log-Beta values
    lose ~1e-12 to cancellation at these large arguments)."""
    if twice_q % 2:                        # q = n + 1/2: Gamma(n+1)/Gamma(n+1/2)
        n = (twice_q - 1) // 2
        return -0.5 * math.log(math.pi) + math.fsum(math.log1p(1.0 / (2 * i - 1)) for i in range(1, n + 1))
    n = twice_q // 2                       # q = n: n Gamma(n+1/2)/Gamma(n+1)
    return math.log(n) + 0.5 * math.log(math.pi) - math.fsum(
        math.log1p(1.0 / (2 * i - 1)) for i in range(1, n + 1))


def sphere_marginal_logc(K: int) -> float:
    """log of the density constant: f(u) = C (1 - u^2/K)^((K-3)/2) on |u| < sqrt K,
    the law of sqrt(K) times one coordinate of a uniform point on S^{K-1}.
    C = 1 / (sqrt(K) B(1/2, (K-1)/2)) and B(1/2, q) = sqrt(pi) Gamma(q)/Gamma(q+1/2)."""
    return -0.5 * math.log(K) - 0.5 * math.log(math.pi) + _log_gamma_ratio_half(K - 1)


def _half_mass(K: int, a: float, b: float) -> float:
    """P(a < U < b) for 0 <= a < b <= sqrt K: u^2/K ~ Beta(1/2, (K-1)/2), so the
    mass is (Ic(a^2/K) - Ic(b^2/K)) / 2 with Ic the regularised upper incomplete
    beta function (kept in complemented form so tails do not cancel)."""
    from scipy.special import betaincc
    p, q = 0.5, (K - 1) / 2.0
    ia = betaincc(p, q, min(a * a / K, 1.0))
    ib = betaincc(p, q, min(b * b / K, 1.0)) if b < math.sqrt(K) else 0.0
    return 0.5 * (ia - ib)


def _half_moment(K: int, a: float, b: float, logc: float) -> float:
    """Integral of u f(u) over (a, b): C K / (2(alpha+1)) [(1-a^2/K)^(alpha+1) -
    (1-b^2/K)^(alpha+1)] (closed form of the antiderivative)."""
    alpha = (K - 3) / 2.0

    def g(u):
        t = 1.0 - u * u / K
        return 0.0 if t <= 0 else math.exp((alpha + 1.0) * math.log1p(-u * u / K))

    return math.exp(logc) * K / (2.0 * (alpha + 1.0)) * (g(a) - g(b))


def lloyd_max(K: int, levels: int, tol: float = 1e-13, max_iter: int = 200000):
    """Symmetric Lloyd-Max quantizer with ``levels`` levels (4 or 16) for the
    density of a sqrt(K)-scaled coordinate of a uniform point on S^{K-1}
    (OrbitQuant abstract: after RPBH each coordinate concentrates on one fixed,
    known marginal, so one Lloyd-Max codebook serves a given input dimension).

    Lloyd's conditions: every centroid is the conditional mean of its cell and
    every boundary is the midpoint of its two centroids.  FP64 Lloyd iteration on
    the positive half (the density is even, so the solution is symmetric with a
    boundary at 0), from evenly spaced centroids, until no value moves more than
    ``tol``.

    Returns (centroids[levels], boundaries[levels-1]) ascending, FP64.

    Pinned by: the fixed-point residuals against direct numerical integration
    of the density (scipy.integrate.quad), total mass 1 and E[U^2] = 1, and the
    Gaussian limit (Max 1960: 4 levels at +-0.4528, +-1.510) in
    tests/test_oracle_codebook.py."""
    if levels % 2:
        raise ValueError("even number of levels")
    h = levels // 2
    logc = sphere_marginal_logc(K)
    top = math.sqrt(K)
    c = [(i + 0.5) * 3.0 / h for i in range(h)]        # positive centroids
    for _ in range(max_iter):
        bnd = [0.0] + [(c[i] + c[i + 1]) / 2.0 for i in range(h - 1)] + [top]
        new = [_half_moment(K, bnd[i], bnd[i + 1], logc) / _half_mass(K, bnd[i], bnd[i + 1])
               for i in range(h)]
        delta = max(abs(x - y) for x, y in zip(new, c))
        c = new
        if delta < tol:
            break
    else:
        raise RuntimeError("Lloyd iteration did not converge")
    pos_b = [(c[i] + c[i + 1]) / 2.0 for i in range(h - 1)]
    cent = np.asarray([-v for v in reversed(c)] + c)
    bnds = np.asarray([-v for v in reversed(pos_b)] + [0.0] + pos_b)
    return cent, bnds


def codebook_tables(K: int, levels: int):
    """The two tables the quantizer uses: FP32 boundaries (rounded from FP64) for
    choosing codes, and the E4M3 bytes of the centroids used by the FP8 GEMM
    (reading: the GEMM needs exactly representable e4m3 operands, so centroids
    are rounded to the nearest e4m3 value)."""
    cent, bnd = lloyd_max(K, levels)
    return bnd.astype(np.float32), e4m3_encode(cent.astype(np.float32))


# ----------------------------------------------------------------------------
# Low-rank (PCA) branch
# ----------------------------------------------------------------------------
def pca_basis(calib_f32: np.ndarray, r: int):
    """Top-r eigenvectors of the uncentered second moment X^T X / n of the
    calibration tokens (DiRotQ abstract: a low-rank subspace capturing dominant
    activation variance via PCA).  FP64; sign fixed so that the largest-magnitude
    entry of each vector is positive.  Returns (U float64 K x r, eigenvalues r).

    Pinned by: U^T U = I, the eigen-equation residual, descending order and
    the sign rule (tests/test_oracle_quant.py::test_pca_basis)."""
    X = calib_f32.astype(np.float64)
    S = X.T @ X / X.shape[0]
    w, V = np.linalg.eigh(S)
    order = np.argsort(w)[::-1][:r]
    w, V = w[order], V[:, order]
    idx = np.argmax(np.abs(V), axis=0)
    V = V * np.sign(V[idx, np.arange(r)])[None, :]
    return V, w


PROJ_CHUNK = 128


def rotate_pca(x_f32: np.ndarray, V_f32: np.ndarray) -> np.ndarray:
    """DiRotQ's full rotation (DiRotQ abstract: the activations rotated into a
    PCA basis, the dominant coordinates kept at higher precision): y = x V with
    V the K x K basis (BF16 values).  Reading: the plain definition, the sum of
    the (exact) products formed in FP64 and rounded once to FP32 -- a tensor
    core's FP32 accumulation is held to it by an error bound, not bit for bit.

    Pinned by: tests/test_oracle_pca_full.py (exact on integer inputs, against
    a float64 loop, orthogonal V preserves norms)."""
    return (np.asarray(x_f32, np.float64) @ np.asarray(V_f32, np.float64)).astype(F32)


def quantize_pca(y_f32: np.ndarray, r: int, fmt: int = INT4, weight_rows: bool = False, group: int = 128):
    """The DiRotQ split of a rotated row (DiRotQ abstract): the first r
    coordinates (the dominant principal directions) kept in BF16 as c, the
    remaining ones quantized.  Reading: the quantized row keeps all K
    positions with the first r set to zero (codes 0), so that the 4-bit GEMM
    runs over K and c L^T adds the r coordinates back.  INT4: per-token absmax
    (activations) or one scale per 128 coordinates (weight rows).
    Returns dict(q, codes, scale, coef)."""
    y = np.asarray(y_f32, F32)
    coef = _bf16_bits(np.ascontiguousarray(y[:, :r]))
    ylo = y.copy()
    ylo[:, :r] = 0
    if fmt != INT4:
        raise ValueError("the PCA rotation quantizes to INT4")
    q, s = quant_int4(ylo, group if weight_rows else None)
    return {"q": q, "codes": pack_nibbles(q), "scale": np.ascontiguousarray(s.T) if weight_rows else s[:, 0],
            "coef": coef, "block_scale": None, "zero_point": None}


def project_coefficients(x_f32: np.ndarray, U_f32: np.ndarray) -> np.ndarray:
    """c = x U in FP32 (DiRotQ abstract: the coefficients of the activation in
    the PCA subspace), returned as FP32 values before their BF16 rounding.

    Reading of the summation order (the pages fix none): the K input channels
    are cut into chunks of 128 consecutive channels; inside a chunk the
    products x_k U_kj are added one after another in natural k order, starting
    from the first product; the chunk partials are then added in chunk order,
    starting from chunk 0.  Every product of two BF16 values is exact in FP32
    (16 significant bits; magnitudes here stay far from the FP32 subnormal
    range), so "add the product" and "fused multiply-add" give the same value.
    K must be a multiple of 128.

    Pinned by: tests/test_oracle_quant.py (an element-by-element float32 loop
    restating this order; inputs on which a BLAS product, a pairwise order, a
    single sequential chain and a 64-wide chunking all give other values)."""
    M, K = x_f32.shape
    if K % PROJ_CHUNK:
        raise ValueError("the projection needs K % 128 == 0")
    r = U_f32.shape[1]
    x = x_f32.astype(F32)
    U = U_f32.astype(F32)
    total = None
    for t in range(K // PROJ_CHUNK):
        part = np.zeros((M, r), dtype=F32)
        for k in range(t * PROJ_CHUNK, (t + 1) * PROJ_CHUNK):
            part = part + x[:, k:k + 1] * U[k:k + 1, :]
        total = part if total is None else total + part
    return total


def residual(x_f32: np.ndarray, c_f32: np.ndarray, U_f32: np.ndarray) -> np.ndarray:
    """x_res[k] = x[k] - sum_j c_j U[k, j] (DiRotQ abstract: the components
    outside the PCA subspace are the ones quantized to 4 bit), with c the
    BF16-rounded coefficients: starting from x[k], the exact products c_j U[k, j]
    are subtracted one after another in order j = 0..r-1, each subtraction
    rounded to FP32.

    Pinned by: tests/test_oracle_quant.py (a float32 loop restating the order;
    inputs on which a BLAS product, the reverse order of j and unrounded
    coefficients give other values)."""
    xr = x_f32.astype(F32).copy()
    for j in range(U_f32.shape[1]):
        xr = xr - c_f32[:, j:j + 1] * U_f32[None, :, j]
    return xr


# ----------------------------------------------------------------------------
# Quantizers (FP32 contract)
# ----------------------------------------------------------------------------
def sum_squares(y: np.ndarray, block: int) -> np.ndarray:
    """Per-row sum of squares: squares rounded to FP32, a perfect pairwise tree
    in natural index order inside each block, block partials added in block
    order."""
    rows, K = y.shape
    s = (y * y).reshape(rows, K // block, block)
    while s.shape[2] > 1:
        s = s[:, :, 0::2] + s[:, :, 1::2]
    s = s[:, :, 0]
    acc = s[:, 0].copy()
    for j in range(1, s.shape[1]):
        acc = acc + s[:, j]
    return acc


def quant_int4(y: np.ndarray, group: int | None = None):
    """Symmetric uniform INT4 on the grid -7..7 (TR-DQ section 3.1, Eq. 1-2 with
    a zero point of 0 and the range set by the absolute maximum, per token, or
    per group of ``group`` rotated coordinates for weight rows):
    amax = max|y|; inv = 7/amax; q = clamp(round_half_even(y inv), -7, 7);
    scale = amax/7.  An all-zero row or group gets scale 0 and codes 0.
    Returns (q int8 rows x K, scale float32 rows x K/group)."""
    rows, K = y.shape
    g = K if group is None else group
    t = y.reshape(rows, K // g, g)
    amax = np.max(np.abs(t), axis=2)
    safe = np.where(amax > 0, amax, F32(1.0))
    inv = (F32(7.0) / safe).astype(F32)
    q = np.clip(np.rint(t * inv[:, :, None]), -7, 7)
    q = np.where(amax[:, :, None] > 0, q, 0).astype(np.int8)
    scale = np.where(amax > 0, (amax / F32(7.0)).astype(F32), F32(0.0)).astype(F32)
    return q.reshape(rows, K), scale


def quant_int4_asym(y: np.ndarray):
    """Asymmetric per-token INT4 (TR-DQ section 3.1, Eq. 1-3): the range
    [min, max] of the row is mapped onto 0..15.  Reading of the garbled signs:
    Eq. 3 gives z = round(min/s), and the code is round(x/s) - z, so that min
    lands on code 0 (adding z, as Eq. 1 prints it, would put min at 2z).  In
    FP32: inv = 15/(max - min); z = rne(min * inv); q = clamp(rne(y * inv) - z,
    0, 15); s = (max - min)/15; dequantized x = s (q + z).  The stored nibble is
    q - 8 (two's complement, -8..7) and the per-token zero point z + 8, so that
    x = s (nibble + zero point) and the GEMM reads signed nibbles like the
    symmetric format.  A constant row (max == min, after rotation only the zero
    row) gets s = 0, nibble -8, zero point 8.
    Returns (nibble int8, scale float32, zero_point float32).

    Pinned by: tests/test_oracle_trdq.py (hand-worked rows with ties, the
    clamp at both ends, the error bound s/2, min and max on codes 0 and 15)."""
    rows, K = y.shape
    y = np.asarray(y, dtype=F32)
    mn = np.min(y, axis=1)
    mx = np.max(y, axis=1)
    rng = (mx - mn).astype(F32)
    ok = rng > 0
    inv = np.where(ok, F32(15.0) / np.where(ok, rng, F32(1.0)), F32(0.0)).astype(F32)
    z = np.rint((mn * inv).astype(F32))
    q = np.clip(np.rint((y * inv[:, None]).astype(F32)) - z[:, None], 0, 15)
    q = np.where(ok[:, None], q, 0)
    z = np.where(ok, z, 0)
    scale = np.where(ok, (rng / F32(15.0)).astype(F32), F32(0.0)).astype(F32)
    return (q - 8).astype(np.int8), scale, (z + 8).astype(F32)


def quant_int8(y: np.ndarray):
    """Symmetric per-token INT8 for the W4A8 setting (TR-DQ section 3.1: b-bit
    uniform quantization with per-token scales for activations, Tables 1-5: W4A8
    and W8A8): amax = max|y|; inv = 127/amax; q = clamp(rne(y inv), -127, 127);
    scale = amax/127.  A zero row gets scale 0 and codes 0.
    Returns (q int8, scale float32).

    Pinned by: tests/test_oracle_trdq.py (hand cases with ties, the row
    maximum on 127, the error bound)."""
    y = np.asarray(y, dtype=F32)
    amax = np.max(np.abs(y), axis=1)
    ok = amax > 0
    inv = np.where(ok, F32(127.0) / np.where(ok, amax, F32(1.0)), F32(0.0)).astype(F32)
    q = np.clip(np.rint((y * inv[:, None]).astype(F32)), -127, 127).astype(np.int8)
    scale = np.where(ok, (amax / F32(127.0)).astype(F32), F32(0.0)).astype(F32)
    return q, scale


def quant_codebook(y: np.ndarray, block: int, boundaries_f32: np.ndarray):
    """Normalise each row to norm sqrt(K) and encode every coordinate as the
    number of codebook boundaries at or below it (OrbitQuant abstract:
    quantizing in a normalised, rotated basis with a Lloyd-Max codebook):
    nrm = sqrt(sum y^2); inv = sqrt(K)/nrm; u = y inv; code = #{i: u >= b_i};
    scale = nrm/sqrt(K).  An all-zero row gets scale 0 and the code of u = 0.
    Returns (codes uint8 rows x K, scale float32 rows)."""
    rows, K = y.shape
    nrm = np.sqrt(sum_squares(y, block)).astype(F32)
    sk = F32(math.sqrt(K))
    safe = np.where(nrm > 0, nrm, F32(1.0))
    inv = (sk / safe).astype(F32)
    u = (y * inv[:, None]).astype(F32)
    u = np.where(nrm[:, None] > 0, u, F32(0.0))
    codes = np.zeros(u.shape, dtype=np.uint8)
    for b in boundaries_f32.astype(F32):
        codes += (u >= b).astype(np.uint8)
    scale = np.where(nrm > 0, (nrm / sk).astype(F32), F32(0.0)).astype(F32)
    return codes, scale


def quant_nvfp4(y: np.ndarray):
    """NVFP4 (DiRotQ abstract: NVFP4 on Blackwell): a per-row FP32 scale that maps
    the row maximum to 6 * 448, then per 16 consecutive coordinates an unsigned
    E4M3 block scale and E2M1 elements:
    amax = max|y|; u = y (2688/amax); scale = amax/2688;
    sb = e4m3(max16|u| / 6); q = e2m1(u * (1/sb)), q = 0 where sb = 0.
    Returns (q nibble uint8 rows x K, sb uint8 rows x K/16, scale float32 rows)."""
    rows, K = y.shape
    amax = np.max(np.abs(y), axis=1)
    safe = np.where(amax > 0, amax, F32(1.0))
    inv_t = (F32(2688.0) / safe).astype(F32)
    u = (y * inv_t[:, None]).astype(F32)
    u = np.where(amax[:, None] > 0, u, F32(0.0))
    scale = np.where(amax > 0, (amax / F32(2688.0)).astype(F32), F32(0.0)).astype(F32)
    ug = u.reshape(rows, K // 16, 16)
    m16 = np.max(np.abs(ug), axis=2)
    sb = e4m3_encode((m16 / F32(6.0)).astype(F32))
    sbv = e4m3_decode(sb).astype(F32)
    rcp = (F32(1.0) / np.where(sbv > 0, sbv, F32(1.0))).astype(F32)
    q = e2m1_encode((ug * rcp[:, :, None]).astype(F32))
    q = np.where(sb[:, :, None] > 0, q, np.uint8(0)).astype(np.uint8)
    return q.reshape(rows, K), sb, scale


# ----------------------------------------------------------------------------
# Packing
# ----------------------------------------------------------------------------
def pack_nibbles(q: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte, element 2j in bits 0-3 and 2j+1 in bits 4-7."""
    q = (q.astype(np.int16) & 0xF).astype(np.uint8)
    return (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)


def sign_magnitude16(q: np.ndarray) -> np.ndarray:
    """The stored form of a 16-level codebook code c (0..15, the count of
    boundaries at or below u).  The codebook of the symmetric marginal is
    symmetric (centroid 15-c = -centroid c), so c is stored as its distance from
    the centre, m = c - 8 for c >= 8 and 7 - c below (bits 0-2), with bit 3 set
    for the lower half: centroid(c) = (bit 3 ? -1 : +1) * centroid(8 + m).  The
    pages fix no bit layout for packed codes; this one lets a consumer read one
    8-entry magnitude table."""
    c = np.asarray(q, dtype=np.int16)
    return np.where(c >= 8, c - 8, (7 - c) | 8).astype(np.uint8)


def code_from_sign_magnitude16(d: np.ndarray) -> np.ndarray:
    """Inverse of sign_magnitude16."""
    d = np.asarray(d, dtype=np.int16)
    return np.where(d >= 8, 7 - (d & 7), 8 + d).astype(np.uint8)


def unpack_nibbles(p: np.ndarray) -> np.ndarray:
    p = np.asarray(p, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def pack_crumbs(q: np.ndarray) -> np.ndarray:
    """2-bit codes, 16 per little-endian 32-bit word: element 16w+i (i < 8) in
    bits 4i..4i+1 of word w, element 16w+8+i in bits 4i+2..4i+3 (nibble i holds
    elements i and i+8).  Row length a multiple of 16."""
    q = (q.astype(np.uint8) & 3).reshape(q.shape[0], -1, 16)
    nib = q[:, :, :8] | (q[:, :, 8:] << 2)                    # nibble i of each word
    byt = nib[:, :, 0::2] | (nib[:, :, 1::2] << 4)             # byte j = nibbles 2j, 2j+1
    return byt.reshape(q.shape[0], -1).astype(np.uint8)


def unpack_crumbs(p: np.ndarray) -> np.ndarray:
    p = np.asarray(p, dtype=np.uint8).reshape(p.shape[0], -1, 4)
    nib = np.empty((p.shape[0], p.shape[1], 8), dtype=np.uint8)
    nib[:, :, 0::2] = p & 0xF
    nib[:, :, 1::2] = p >> 4
    out = np.concatenate([nib & 3, nib >> 2], axis=2)           # elements 0-7, then 8-15
    return out.reshape(p.shape[0], -1)


def int4_from_nibble(n: np.ndarray) -> np.ndarray:
    n = np.asarray(n, dtype=np.int16) & 0xF
    return np.where(n >= 8, n - 16, n).astype(np.int8)


# ----------------------------------------------------------------------------
# The hot path, end to end
# ----------------------------------------------------------------------------
def rotate_quantize(x_bf16_f32: np.ndarray, fmt: int, block: int, sign, perm,
                    boundaries_f32=None, U_f32=None, weight_rows: bool = False,
                    group: int = 128, zz_perm=None):
    """Rotate, normalise, quantize and pack rows (activation rows, or weight rows
    for W' = W R^T when ``weight_rows``).

    With ``U_f32`` (K x r BF16 values as FP32): activation rows first take
    c = bf16(x U) and quantize the residual x - c U^T; weight rows take
    L = bf16(W U) and quantize the full row (y = x_res W^T + c (W U)^T, DiRotQ
    abstract).

    With ``zz_perm``: the TR-DQ double rotation R2 P R1 (``rotate_double``;
    ``perm`` is then not used).  ``fmt`` INT4A: asymmetric per-token INT4
    (``quant_int4_asym``; activations only).

    Returns a dict with 'codes' (packed uint8), 'q' (unpacked codes), 'scale',
    'block_scale' (NVFP4, logical rows x K/16), 'zero_point' (INT4A) and 'coef'
    (BF16 bits of c or L)."""
    x = np.asarray(x_bf16_f32, dtype=F32)
    out = {"coef": None, "block_scale": None, "zero_point": None}
    if U_f32 is not None:
        cf = project_coefficients(x, U_f32)
        cb = _bf16_bits(cf)
        out["coef"] = cb
        if not weight_rows:
            x = residual(x, _bf16_f32(cb), U_f32)
    y = rotate(x, sign, perm, block) if zz_perm is None else rotate_double(x, sign, zz_perm, block)
    if fmt == INT8:
        # per token for activations; for weight rows one scale per output
        # channel (TR-DQ section 3.1, after Eq. 3: per-token activations,
        # per-channel weights) -- the same per-row quantizer
        q, s = quant_int8(y)
        out["q"], out["codes"], out["scale"] = q, q.view(np.uint8).copy(), s
    elif fmt == INT4A:
        if weight_rows:
            raise ValueError("asymmetric INT4 is an activation format")
        q, s, zp = quant_int4_asym(y)
        out["q"], out["codes"], out["scale"], out["zero_point"] = q, pack_nibbles(q), s, zp
    elif fmt == INT4:
        q, s = quant_int4(y, group if weight_rows else None)
        out["q"], out["codes"] = q, pack_nibbles(q)
        # weight-row group scales are stored group-major, [K/group][N]
        out["scale"] = np.ascontiguousarray(s.T) if weight_rows else s[:, 0]
    elif fmt in (LM16, LM4):
        q, s = quant_codebook(y, block, boundaries_f32)
        out["q"], out["scale"] = q, s
        out["codes"] = pack_crumbs(q) if fmt == LM4 else pack_nibbles(sign_magnitude16(q))
    elif fmt == NVFP4:
        q, sb, s = quant_nvfp4(y)
        out["q"], out["codes"], out["block_scale"], out["scale"] = q, pack_nibbles(q), sb, s
    else:
        raise ValueError(fmt)
    return out


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(a, dtype=F32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _bf16_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(F32)


def dequant_values(q: np.ndarray, fmt: int, block_scale=None, centroids_e4m3=None, zero_point=None):
    """FP64 operand values the GEMM multiplies, before the per-row/per-group
    scales: INT4 integers (asymmetric: nibble + per-row zero point), e4m3
    centroid values, or e2m1 x e4m3 block scale."""
    if fmt == INT8:
        return np.asarray(q).view(np.int8).astype(np.float64)
    if fmt == INT4A:
        n = int4_from_nibble(q) if q.dtype == np.uint8 else q
        return n.astype(np.float64) + np.asarray(zero_point, np.float64)[:, None]
    if fmt == INT4:
        return int4_from_nibble(q).astype(np.float64) if q.dtype == np.uint8 else q.astype(np.float64)
    if fmt in (LM16, LM4):
        return e4m3_decode(centroids_e4m3)[q.astype(np.int64)]
    if fmt == NVFP4:
        v = e2m1_decode(q)
        sb = e4m3_decode(block_scale)
        return v * np.repeat(sb, 16, axis=1)
    raise ValueError(fmt)


def reference_gemm(a_fmt: int, w_fmt: int, qa, sa, qw, sw, a_bs=None, w_bs=None,
                   a_cent=None, w_cent=None, c_bf16=None, L_bf16=None, group: int = 128, a_zp=None):
    """FP64 reference output Y (M x N) over the dequantized values:

    * INT4: Y = s_a[m] sum_g s_w[g, n] (sum_{k in g} qa qw), integer partials exact
      (asymmetric activations: qa = nibble + zero point, still integers);
    * codebook / NVFP4: Y = s_a[m] s_w[n] sum_k a_k w_k with dequantized values;
    * plus sum_j c[m, j] L[n, j] when the low-rank branch is present.

    ``qa``/``qw`` are unpacked codes (M x K, N x K); INT4 weight scales are
    [K/group, N] (group-major); other weight scales are per row [N]."""
    A = dequant_values(qa, a_fmt, a_bs, a_cent, a_zp)
    B = dequant_values(qw, w_fmt, w_bs, w_cent)
    if w_fmt == INT4:
        K = A.shape[1]
        Y = np.zeros((A.shape[0], B.shape[0]))
        for g in range(K // group):
            P = A[:, g * group:(g + 1) * group] @ B[:, g * group:(g + 1) * group].T
            Y += P * np.asarray(sw, dtype=np.float64)[g][None, :]
        Y *= np.asarray(sa, dtype=np.float64)[:, None]
    else:
        Y = (A @ B.T) * np.asarray(sa, np.float64)[:, None] * np.asarray(sw, np.float64)[None, :]
    if c_bf16 is not None:
        Y += _bf16_f32(c_bf16).astype(np.float64) @ _bf16_f32(L_bf16).astype(np.float64).T
    return Y


def int4_e4m3_lut() -> np.ndarray:
    """E4M3 bytes of the INT4 nibble values 0..7, -8..-1 (nibble order), for
    operands the FP8 GEMM multiplies; every integer in -7..7 is exact in E4M3."""
    vals = int4_from_nibble(np.arange(16, dtype=np.uint8)).astype(np.float32)
    return e4m3_encode(vals)
