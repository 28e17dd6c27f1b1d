"""Pins that tell the oracle's readings apart from their plausible alternatives.

The pages fix the NVFP4 two-level scaling and ask for the layer norm to be
fused into the preprocessing (SharQ abstract), but no page gives the order of
the fp32 operations.  The oracle takes one reading per point; these tests pin
it with inputs on which the alternatives give a DIFFERENT result, so that the
reading cannot drift without a test failing.  Expected values come from exact
rational arithmetic with an IEEE binary32 round-to-nearest-even written here
from the format's definition (no fp32 library call), or are derived by hand in
the comments.

Readings pinned:
* NVFP4 block scale s = (amax / 6) * g_enc, each step rounded once (amax / 6
  is the block's decode scale: the largest E2M1 magnitude lands on the block
  amax; times g_enc it is stated in units of the tensor decode scale).  The
  folded alternative amax * (g_enc / 6) gives another E4M3 code on the cases
  built below.
* RMSNorm sum of squares: 16-element chunk sums by sequential fused
  multiply-add in ascending K order, then a pairwise tree over ADJACENT chunk
  sums zero padded to a power of two.  A halving tree (a[i] + a[i + h]), a plain
  sequential sum, separate multiply-then-add inside a chunk and descending
  order each give another rstd on the rows below.
"""
import math
from fractions import Fraction as Fr

import numpy as np

import oracle


# --------------------------------------------------------------- exact fp32
def rn_f32(x: Fr) -> Fr:
    """IEEE binary32 round to nearest, ties to even, of an exact rational (finite result)."""
    if x == 0:
        return Fr(0)
    sign = 1 if x > 0 else -1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fr(2) ** e > a:
        e -= 1
    while Fr(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)  # subnormals share the smallest normal exponent's ulp
    ulp = Fr(2) ** (e - 23)
    m = a / ulp
    q = m.numerator // m.denominator
    rem = m - q
    if rem > Fr(1, 2) or (rem == Fr(1, 2) and q % 2 == 1):
        q += 1
    return sign * q * ulp


def next_f32(x: Fr, up: bool) -> Fr:
    """The neighbouring binary32 value of a positive binary32 value x."""
    v = np.float32(float(x))
    return Fr(float(np.nextafter(v, np.float32(np.inf if up else 0.0))))


def rn_sqrt_f32(m: Fr) -> Fr:
    """Correctly rounded binary32 square root of a non-negative binary32 value,
    decided exactly: y is the result iff sqrt(m) lies between y's two midpoints."""
    y = Fr(float(np.float32(math.sqrt(float(m)))))
    for _ in range(4):
        lo = (y + next_f32(y, False)) / 2
        hi = (y + next_f32(y, True)) / 2
        if lo * lo <= m <= hi * hi:
            return y
        y = next_f32(y, m > hi * hi)
    raise AssertionError("sqrt search did not converge")


E4M3_VALUES = [Fr(c & 7, 1) * Fr(2) ** -9 if (c >> 3) == 0 else (1 + Fr(c & 7, 8)) * Fr(2) ** ((c >> 3) - 7)
               for c in range(127)]  # codes 0..126; 126 = 448


def e4m3_nearest(s: Fr) -> int:
    """E4M3 code of s >= 0: nearest finite value, ties to the even code, above 448 -> 448."""
    best, bd = 0, None
    for c, v in enumerate(E4M3_VALUES):
        d = abs(v - s)
        if bd is None or d < bd or (d == bd and c % 2 == 0):
            best, bd = c, d
    return best


# ----------------------------------------------------- NVFP4 block scale
def _scale_code(amax: Fr, g_enc: Fr, folded: bool) -> int:
    if folded:
        s = rn_f32(amax * rn_f32(g_enc / 6))
    else:
        s = rn_f32(rn_f32(amax / 6) * g_enc)
    return e4m3_nearest(s)


def _order_cases():
    """(amax, g_enc, A) near E4M3 rounding boundaries on which the two orders
    disagree (g_enc = rn(2688 / A), A a binary32 tensor amax): amax is walked
    ulp by ulp around 6 * midpoint / g_enc."""
    rng = np.random.default_rng(5)
    mids = [(E4M3_VALUES[c] + E4M3_VALUES[c + 1]) / 2 for c in range(8, 126)]
    cases = []
    for i in range(60):
        big_a = Fr(float(np.float32(rng.uniform(0.5, 400.0))))
        g_enc = rn_f32(Fr(2688) / big_a)
        mid = mids[int(rng.integers(len(mids)))]
        a = rn_f32(6 * mid / g_enc)
        for _ in range(12):
            a = next_f32(a, False)
        for _ in range(24):
            if _scale_code(a, g_enc, False) != _scale_code(a, g_enc, True):
                cases.append((a, g_enc, big_a))
            a = next_f32(a, True)
    return cases


def test_nvfp4_block_scale_divides_amax_by_6_before_g_enc():
    cases = _order_cases()
    assert len(cases) >= 20, f"only {len(cases)} order-discriminating cases found"
    for amax, g_enc, _ in cases:
        exp = _scale_code(amax, g_enc, folded=False)
        # the block's values: its amax and a few smaller ones (the amax alone sets the scale)
        v = np.array([float(amax), -float(amax) / 3, 0.0, float(amax) / 7] * 4, np.float32)
        assert Fr(float(np.abs(v).max())) == amax
        code, _ = oracle.quant_block(v, "nvfp4", float(g_enc))
        assert code == exp, (float(amax), float(g_enc), code, exp)
        assert code != _scale_code(amax, g_enc, folded=True)


def test_nvfp4_block_scale_through_prepare():
    """The same order inside the whole preprocessing (4:8 pair, no norm, tensor
    amax A given by the caller).  Row: [A, 0, A, 0, amax, 0, ...]: pairs 0 and 1
    score A and are kept, pair 2 scores amax < A (amax = 6 * mid / g_enc with an
    E4M3 midpoint mid < 448) and is dropped, so residual block 0 holds amax
    itself plus the kept values' rounding errors (about A * 2^-23, far below
    amax): its scale code is the pinned one."""
    for amax, g_enc, big_a in _order_cases()[:8]:
        k = 256
        x = np.zeros((1, k), np.float32)
        x[0, [0, 2]] = float(big_a)
        x[0, 4] = float(amax)
        prep = oracle.prepare(x, "nvfp4", "4:8pair", act_amax=float(big_a))
        assert Fr(float(prep["tensor"][1])) == g_enc
        assert oracle.mask(x, "4:8pair")[0, :8].tolist() == [1, 1, 1, 1, 0, 0, 0, 0]
        exp = _scale_code(amax, g_enc, folded=False)
        assert prep["res_scales"][0, 0] == exp
        assert exp != _scale_code(amax, g_enc, folded=True)


# ------------------------------------------------------------- RMSNorm order
def _exact_rstd(total: Fr, k: int, eps: Fr = Fr(0)) -> Fr:
    mean = rn_f32(total / k)
    return rn_f32(1 / rn_sqrt_f32(rn_f32(mean + eps)))


def test_rmsnorm_tree_over_adjacent_chunk_sums():
    """k = 128: chunk sums [2^24, 3, 1, 1, 2, 3, 3, 1] (all exact: one element
    4096, then runs of ones).  With fp32 ties to even (ulp 2 at 2^24):
      adjacent pairs: (2^24+3 -> 2^24+4), 2, 5, 4; then 2^24+6, 9; then 2^24+15 -> 2^24+16
      halving tree:   2^24+2, 6, 4, 2; then 2^24+6, 8; then 2^24+14
      sequential:     2^24+4, +4, +4, +6, +8, +12, +12 -> 2^24+12
      chunks of 32:   2^24 (each +1 absorbed by a tie to even), 2, 5, 4; then 2^24+2, 9 -> 2^24+12."""
    x = np.zeros(128, np.float32)
    x[0] = 4096.0
    for j, n_ones in enumerate([3, 1, 1, 2, 3, 3, 1], start=1):
        x[16 * j: 16 * j + n_ones] = 1.0
    r = Fr(oracle.rms_rstd(x, 0.0))
    adjacent, halving, sequential = (_exact_rstd(Fr(2 ** 24 + d), 128) for d in (16, 14, 12))
    assert len({adjacent, halving, sequential}) == 3  # the row tells the orders apart
    assert r == adjacent


# a chunk of 16 fp32 values whose sum of squares depends on the order of the
# operations (found by a seeded search); ascending fused multiply-adds
_CHUNK = [0.5578336119651794, 1.3086563348770142, 0.4195121228694916, 0.9280189871788025,
          0.9386432766914368, 0.6871419548988342, 1.1839369535446167, 0.9399011135101318,
          0.8689395189285278, 1.1559525728225708, 0.8570262789726257, 1.4166940450668335,
          1.1054365634918213, 0.8577001094818115, 0.41672050952911377, 0.6076740622520447]


def _chunk_sum(vals, fused: bool) -> Fr:
    acc = Fr(0)
    for v in vals:
        sq = Fr(v) * Fr(v)
        acc = rn_f32(sq + acc) if fused else rn_f32(rn_f32(sq) + acc)
    return acc


def test_rmsnorm_chunk_sum_is_ascending_fused_multiply_add():
    x = np.array(_CHUNK, np.float32)
    assert all(Fr(float(v)) == Fr(c) for v, c in zip(x, _CHUNK))  # exact binary32 inputs
    r = Fr(oracle.rms_rstd(x, 0.0))
    fma_up = _exact_rstd(_chunk_sum(_CHUNK, True), 16)
    mul_add = _exact_rstd(_chunk_sum(_CHUNK, False), 16)
    fma_down = _exact_rstd(_chunk_sum(_CHUNK[::-1], True), 16)
    assert fma_up != mul_add and fma_up != fma_down
    assert r == fma_up


def test_rmsnorm_eps_added_to_the_rounded_mean():
    """x = [3, 0, ..., 0] (k = 16): sum of squares 9, mean 9/16 (exact); eps is
    added to the rounded mean, not to the sum before the division."""
    x = np.zeros(16, np.float32)
    x[0] = 3.0
    eps = Fr(float(np.float32(1e-6)))
    r = Fr(oracle.rms_rstd(x, float(eps)))
    after = _exact_rstd(Fr(9), 16, eps)
    before = rn_f32(1 / rn_sqrt_f32(rn_f32(rn_f32(9 + eps) / 16)))
    assert after != before
    assert r == after
