"""Pins of the oracle's binary64 -> bf16 rounding (the FP32-accumulate ->
BF16 output of the grouped GEMM, paper Sec. 3.4 / App. D.1, applied to the
oracle's exact sums): round once to the nearest bf16 number, an exact tie to
the even fraction, overflow to infinity past the last midpoint.

The second oracle here is a brute-force search in exact rational arithmetic
(fractions.Fraction) over the bf16 bit patterns next to the value; it shares
no formula with the C code (which scales by the bf16 spacing)."""
import math
import struct
from fractions import Fraction

import numpy as np

import oracle as O
import synthetic as S


def _bf16_value(bits: int) -> Fraction:
    """Exact value of a finite bf16 bit pattern."""
    f = struct.unpack("<f", struct.pack("<I", (bits & 0xFFFF) << 16))[0]
    return Fraction(f)


def _nearest_bf16_bruteforce(v: float) -> int:
    """Nearest finite-or-infinite bf16 to v by exact comparison against the
    bf16 patterns around v's binary32 neighbourhood; ties to the even pattern."""
    if v == 0.0:
        return 0x8000 if math.copysign(1.0, v) < 0 else 0
    sign = 0x8000 if v < 0 else 0
    a = Fraction(abs(v))
    # candidate magnitudes: every positive bf16 pattern whose value brackets a;
    # find the pattern t with value(t) <= a < value(t+1) by bisection over
    # the ordered finite patterns 0x0000 .. 0x7F7F
    lo, hi = 0, 0x7F7F
    if a >= _bf16_value(hi):
        lo = hi
    else:
        while hi - lo > 1:
            mid = (lo + hi) // 2
            if _bf16_value(mid) <= a:
                lo = mid
            else:
                hi = mid
    cands = [lo, lo + 1]
    vals = []
    for c in cands:
        if c == 0x7F80:                      # the next step past the largest finite number
            vals.append(Fraction(2) ** 128)  # infinity's place on the grid
        else:
            vals.append(_bf16_value(c))
    d0, d1 = a - vals[0], vals[1] - a
    if d0 < d1:
        best = cands[0]
    elif d1 < d0:
        best = cands[1]
    else:
        best = cands[0] if cands[0] % 2 == 0 else cands[1]
    return sign | best


def _check(v):
    got = O.bf16_round(v)
    want = _nearest_bf16_bruteforce(v)
    assert got == want, (v.hex(), hex(got), hex(want))


def test_exact_bf16_values_are_fixed_points():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 0x7F80, size=400)
    for b in bits:
        v = float(_bf16_value(int(b)))
        assert O.bf16_round(v) == int(b)
        assert O.bf16_round(-v) == (int(b) | 0x8000) or v == 0.0


def test_midpoints_tie_to_even_and_near_midpoints_round_away_from_tie():
    """At an exact midpoint the even pattern wins; 2^-40 (relative) to either
    side decides by distance.  A binary32 intermediate would collapse the
    near-midpoint values onto the midpoint and round them to even: these
    cases are the ones double rounding gets wrong."""
    rng = np.random.default_rng(2)
    for b in list(rng.integers(0x0080, 0x7F7F, size=300)) + [0x3F80, 0x3F81, 0x0080, 0x7F7E]:
        b = int(b)
        a, c = _bf16_value(b), _bf16_value(b + 1)
        mid = (a + c) / 2
        m = float(mid)
        assert Fraction(m) == mid                              # exact in binary64
        even = b if b % 2 == 0 else b + 1
        assert O.bf16_round(m) == even
        up = m * (1.0 + 2.0 ** -40)
        dn = m * (1.0 - 2.0 ** -40)
        assert O.bf16_round(up) == b + 1, (hex(b), up.hex())
        assert O.bf16_round(dn) == b, (hex(b), dn.hex())
        assert O.bf16_round(-up) == (b + 1) | 0x8000
        _check(up)
        _check(dn)


def test_subnormal_and_overflow_edges():
    tiny = 2.0 ** -133                                         # smallest bf16 subnormal
    assert O.bf16_round(tiny) == 0x0001
    assert O.bf16_round(tiny / 2) == 0x0000                    # tie between 0 and the first subnormal: even
    assert O.bf16_round(tiny / 2 * (1 + 2.0 ** -40)) == 0x0001
    assert O.bf16_round(tiny * 1.5) == 0x0002                  # tie 1 | 2: even
    assert O.bf16_round(tiny * 2.5) == 0x0002                  # tie 2 | 3: even
    assert O.bf16_round(2.0 ** -126) == 0x0080                 # smallest normal
    assert O.bf16_round(2.0 ** -126 - tiny / 4) == 0x0080      # rounds up into the normals
    assert O.bf16_round(1e-300) == 0x0000
    assert O.bf16_round(-1e-300) == 0x8000
    big = float(_bf16_value(0x7F7F))                           # (2 - 2^-7) 2^127
    assert O.bf16_round(big) == 0x7F7F
    last_mid = 2.0 ** 127 * (2.0 - 2.0 ** -8)
    assert O.bf16_round(last_mid) == 0x7F80                    # tie with infinity: the even side
    assert O.bf16_round(last_mid * (1 - 2.0 ** -40)) == 0x7F7F
    assert O.bf16_round(1e300) == 0x7F80
    assert O.bf16_round(-1e300) == 0xFF80
    assert O.bf16_round(0.0) == 0x0000
    assert O.bf16_round(-0.0) == 0x8000


def test_random_sweep_against_bruteforce():
    rng = np.random.default_rng(3)
    vals = rng.normal(0, 1, 300) * 2.0 ** rng.integers(-140, 130, 300)
    for v in vals:
        _check(float(v))


def test_gemm_output_is_the_once_rounded_exact_sum():
    """The oracle's grouped GEMM rounds its exact binary64 result once."""
    E, M, K, T, k, seed = 3, 32, 256, 20, 2, 31
    w = np.stack([S.expert_weights_bf16_np(seed, 0, e, M, K) for e in range(E)])
    pk = O.pack_weights(w)
    x = S.activations_bf16_np(seed, T, K)
    rt = O.route(S.uniform_logits_np(seed, T, E), k)
    ga = np.full(E, O.act_global_scale(x), np.float32)
    a_c, a_s = O.permute_quantize(x, rt, ga)
    y, _, exact = O.grouped_gemm(pk, a_c, a_s, rt.offsets, ga, want_exact=True)
    flat_y, flat_x = y.ravel(), exact.ravel()
    for i in range(0, flat_y.size, 7):
        assert int(flat_y[i]) == _nearest_bf16_bruteforce(float(flat_x[i]))
