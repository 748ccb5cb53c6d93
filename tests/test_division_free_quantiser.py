"""The NVFP4 quantiser's unit-global form divides by no block scale: for the
quotient x / d (x a BF16 value, d = value(sf) an E4M3 scale) it takes
y = RN(1/d), q0 = RN(x * y), r = RN(x - q0 * d) (an FMA; exact) and
q = RN(q0 + r * y) -- Markstein's correction (P. Markstein, IBM J. Res. Dev.
34(1), 1990).  The codes it produces are those of the IEEE division only if q
equals RN(x / d) wherever the E2M1 code can tell them apart.  This checks that,
in exact arithmetic emulated on float64, for every finite BF16 x a block with
scale d can hold and every positive finite E4M3 d: any difference lies below
2^-100 in magnitude with the same sign (a zero code either way)."""
import numpy as np

F32 = np.float32


def _e4m3_positive_values():
    out = []
    for b in range(1, 0x7F):
        e, m = (b >> 3) & 15, b & 7
        out.append((m / 8) * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return out


def _rn32_of_sum(a64, b64):
    """RN to FP32 of the exact a + b (a, b float64 holding exact values), via
    TwoSum and a midpoint fix-up for the double rounding."""
    s = a64 + b64
    bb = s - a64
    err = (a64 - (s - bb)) + (b64 - bb)
    c = s.astype(F32)
    cd = c.astype(np.float64)
    toward = np.where(s > cd, F32(np.inf), F32(-np.inf))
    nxt = np.nextafter(c, toward).astype(np.float64)
    at_mid = np.abs(s - cd) == np.abs(nxt - cd) / 2
    move = at_mid & (err != 0) & (np.sign(err) == np.sign(nxt - cd))
    return np.where(move, nxt.astype(F32), c)


def test_markstein_quotient_gives_the_division_codes():
    bits = np.arange(1 << 16, dtype=np.uint32)
    x_all = (bits << 16).view(F32)
    x_all = x_all[np.isfinite(x_all)]
    with np.errstate(over="ignore", invalid="ignore", under="ignore"):
        for d64 in _e4m3_positive_values():
            d = F32(d64)
            # a block with scale d holds |x| <= amax < 6 * (d + half an E4M3 step) (< 9 d);
            # the saturated scale 448 holds any x
            x = x_all if d64 == 448.0 else x_all[np.abs(x_all) <= 10 * d64]
            y = F32(1) / d
            q0 = (x * y).astype(F32)
            r = (x.astype(np.float64) - q0.astype(np.float64) * d64).astype(F32)  # exact residual, one rounding
            q = _rn32_of_sum(q0.astype(np.float64), r.astype(np.float64) * np.float64(y))
            ref = (x / d).astype(F32)
            diff = q != ref
            assert not np.any(np.abs(ref[diff]) >= 2.0 ** -100), d64
            assert not np.any(np.abs(q[diff]) >= 2.0 ** -100), d64
            assert np.array_equal(np.signbit(q[diff]), np.signbit(ref[diff])), d64
            # the quotients a code can see (|q| >= 2^-100) are the division's exactly
            big = np.abs(ref) >= 2.0 ** -100
            assert np.array_equal(q[big], ref[big]), d64
