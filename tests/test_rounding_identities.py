"""Arithmetic facts the CUDA rounding code relies on, checked on the CPU.

The step kernel rounds in forms that differ from the oracle's plain
statement but must give the same integers:

- Bounded Directional Rounding needs no clamp to [-qmax, qmax]: a step up
  from n = qmax needs y = x * inv > qmax, which only x = A (the column's
  absmax) can reach, and then also p < deq < A with p = RN(qmax * RN(A/qmax));
  no float lies strictly between p and A whenever A * inv > qmax. Checked
  exhaustively over every binary32 significand of A for qmax 7 and 127 (the
  quantities scale exactly with A's exponent over the range the step uses).
- Stochastic rounding compares its 23-bit draw u with the rounded fraction
  fr as 1 + u < RU(1 + fr), RU = rounding up to binary32.

Sources: "Preserving Updates in Low-Bit Recurrent State Quantization"
(abstract: Bounded Directional Rounding); "Quantizing Recurrent Language
Models Is Easier Than You Think" (abstract: stochastic rounding).
"""
import numpy as np

F32, F64 = np.float32, np.float64


def _all_significands():
    bits = np.arange(1 << 23, dtype=np.uint32) | np.uint32(0x3F800000)
    return bits.view(F32)                                  # every float in [1, 2)


def test_only_the_absmax_exceeds_qmax():
    A = _all_significands()
    below = np.nextafter(A, F32(0))
    for q in (7, 127):
        inv = F32(q) / A                                   # RN(qmax / A)
        assert not np.any(below.astype(F64) * inv.astype(F64) > q)
        assert np.all(A.astype(F64) * inv.astype(F64) < q + 0.5)   # rint(y) stays in range


def test_bdr_step_past_qmax_is_impossible():
    A = _all_significands()
    for q in (7, 127):
        s = A / F32(q)                                     # RN(A / qmax), the new scale
        inv = F32(q) / A
        p = F32(q) * s                                     # RN(qmax * s')
        over = A.astype(F64) * inv.astype(F64) > q         # y = A * inv > qmax
        assert over.sum() > 1 << 20                        # the case does arise often
        room = np.nextafter(p, F32(np.inf)) < A            # a float deq with p < deq < A
        assert not np.any(over & room)


def _ru_one_plus(fr):
    """RU(1 + fr) for binary32 fr (|fr| < 2): 1 + fr is exact in float64 unless
    0 < |fr| < 2^-29, where it lies strictly between 1 and its binary32
    neighbour on the side of fr's sign."""
    v = 1.0 + fr.astype(F64)
    r = v.astype(F32)
    lo = r.astype(F64) < v
    r[lo] = np.nextafter(r[lo], F32(np.inf))
    tiny = (np.abs(fr) < 2.0 ** -29) & (fr != 0)
    r[tiny & (fr > 0)] = F32(1.0 + 2.0 ** -23)
    r[tiny & (fr < 0)] = F32(1.0)
    return r


def test_sr_compare_through_round_up():
    rng = np.random.default_rng(7)
    n = 200_000
    # fractions: random, tiny, near 1, on and off the 2^-23 grid, and outside [0, 1]
    fr = np.concatenate([
        rng.random(n).astype(F32),
        (rng.random(n) * 2.0 ** -rng.integers(10, 60, n)).astype(F32),
        (1.0 - rng.random(n) * 2.0 ** -rng.integers(18, 30, n)).astype(F32),
        (rng.integers(0, 1 << 23, n) * 2.0 ** -23).astype(F32),
        F32([0.0, 1.0, 1.0 + 2.0 ** -23, 1.5, -2.0 ** -30, -2.0 ** -17, -0.0]),
    ])
    g = _ru_one_plus(fr)                                   # RU(1 + fr)
    grid = np.floor(fr.astype(F64) * 2.0 ** 23)
    for off in (-2, -1, 0, 1, 2):
        m = np.clip(grid + off, 0, (1 << 23) - 1)
        u = (m * 2.0 ** -23).astype(F32)                   # the draw, exact
        u1 = (1.0 + m * 2.0 ** -23).astype(F32)            # 1 + u, exact
        np.testing.assert_array_equal(u < fr, u1 < g)
