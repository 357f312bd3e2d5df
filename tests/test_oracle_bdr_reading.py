"""Pins of the oracle's study of the other Bounded Directional Rounding
reading (update = the additive term k_i w_j; "Preserving Updates in Low-Bit
Recurrent State Quantization", abstract). The library reads the update as
x - deq; these tests fix what the study function computes."""
import numpy as np

import oracle
from tests.test_oracle_pins import _one_step_parts

F32 = np.float32


def _case(seed, n=6, d_k=64, d_v=64, group=32, gate_one=False, qmax=127):
    rng = np.random.default_rng(seed)
    S0 = (rng.standard_normal((n, d_k, d_v)) * 0.02).astype(F32)
    pm = np.full(1, 8 if qmax == 127 else 4, np.uint8)
    th = np.zeros(n, np.int32)
    codes, scales = oracle.import_fp32(S0, pm, th, group=group)
    q = rng.standard_normal((n, d_k)).astype(F32)
    k = rng.standard_normal((n, d_k)).astype(F32)
    v = rng.standard_normal((n, d_v)).astype(F32)
    g = np.ones((n, d_k), F32) if gate_one else \
        np.exp(-np.log1p(np.exp(rng.standard_normal((n, d_k)) - 3.0))).astype(F32)
    return codes, scales, q, k, v, g, pm, th


def test_equals_the_library_reading_where_the_two_updates_agree_in_sign():
    # gates 1: x - deq = RN(deq + k_i v_j) - deq has the sign of k_i v_j
    # whenever k_i v_j moves x at all; then both readings are one rule
    for qmax in (127, 7):
        codes, scales, q, k, v, g, pm, th = _case(3, gate_one=True, qmax=qmax)
        deq = codes.astype(F32) * np.repeat(scales, 32, axis=1)
        kw = k[:, :, None] * v[:, None, :]
        x = deq + kw                                           # fma(1, deq, kw) = RN(deq + kw)
        assert np.array_equal(np.sign(x - deq), np.sign(kw))
        c1, s1 = codes.copy(), scales.copy()
        c2, s2 = codes.copy(), scales.copy()
        o1 = oracle.bdr_additive_step(c1, s1, q, k, v, g, group=32, qmax=qmax)
        tb = np.zeros(len(th), np.int32)
        o2 = oracle.step(c2, s2, q, k, v, g, None, pm, tb, th, group=32, update_kind=0,
                         gate_kind=1, mode=oracle.ROUND_BDR)
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(c1, c2)
        np.testing.assert_array_equal(s1.view(np.uint32), s2.view(np.uint32))


def test_never_moves_against_the_additive_term():
    # The rule with delta := k_i w_j: the stored value never ends on the
    # other side of deq than k_i w_j unless the code took the bounded step
    # (ceil or floor of y); where round-to-nearest does not reverse against
    # k_i w_j, the result is round-to-nearest.
    group = 8
    reversals = 0
    for bits in (8, 4):
        qmax = 127 if bits == 8 else 7
        rng = np.random.default_rng(91 + bits)
        for trial in range(10):
            codes, scales, pm, q, k, v, g, deq, x = _one_step_parts(rng, bits, oracle.ROUND_BDR,
                                                                    n=2, group=group)
            c_rtn, s_rtn = codes.copy(), scales.copy()
            oracle.step(c_rtn, s_rtn, q, k, v, g, None, pm, [0, 1], [0, 0], group=group,
                        update_kind=oracle.UPDATE_GATED, gate_kind=oracle.GATE_PER_KEY,
                        mode=oracle.ROUND_RTN)
            c, s = codes.copy(), scales.copy()
            oracle.bdr_additive_step(c, s, q, k, v, g, group=group, qmax=qmax)
            np.testing.assert_array_equal(s, s_rtn)
            sc = np.repeat(s, group, axis=1)
            A = np.repeat(np.abs(x).reshape(2, -1, group, x.shape[2]).max(axis=2), group, axis=1)
            inv = np.where(sc > 0, F32(qmax) / np.where(sc > 0, A, 1), 0).astype(F32)
            y = x.astype(np.float64) * inv.astype(np.float64)           # exact product
            kw = (k[:, :, None] * v[:, None, :]).astype(F32)
            moved = ((c.astype(F32) * sc).astype(F32) - deq).astype(F32)
            up = c == np.clip(np.ceil(y), -qmax, qmax)
            dn = c == np.clip(np.floor(y), -qmax, qmax)
            ok = (kw == 0) | (moved * np.sign(kw) >= 0) | ((kw > 0) & up) | ((kw < 0) & dn)
            assert ok.all()
            rtn_moved = ((c_rtn.astype(F32) * sc).astype(F32) - deq).astype(F32)
            no_rev = ~(((kw > 0) & (rtn_moved < 0)) | ((kw < 0) & (rtn_moved > 0)))
            np.testing.assert_array_equal(c[no_rev], c_rtn[no_rev])
            reversals += int((~no_rev).sum())
    assert reversals > 0
