"""Pins of the oracle's multi-token (chunked) update and of its bfloat16 rounding.

Chunked update: T tokens applied to the fp32 state one after the other, one
requantization at the end. It is pinned to the unquantized recurrence (itself
pinned to its closed form and to the fp64 matrix recurrence in
test_oracle_pins.py) composed with round-to-nearest import, to fp64 brute force
for the delta rule, and to the invariants of SR and BDR taken relative to the
state at the chunk's start.

bfloat16: pinned to hand-worked patterns (ties, overflow, signed zeros, NaN),
to torch's float32 -> bfloat16 conversion (a library routine) and to the
nearest-value property by brute force.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.test_oracle_pins import _quant_state

F32 = np.float32


def _chunk_inputs(rng, T, n, d_k, d_v, per_key=True, delta=False):
    q = rng.standard_normal((T, n, d_k)).astype(F32)
    k = rng.standard_normal((T, n, d_k)).astype(F32)
    k /= np.linalg.norm(k, axis=2, keepdims=True)
    v = rng.standard_normal((T, n, d_v)).astype(F32)
    if per_key:
        g = np.exp(-np.log1p(np.exp(rng.normal(-2.0, 1.0, (T, n, d_k))))).astype(F32)
    else:
        g = (1 / (1 + np.exp(-rng.normal(2.0, 1.0, (T, n))))).astype(F32)
    beta = (1 / (1 + np.exp(-rng.normal(0, 1, (T, n))))).astype(F32) if delta else None
    return q, k.astype(F32), v, g, beta


def _unquantized(deq, q, k, v, g, beta, upd, gate):
    """The fp32 recurrence token by token from the dequantized state."""
    S = deq.copy()
    outs = []
    for t in range(q.shape[0]):
        outs.append(oracle.fp32_step(S, q[t], k[t], v[t], g[t], None if beta is None else beta[t],
                                     update_kind=upd, gate_kind=gate))
    return S, np.stack(outs)


CASES = [(oracle.UPDATE_GATED, oracle.GATE_PER_KEY), (oracle.UPDATE_GATED, oracle.GATE_SCALAR),
         (oracle.UPDATE_DELTA, oracle.GATE_SCALAR)]


@pytest.mark.parametrize("upd,gate", CASES)
@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("T", [2, 5])
def test_chunk_rtn_is_recurrence_then_one_import(upd, gate, bits, T):
    rng = np.random.default_rng(1000 * T + 10 * bits + upd + gate)
    n, d_k, d_v, group = 3, 16, 8, 8
    _, codes, scales, pm = _quant_state(rng, n, d_k, d_v, group, bits)
    q, k, v, g, beta = _chunk_inputs(rng, T, n, d_k, d_v, per_key=gate == oracle.GATE_PER_KEY,
                                     delta=upd == oracle.UPDATE_DELTA)
    deq = oracle.dequant(codes, scales, group=group)
    S_T, o_ref = _unquantized(deq, q, k, v, g, beta, upd, gate)
    c_ref, s_ref = oracle.import_fp32(S_T, pm, np.zeros(n, np.int32), group=group)
    out = oracle.chunk_step(codes, scales, q, k, v, g, beta, pm, np.arange(n), np.zeros(n),
                            group=group, update_kind=upd, gate_kind=gate, mode=oracle.ROUND_RTN)
    np.testing.assert_array_equal(out, o_ref)
    np.testing.assert_array_equal(codes, c_ref)
    np.testing.assert_array_equal(scales, s_ref)


def test_chunk_delta_tracks_fp64_matrix_recurrence():
    """alpha_t (I - beta_t k_t k_t^T) S + beta_t k_t v_t^T over the chunk, in fp64."""
    rng = np.random.default_rng(31)
    T, n, d_k, d_v, group = 6, 1, 8, 8, 8
    _, codes, scales, pm = _quant_state(rng, n, d_k, d_v, group, 8)
    q, k, v, a, beta = _chunk_inputs(rng, T, n, d_k, d_v, per_key=False, delta=True)
    Sd = oracle.dequant(codes, scales, group=group)[0].astype(np.float64)
    out = oracle.chunk_step(codes, scales, q, k, v, a, beta, pm, [0], [0], group=group,
                            update_kind=oracle.UPDATE_DELTA, gate_kind=oracle.GATE_SCALAR,
                            mode=oracle.ROUND_RTN)
    for t in range(T):
        kk = k[t, 0].astype(np.float64)
        A = float(a[t, 0]) * (np.eye(d_k) - float(beta[t, 0]) * np.outer(kk, kk))
        Sd = A @ Sd + float(beta[t, 0]) * np.outer(kk, v[t, 0].astype(np.float64))
        ref = Sd.T @ q[t, 0].astype(np.float64)
        assert np.max(np.abs(out[t, 0] - ref)) <= 1e-5 * max(1.0, np.max(np.abs(ref))), t
    # the one requantization leaves the state within half a step of the exact one
    S_q = oracle.dequant(codes, scales, group=group)[0].astype(np.float64)
    half = np.repeat(scales[0], group, axis=0).astype(np.float64) / 2
    assert np.all(np.abs(S_q - Sd) <= half * (1 + 1e-5) + 1e-5 * np.abs(Sd).max())


def test_chunk_of_one_token_is_the_decode_step():
    rng = np.random.default_rng(5)
    n, d_k, d_v, group = 4, 16, 16, 8
    for mode in (oracle.ROUND_RTN, oracle.ROUND_SR, oracle.ROUND_BDR):
        _, codes, scales, pm = _quant_state(rng, n, d_k, d_v, group, 8)
        c2, s2 = codes.copy(), scales.copy()
        q, k, v, g, _ = _chunk_inputs(rng, 1, n, d_k, d_v)
        out = oracle.chunk_step(codes, scales, q, k, v, g, None, pm, np.arange(n), np.zeros(n),
                                group=group, update_kind=oracle.UPDATE_GATED,
                                gate_kind=oracle.GATE_PER_KEY, mode=mode, seed=3, step=9)
        o2 = oracle.step(c2, s2, q[0], k[0], v[0], g[0], None, pm, np.arange(n), np.zeros(n),
                         group=group, update_kind=oracle.UPDATE_GATED,
                         gate_kind=oracle.GATE_PER_KEY, mode=mode, seed=3, step=9)
        np.testing.assert_array_equal(out[0], o2)
        np.testing.assert_array_equal(codes, c2)
        np.testing.assert_array_equal(scales, s2)


def test_chunk_of_identity_tokens_leaves_state_unchanged():
    """Tokens with decay 1 and key 0 do not change the state; the one
    requantization of an imported state gives it back bit for bit."""
    rng = np.random.default_rng(8)
    n, d_k, d_v, group, T = 2, 16, 16, 8, 4
    for bits in (8, 4):
        _, codes, scales, pm = _quant_state(rng, n, d_k, d_v, group, bits)
        c0, s0 = codes.copy(), scales.copy()
        q, _, v, _, _ = _chunk_inputs(rng, T, n, d_k, d_v)
        oracle.chunk_step(codes, scales, q, np.zeros_like(q), v, np.ones((T, n, d_k), F32), None,
                          pm, np.arange(n), np.zeros(n), group=group,
                          update_kind=oracle.UPDATE_GATED, gate_kind=oracle.GATE_PER_KEY,
                          mode=oracle.ROUND_RTN)
        np.testing.assert_array_equal(codes, c0)
        np.testing.assert_array_equal(scales, s0)


@pytest.mark.parametrize("bits", [8, 4])
def test_chunk_bdr_bounded_toward_the_chunk_update(bits):
    """BDR at the chunk's end: the update is x_T - deq_0 (the whole chunk's
    change). An element never moves against it unless it sits on the adjacent
    grid point in its direction; elsewhere BDR is round-to-nearest."""
    rng = np.random.default_rng(90 + bits)
    n, d_k, d_v, group, T = 2, 16, 16, 8, 3
    qmax = 127 if bits == 8 else 7
    reversals = 0
    for trial in range(20):
        _, codes, scales, pm = _quant_state(rng, n, d_k, d_v, group, bits)
        q, k, v, g, _ = _chunk_inputs(rng, T, n, d_k, d_v)
        q *= F32(0.1)
        deq = oracle.dequant(codes, scales, group=group)
        x, _ = _unquantized(deq, q, k, v, g, None, oracle.UPDATE_GATED, oracle.GATE_PER_KEY)
        c_rtn, s_rtn = codes.copy(), scales.copy()
        args = (q, k, v, g, None, pm, np.arange(n), np.zeros(n))
        kw = dict(group=group, update_kind=oracle.UPDATE_GATED, gate_kind=oracle.GATE_PER_KEY)
        oracle.chunk_step(c_rtn, s_rtn, *args, mode=oracle.ROUND_RTN, **kw)
        oracle.chunk_step(codes, scales, *args, mode=oracle.ROUND_BDR, **kw)
        np.testing.assert_array_equal(scales, s_rtn)
        sc = np.repeat(scales, group, axis=1)
        A = np.repeat(np.abs(x).reshape(n, -1, group, d_v).max(axis=2), group, axis=1)
        inv = np.where(sc > 0, F32(qmax) / np.where(sc > 0, A, 1), 0).astype(F32)
        y = x.astype(np.float64) * inv.astype(np.float64)
        delta = (x - deq).astype(F32)
        moved = ((codes.astype(F32) * sc).astype(F32) - deq).astype(F32)
        up = codes == np.clip(np.ceil(y), -qmax, qmax)
        dn = codes == np.clip(np.floor(y), -qmax, qmax)
        ok = (delta == 0) | (moved * np.sign(delta) >= 0) | ((delta > 0) & up) | ((delta < 0) & dn)
        assert ok.all()
        rtn_moved = ((c_rtn.astype(F32) * sc).astype(F32) - deq).astype(F32)
        no_rev = ~(((delta > 0) & (rtn_moved < 0)) | ((delta < 0) & (rtn_moved > 0)))
        np.testing.assert_array_equal(codes[no_rev], c_rtn[no_rev])
        reversals += int((~no_rev).sum())
    assert reversals > 0


def test_chunk_sr_is_unbiased_about_the_chunk_end_state():
    rng = np.random.default_rng(66)
    n, d_k, d_v, group, T = 1, 16, 16, 8, 3
    _, codes, scales, pm = _quant_state(rng, n, d_k, d_v, group, 8)
    q, k, v, g, _ = _chunk_inputs(rng, T, n, d_k, d_v)
    deq = oracle.dequant(codes, scales, group=group)
    x, _ = _unquantized(deq, q, k, v, g, None, oracle.UPDATE_GATED, oracle.GATE_PER_KEY)
    N = 4000
    acc = np.zeros((d_k, d_v))
    for seed in range(N):
        c, s = codes.copy(), scales.copy()
        oracle.chunk_step(c, s, q, k, v, g, None, pm, [0], [0], group=group,
                          update_kind=oracle.UPDATE_GATED, gate_kind=oracle.GATE_PER_KEY,
                          mode=oracle.ROUND_SR, seed=seed, step=2)
        acc += c[0]
    sc = np.repeat(s[0], group, axis=0).astype(np.float64)
    mean = acc / N * sc
    xd = x[0].astype(np.float64)
    y = xd / np.where(sc > 0, sc, 1)
    fr = y - np.floor(y)
    sigma = sc * np.sqrt(fr * (1 - fr) / N)
    ok = np.abs(mean - xd) <= 3 * sigma + 1e-5 * np.abs(xd)
    assert ok.mean() >= 0.99


# ------------------------------------------------------------ bfloat16 ---

HAND_BF16 = [
    (1.0, 0x3F80), (-2.0, 0xC000),
    (1.0 + 2.0 ** -8, 0x3F80),            # halfway between 1 and 1 + 2^-7: even is 1
    (1.0 + 3 * 2.0 ** -8, 0x3F82),        # halfway between 1 + 2^-7 and 1 + 2^-6: even is the latter
    (-(1.0 + 2.0 ** -8 + 2.0 ** -20), 0xBF81),   # just past halfway: away from zero
    (0.0, 0x0000), (-0.0, 0x8000),
    (float("inf"), 0x7F80), (float("-inf"), 0xFF80),
    (3.3895313892515355e38, 0x7F7F),      # largest finite bfloat16
    (3.4028234663852886e38, 0x7F80),      # largest float32: past the midpoint, overflows
    (2.0 ** -133, 0x0001),                # smallest bfloat16 subnormal, exact
    (2.0 ** -134, 0x0000),                # half of it: tie to even (zero)
    (3 * 2.0 ** -134, 0x0002),            # 1.5 ulp: tie to even (2 ulp)
]


@pytest.mark.parametrize("x,pattern", HAND_BF16)
def test_bf16_hand_patterns(x, pattern):
    assert int(oracle.bf16_rne(np.array([x], F32))[0]) == pattern


def test_bf16_nan_is_quiet_nan_of_same_sign():
    got = oracle.bf16_rne(np.array([np.nan, -np.nan], F32))
    assert [int(g) for g in got] == [0x7FC0, 0xFFC0]


def test_bf16_matches_torch_conversion():
    rng = np.random.default_rng(4)
    bits = rng.integers(0, 2 ** 32, 200_000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(F32)
    x = x[~np.isnan(x)]
    ours = oracle.bf16_rne(x)
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def test_bf16_round_trip_of_every_finite_pattern():
    u = np.arange(2 ** 16, dtype=np.uint32).astype(np.uint16)
    f = oracle.bf16_to_f32(u)
    keep = ~np.isnan(f)
    np.testing.assert_array_equal(oracle.bf16_rne(f[keep]), u[keep])


def test_bf16_is_nearest_by_brute_force():
    rng = np.random.default_rng(12)
    x = (rng.standard_normal(20_000) * np.exp2(rng.integers(-30, 30, 20_000))).astype(F32)
    r = oracle.bf16_rne(x)
    rv = oracle.bf16_to_f32(r).astype(np.float64)
    xd = x.astype(np.float64)
    for step in (-1, 1):
        nb = oracle.bf16_to_f32((r.astype(np.int32) + step).astype(np.uint16)).astype(np.float64)
        assert np.all(np.abs(xd - rv) <= np.abs(xd - nb))
