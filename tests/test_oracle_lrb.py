"""Pins of the oracle's Low-Rank Bypass step (the readings are stated at
orc_lrb_step in oracle/lrs_oracle.c).

Between merges the quantized part only decays, so it must match the plain
decode step given a zero key; the buffer must hold the decayed rank-1 updates
(fp64 recurrence); the output and the delta rule's w must read the effective
state deq + U V^T (fp64); a merge adds exactly the elements of U V^T of at
least half a quantization step and empties the buffer; and updates too small
for the quantized state alone accumulate in the buffer until they are merged.
"""
import numpy as np
import pytest

import oracle

F32 = np.float32
CASES = [(oracle.UPDATE_GATED, oracle.GATE_PER_KEY), (oracle.UPDATE_GATED, oracle.GATE_SCALAR),
         (oracle.UPDATE_DELTA, oracle.GATE_SCALAR)]


def _setup(rng, n, d_k, d_v, group, bits, scale=0.3):
    S0 = (rng.standard_normal((n, d_k, d_v)) * scale).astype(F32)
    pm = np.array([bits], np.uint8)
    codes, scales = oracle.import_fp32(S0, pm, np.zeros(n, np.int32), group=group)
    return codes, scales, pm


def _inputs(rng, n, d_k, d_v, upd, gate, vscale=0.05):
    q = rng.standard_normal((n, d_k)).astype(F32)
    k = rng.standard_normal((n, d_k)).astype(F32)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = (rng.standard_normal((n, d_v)) * vscale).astype(F32)
    if gate == oracle.GATE_PER_KEY:
        g = rng.uniform(0.9, 1.0, (n, d_k)).astype(F32)
    else:
        g = rng.uniform(0.9, 1.0, (n, 1)).astype(F32)
    beta = rng.uniform(0.2, 0.9, n).astype(F32) if upd == oracle.UPDATE_DELTA else None
    return q, k.astype(F32), v, g, beta


@pytest.mark.parametrize("upd,gate", CASES)
@pytest.mark.parametrize("mode", [oracle.ROUND_RTN, oracle.ROUND_SR, oracle.ROUND_BDR])
def test_between_merges_state_only_decays(upd, gate, mode):
    rng = np.random.default_rng(upd * 10 + gate + 3 * mode)
    n, d_k, d_v, group, r = 3, 16, 8, 8, 4
    codes, scales, pm = _setup(rng, n, d_k, d_v, group, 8)
    U = np.zeros((n, r, d_k), F32)
    V = np.zeros((n, r, d_v), F32)
    c2, s2 = codes.copy(), scales.copy()
    kw = dict(group=group, update_kind=upd, gate_kind=gate, mode=mode, seed=5)
    for t in range(r - 1):                       # steps 0..r-2 never merge
        q, k, v, g, beta = _inputs(rng, n, d_k, d_v, upd, gate)
        oracle.lrb_step(codes, scales, U, V, q, k, v, g, beta, pm, np.arange(n), np.zeros(n),
                        rank=r, step=t, **kw)
        oracle.step(c2, s2, q, np.zeros_like(k), v, g, beta, pm, np.arange(n), np.zeros(n),
                    step=t, **kw)
        np.testing.assert_array_equal(codes, c2)
        np.testing.assert_array_equal(scales, s2)


@pytest.mark.parametrize("upd,gate", CASES)
def test_buffer_output_and_w_read_the_effective_state(upd, gate):
    rng = np.random.default_rng(40 + upd * 10 + gate)
    n, d_k, d_v, group, r = 2, 16, 8, 8, 4
    codes, scales, pm = _setup(rng, n, d_k, d_v, group, 8)
    U = np.zeros((n, r, d_k), F32)
    V = np.zeros((n, r, d_v), F32)
    Ud = np.zeros((n, r, d_k))                  # fp64 recurrence of the buffer
    for t in range(r - 1):
        q, k, v, g, beta = _inputs(rng, n, d_k, d_v, upd, gate)
        deq32 = oracle.dequant(codes, scales, group=group)
        deq = deq32.astype(np.float64)
        S_eff = deq + np.einsum("nli,nlj->nij", U.astype(np.float64), V.astype(np.float64))
        out, x = oracle.lrb_step(codes, scales, U, V, q, k, v, g, beta, pm, np.arange(n),
                                 np.zeros(n), group=group, update_kind=upd, gate_kind=gate,
                                 mode=oracle.ROUND_RTN, rank=r, step=t, want_x=True)
        gd = np.broadcast_to(g.astype(np.float64), (n, d_k))
        if upd == oracle.UPDATE_DELTA:
            a = g[:, 0].astype(np.float64)
            u = np.einsum("ni,nij->nj", k.astype(np.float64), S_eff)
            w = beta[:, None] * (v - a[:, None] * u)
        else:
            w = v.astype(np.float64)
        np.testing.assert_allclose(V[:, t], w, rtol=1e-5, atol=1e-7)        # appended w
        np.testing.assert_array_equal(U[:, t], k)                            # appended k
        Ud[:, :t] *= gd[:, None, :]
        Ud[:, t] = k
        np.testing.assert_allclose(U, Ud, rtol=1e-5, atol=1e-12)
        # x = RN(g deq): the quantized part only decays
        np.testing.assert_array_equal(x, (g[:, :, None] * deq32).astype(F32))
        x_eff = x.astype(np.float64) + np.einsum("nli,nlj->nij", U.astype(np.float64),
                                                  V.astype(np.float64))
        ref = np.einsum("ni,nij->nj", q.astype(np.float64), x_eff)
        assert np.max(np.abs(out - ref)) <= 1e-5 * max(1.0, np.abs(ref).max())


@pytest.mark.parametrize("bits", [8, 4])
def test_merge_adds_large_elements_and_empties_buffer(bits):
    rng = np.random.default_rng(70 + bits)
    n, d_k, d_v, group, r = 2, 16, 8, 8, 3
    merged_any = kept_any = False
    for trial in range(6):
        codes, scales, pm = _setup(rng, n, d_k, d_v, group, bits)
        U = np.zeros((n, r, d_k), F32)
        V = np.zeros((n, r, d_v), F32)
        for t in range(r):
            q, k, v, g, _ = _inputs(rng, n, d_k, d_v, oracle.UPDATE_GATED, oracle.GATE_PER_KEY,
                                    vscale=0.02 * (trial + 1))
            s_old = np.repeat(scales, group, axis=1).astype(np.float64)
            deq = oracle.dequant(codes, scales, group=group)
            if t == r - 1:
                Ud = U.astype(np.float64).copy()
                Ud[:, :t] *= g.astype(np.float64)[:, None, :]
                Ud[:, t] = k
                Vd = V.astype(np.float64).copy()
                Vd[:, t] = v
                M = np.einsum("nli,nlj->nij", Ud, Vd)
            out, x = oracle.lrb_step(codes, scales, U, V, q, k, v, g, None, pm, np.arange(n),
                                     np.zeros(n), group=group, update_kind=oracle.UPDATE_GATED,
                                     gate_kind=oracle.GATE_PER_KEY, mode=oracle.ROUND_RTN,
                                     rank=r, step=t, want_x=True)
        base = (g[:, :, None] * deq).astype(F32).astype(np.float64)     # RN(g deq)
        big = np.abs(M) >= 0.5 * s_old * (1 + 1e-4)
        small = np.abs(M) <= 0.5 * s_old * (1 - 1e-4)
        np.testing.assert_array_equal(x[small], base[small])
        np.testing.assert_allclose(x[big], base[big] + M[big], rtol=1e-5, atol=1e-6)
        merged_any |= bool(big.any())
        kept_any |= bool(small.any())
        assert not U.any() and not V.any()
    assert merged_any and kept_any


def test_small_updates_survive_through_the_buffer():
    """Updates each below half a quantization step: the plain step rounds
    every one of them away, the buffer accumulates them until the merge moves
    the state."""
    n, d_k, d_v, group, r = 1, 8, 8, 8, 4
    S0 = np.zeros((n, d_k, d_v), F32)
    S0[0, 0, :] = 1.0                          # scale 1/127 in every column
    pm = np.array([8], np.uint8)
    codes, scales = oracle.import_fp32(S0, pm, [0], group=group)
    c_plain, s_plain = codes.copy(), scales.copy()
    U = np.zeros((n, r, d_k), F32)
    V = np.zeros((n, r, d_v), F32)
    k = np.zeros((n, d_k), F32)
    k[0, 3] = 1.0                               # updates land in row 3 only
    v = np.full((n, d_v), 0.3 / 127, F32)       # 0.3 of a quantization step per step
    q = np.ones((n, d_k), F32)
    g = np.ones((n, d_k), F32)
    kw = dict(group=group, update_kind=oracle.UPDATE_GATED, gate_kind=oracle.GATE_PER_KEY,
              mode=oracle.ROUND_RTN)
    for t in range(r):
        oracle.step(c_plain, s_plain, q, k, v, g, None, pm, [0], [0], step=t, **kw)
        oracle.lrb_step(codes, scales, U, V, q, k, v, g, None, pm, [0], [0], rank=r, step=t, **kw)
        if t < r - 1:
            assert not codes[0, 3].any()
    assert not c_plain[0, 3].any()              # lost by the plain step
    assert (codes[0, 3] == 1).all()             # 4 x 0.3 steps merged: one grid step up


def test_merge_threshold_is_inclusive():
    """An element of the buffer exactly half a quantization step is merged
    (the threshold is |M| >= s/2). Powers of two keep every sum exact."""
    n, d_k, d_v, group, r = 1, 8, 8, 8, 4
    S0 = np.zeros((n, d_k, d_v), F32)
    S0[0, 0, :] = F32(127 * 2.0 ** -7)          # scale exactly 2^-7
    pm = np.array([8], np.uint8)
    codes, scales = oracle.import_fp32(S0, pm, [0], group=group)
    assert (scales == F32(2.0 ** -7)).all()
    U = np.zeros((n, r, d_k), F32)
    V = np.zeros((n, r, d_v), F32)
    k = np.zeros((n, d_k), F32)
    k[0, 5] = 1.0
    v = np.full((n, d_v), 2.0 ** -10, F32)      # four of them make 2^-8 = s/2
    q, g = np.ones((n, d_k), F32), np.ones((n, d_k), F32)
    for t in range(r):
        _, x = oracle.lrb_step(codes, scales, U, V, q, k, v, g, None, pm, [0], [0], group=group,
                               update_kind=oracle.UPDATE_GATED, gate_kind=oracle.GATE_PER_KEY,
                               mode=oracle.ROUND_RTN, rank=r, step=t, want_x=True)
    np.testing.assert_array_equal(x[0, 5], np.full(d_v, 2.0 ** -8, F32))
