"""Pins of the oracle's per-channel (per key-row group) precision.

The sources allow the decay-based precision choice per head or per channel.
Here a channel block is one scale group of `group` key rows. The pins: a
per-group map that gives every group its head's width reproduces the per-head
oracle; with mixed widths, every group's codes and scales are those of a
per-head run at that group's width (requantization is local to a group and the
update does not depend on the widths), and the outputs do not depend on the
widths at all; the map itself is the ranking of per-block mean decays.
"""
import numpy as np
import pytest

import oracle
from tests.test_oracle_chunk_bf16 import _chunk_inputs

F32 = np.float32
MODES = (oracle.ROUND_RTN, oracle.ROUND_SR, oracle.ROUND_BDR)


def _state(rng, n, d_k, d_v, group, bits):
    S0 = rng.standard_normal((n, d_k, d_v)).astype(F32)
    return oracle.import_fp32(S0, np.array([bits], np.uint8), np.zeros(n, np.int32), group=group)


@pytest.mark.parametrize("mode", MODES)
def test_uniform_group_map_is_the_head_map(mode):
    rng = np.random.default_rng(3 + mode)
    n, d_k, d_v, group = 4, 32, 16, 8
    for bits in (8, 4):
        codes, scales = _state(rng, n, d_k, d_v, group, bits)
        c2, s2 = codes.copy(), scales.copy()
        q, k, v, g, _ = _chunk_inputs(rng, 1, n, d_k, d_v)
        kw = dict(group=group, update_kind=oracle.UPDATE_GATED, gate_kind=oracle.GATE_PER_KEY,
                  mode=mode, seed=4, step=2)
        o1 = oracle.step(codes, scales, q[0], k[0], v[0], g[0], None, np.array([bits], np.uint8),
                         np.arange(n), np.zeros(n), **kw)
        o2 = oracle.step(c2, s2, q[0], k[0], v[0], g[0], None,
                         np.full((1, d_k // group), bits, np.uint8), np.arange(n), np.zeros(n),
                         **kw)
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(codes, c2)
        np.testing.assert_array_equal(scales, s2)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("delta", [False, True])
@pytest.mark.parametrize("T", [1, 3])
def test_mixed_groups_are_groupwise_head_runs(mode, delta, T):
    rng = np.random.default_rng(10 * T + mode + 5 * delta)
    n, d_k, d_v, group = 3, 32, 16, 8
    G = d_k // group
    pm = np.array([[8, 4, 4, 8]], np.uint8)
    # a logical state whose groups hold codes within each group's range
    codes8, scales = _state(rng, n, d_k, d_v, group, 8)
    codes = codes8.copy()
    for gi in range(G):
        if pm[0, gi] == 4:
            rows = slice(gi * group, (gi + 1) * group)
            codes[:, rows] = np.clip(codes[:, rows] // 18, -7, 7)
    q, k, v, g, beta = _chunk_inputs(rng, T, n, d_k, d_v, per_key=not delta, delta=delta)
    kw = dict(group=group, update_kind=oracle.UPDATE_DELTA if delta else oracle.UPDATE_GATED,
              gate_kind=oracle.GATE_SCALAR if delta else oracle.GATE_PER_KEY, mode=mode,
              seed=11, step=5)
    runs = {}
    for name, m in (("pg", pm), ("8", np.array([8], np.uint8)), ("4", np.array([4], np.uint8))):
        c, s = codes.copy(), scales.copy()
        o = oracle.chunk_step(c, s, q, k, v, g, beta, m, np.arange(n), np.zeros(n), **kw)
        runs[name] = (c, s, o)
    np.testing.assert_array_equal(runs["pg"][2], runs["8"][2])
    np.testing.assert_array_equal(runs["pg"][2], runs["4"][2])
    for gi in range(G):
        ref = runs[str(pm[0, gi])]
        rows = slice(gi * group, (gi + 1) * group)
        np.testing.assert_array_equal(runs["pg"][0][:, rows], ref[0][:, rows])
        np.testing.assert_array_equal(runs["pg"][1][:, gi], ref[1][:, gi])


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("delta", [False, True])
@pytest.mark.parametrize("step", [4, 7])                 # rank 4: step 7 merges, step 4 does not
def test_lrb_mixed_groups_are_groupwise_head_runs(mode, delta, step):
    """The same pins for the decode step with a Low-Rank Bypass buffer: with
    codes valid at both widths, a per-group map gives the outputs and buffer
    of both per-head runs, and each group the codes and scales of the run at
    its width; a uniform per-group map is the per-head map."""
    rng = np.random.default_rng(40 + 7 * mode + 3 * delta + step)
    n, d_k, d_v, group, rank = 3, 32, 16, 8, 4
    G = d_k // group
    pm = np.array([[4, 8, 8, 4]], np.uint8)
    codes8, scales = _state(rng, n, d_k, d_v, group, 8)
    codes = codes8.copy()
    for gi in range(G):
        if pm[0, gi] == 4:
            rows = slice(gi * group, (gi + 1) * group)
            codes[:, rows] = np.clip(codes[:, rows] // 18, -7, 7)
    q, k, v, g, beta = _chunk_inputs(rng, 1, n, d_k, d_v, per_key=not delta, delta=delta)
    m = step % rank
    U0 = np.zeros((n, rank, d_k), F32)
    V0 = np.zeros((n, rank, d_v), F32)
    U0[:, :m] = 0.3 * rng.standard_normal((n, m, d_k)).astype(F32)
    V0[:, :m] = 0.3 * rng.standard_normal((n, m, d_v)).astype(F32)
    kw = dict(group=group, update_kind=oracle.UPDATE_DELTA if delta else oracle.UPDATE_GATED,
              gate_kind=oracle.GATE_SCALAR if delta else oracle.GATE_PER_KEY, mode=mode,
              rank=rank, seed=13, step=step)
    runs = {}
    maps = (("pg", pm), ("8", np.array([8], np.uint8)), ("4", np.array([4], np.uint8)),
            ("pg8", np.full((1, G), 8, np.uint8)))
    for name, mp in maps:
        c, sc, U, V = codes.copy(), scales.copy(), U0.copy(), V0.copy()
        o = oracle.lrb_step(c, sc, U, V, q[0], k[0], v[0], g[0], None if beta is None else beta[0],
                            mp, np.arange(n), np.zeros(n), **kw)
        runs[name] = (c, sc, o, U, V)
    for other in ("8", "4"):
        for idx in (2, 3, 4):                      # output, U, V
            np.testing.assert_array_equal(runs["pg"][idx], runs[other][idx])
    for idx in range(5):
        np.testing.assert_array_equal(runs["pg8"][idx], runs["8"][idx])
    for gi in range(G):
        ref = runs[str(pm[0, gi])]
        rows = slice(gi * group, (gi + 1) * group)
        np.testing.assert_array_equal(runs["pg"][0][:, rows], ref[0][:, rows])
        np.testing.assert_array_equal(runs["pg"][1][:, gi], ref[1][:, gi])
    if m + 1 == rank:
        assert not runs["pg"][3].any() and not runs["pg"][4].any()     # emptied by the merge


def test_import_per_group_widths():
    rng = np.random.default_rng(2)
    n, d_k, d_v, group = 2, 16, 8, 4
    S0 = rng.standard_normal((n, d_k, d_v)).astype(F32)
    pm = np.array([[4, 8, 8, 4], [8, 8, 4, 4]], np.uint8)
    th = np.array([0, 1], np.int32)
    c, s = oracle.import_fp32(S0, pm, th, group=group)
    for t in range(n):
        for gi in range(4):
            bits = pm[th[t], gi]
            qmax = 127 if bits == 8 else 7
            rows = slice(gi * group, (gi + 1) * group)
            A = np.abs(S0[t, rows]).max(axis=0)
            np.testing.assert_array_equal(s[t, gi], (A / F32(qmax)).astype(F32))
            assert np.abs(c[t, rows]).max() <= qmax
            assert np.abs(c[t, rows]).max() == qmax      # the largest element hits the range


def test_invalid_group_map_rejected():
    codes = np.zeros((1, 16, 8), np.int8)
    scales = np.zeros((1, 2, 8), F32)
    x = np.zeros((1, 16), F32)
    with pytest.raises(ValueError):
        oracle.step(codes, scales, x, x, np.zeros((1, 8), F32), np.ones((1, 16), F32), None,
                    np.array([[8, 5]], np.uint8), [0], [0], group=8,
                    update_kind=oracle.UPDATE_GATED, gate_kind=oracle.GATE_PER_KEY, mode=0)
    with pytest.raises(ValueError):
        oracle.step(codes, scales, x, x, np.zeros((1, 8), F32), np.ones((1, 16), F32), None,
                    np.array([[8, 4, 4]], np.uint8), [0], [0], group=8,
                    update_kind=oracle.UPDATE_GATED, gate_kind=oracle.GATE_PER_KEY, mode=0)


def test_per_block_decay_ranking_hand_example():
    """Per-key decay [steps][H][d_k] viewed as [steps][H*G][group]: the block
    means rank the (head, group) blocks; the slowest-decaying half is int8."""
    H, d_k, group = 2, 8, 4
    decay = np.zeros((3, H, d_k), F32)
    # block means: (h0,g0)=0.9 (h0,g1)=0.5 (h1,g0)=0.7 (h1,g1)=0.95
    for (h, gi), m in {(0, 0): 0.9, (0, 1): 0.5, (1, 0): 0.7, (1, 1): 0.95}.items():
        decay[:, h, gi * group:(gi + 1) * group] = m
    decay[0, 0, 0] += F32(0.03)          # means are over steps and the block's keys
    decay[1, 0, 0] -= F32(0.03)
    means = oracle.decay_means(decay.reshape(3, H * 2, group))
    np.testing.assert_allclose(means, [0.9, 0.5, 0.7, 0.95], rtol=1e-6)
    pm = oracle.precision_map(means, 2).reshape(H, 2)
    np.testing.assert_array_equal(pm, [[8, 4], [4, 8]])
