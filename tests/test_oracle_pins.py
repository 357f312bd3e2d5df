"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks the oracle against something fixed independently of it:
published generator outputs, hand-derived steps (tests/golden/), the closed form
of the unquantized gated recurrence, an fp64 brute-force matrix recurrence for
the delta rule, special cases, and the invariants of the three rounding modes.
"""
import numpy as np
import pytest

import oracle
from tests.conftest import read_fixture, golden_path

F32 = np.float32
GAMMA = 0x9E3779B97F4A7C15
M64 = (1 << 64) - 1


# ------------------------------------------------------------------ hash ---

def _published_sequences():
    seqs, cur = {}, None
    with open(golden_path("splitmix64_vectors.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("seed"):
                cur = int(line.split()[1])
                seqs[cur] = []
            else:
                seqs[cur].append(int(line, 0))
    return seqs


def test_splitmix64_published_vectors():
    for seed, outs in _published_sequences().items():
        # a generator with state s returns mix(s), mix(s + gamma), ...
        got = [oracle.splitmix64((seed + n * GAMMA) & M64) for n in range(len(outs))]
        assert got == outs, seed


def test_hash_chain_reduces_to_published_outputs():
    """Choosing each coordinate equal to the previous link makes every xor
    vanish, so each link of the chain is mix(0) or mix(gamma), published values.
    Pins the order of the links and the halves (b, i high; h, j low)."""
    o1, o2 = _published_sequences()[0][:2]    # mix(0), mix(gamma)
    # seed 0 -> k0 = o1; step = o1 -> k1 = mix(0) = o1; (b,h) = o1 -> k2 = o1;
    # (i,j) = o1 -> r = o1
    hi, lo = o1 >> 32, o1 & 0xFFFFFFFF
    assert oracle.hash64(0, o1, hi, lo, hi, lo) == o1
    # last link: (i,j) = o1 ^ gamma -> r = mix(gamma) = o2
    x = o1 ^ GAMMA
    assert oracle.hash64(0, o1, hi, lo, x >> 32, x & 0xFFFFFFFF) == o2
    # swapping the halves breaks the chain
    assert oracle.hash64(0, o1, lo, hi, hi, lo) != o1
    assert oracle.hash64(0, o1, hi, lo, lo, hi) != o1


def test_uniform_grid_and_range():
    assert oracle.uniform(0) == 0.0
    assert oracle.uniform((1 << 41) - 1) == 0.0
    assert oracle.uniform(1 << 41) == 2.0 ** -23
    assert oracle.uniform(M64) == 1.0 - 2.0 ** -23
    rng = np.random.default_rng(0)
    u = np.array([oracle.uniform(int(r)) for r in rng.integers(0, 2**63, 4096, dtype=np.int64)])
    assert np.all((u >= 0) & (u < 1))
    assert np.all(u * 2**23 == np.floor(u * 2**23))


def test_hash_uniforms_are_uniform():
    # chi-square over 16 bins for 2^14 consecutive elements of one tile
    n, bins = 1 << 14, 16
    u = np.array([oracle.uniform(oracle.hash64(7, 3, 1, 2, i // 128, i % 128)) for i in range(n)])
    counts = np.bincount((u * bins).astype(int), minlength=bins)
    chi2 = ((counts - n / bins) ** 2 / (n / bins)).sum()
    assert chi2 < 37.7  # 99.9% quantile of chi-square with 15 dof


# ------------------------------------------------------ hand examples ---

def _load_case(name):
    fx = read_fixture(name)
    d_k, d_v, group = (int(fx[k][0]) for k in ("d_k", "d_v", "group"))
    bits = int(fx["bits"][0])
    upd = oracle.UPDATE_DELTA if fx["update"][0] == "delta" else oracle.UPDATE_GATED
    gate = oracle.GATE_PER_KEY if fx["gate"][0] == "per_key" else oracle.GATE_SCALAR
    arr = lambda key, dt=F32: np.array([float(x) for x in fx[key]], dt)
    case = dict(
        d_k=d_k, d_v=d_v, group=group, bits=bits, upd=upd, gate=gate,
        codes=np.array([int(x) for x in fx["codes_old"]], np.int8).reshape(1, d_k, d_v),
        scales=arr("scales_old").reshape(1, d_k // group, d_v),
        gates=arr("gates").reshape(1, -1), k=arr("k").reshape(1, d_k),
        v=arr("v").reshape(1, d_v), q=arr("q").reshape(1, d_k), out=arr("out"),
        beta=arr("beta") if "beta" in fx else None, fx=fx,
    )
    num_q = [r.split("/") for r in fx["scales_new_ratio"]]
    case["scales_new"] = np.array([F32(float(a)) / F32(float(b)) for a, b in num_q],
                                  F32).reshape(d_k // group, d_v)
    return case


def _run_case(c, mode, seed=0, step=0):
    codes, scales = c["codes"].copy(), c["scales"].copy()
    out = oracle.step(codes, scales, c["q"], c["k"], c["v"], c["gates"], c["beta"],
                      np.array([c["bits"]], np.uint8), [0], [0], group=c["group"],
                      update_kind=c["upd"], gate_kind=c["gate"], mode=mode, seed=seed, step=step)
    return codes[0], scales[0], out[0]


@pytest.mark.parametrize("name", ["hand_gla_int8_rtn_4x2.txt", "hand_gla_int8_bdr_2x2.txt",
                                  "hand_gdn_int4_rtn_2x2.txt", "hand_gla_int8_ties_2x2.txt",
                                  "hand_clamp_int8_1x2.txt", "hand_exact_product_int8_2x2.txt",
                                  "hand_bdr_zero_move_int8_2x2.txt"])
def test_hand_examples_rtn(name):
    c = _load_case(name)
    codes, scales, out = _run_case(c, oracle.ROUND_RTN)
    expect = np.array([int(x) for x in c["fx"]["codes_rtn"]], np.int8).reshape(c["d_k"], c["d_v"])
    np.testing.assert_array_equal(out, c["out"])
    np.testing.assert_array_equal(scales, c["scales_new"])
    np.testing.assert_array_equal(codes, expect)


HAND_BDR = ["hand_gla_int8_bdr_2x2.txt", "hand_clamp_int8_1x2.txt",
            "hand_exact_product_int8_2x2.txt", "hand_bdr_zero_move_int8_2x2.txt"]


@pytest.mark.parametrize("name", HAND_BDR)
def test_hand_example_bdr(name):
    c = _load_case(name)
    codes, scales, out = _run_case(c, oracle.ROUND_BDR)
    expect = np.array([int(x) for x in c["fx"]["codes_bdr"]], np.int8).reshape(c["d_k"], c["d_v"])
    np.testing.assert_array_equal(codes, expect)
    np.testing.assert_array_equal(scales, c["scales_new"])
    np.testing.assert_array_equal(out, c["out"])


@pytest.mark.parametrize("seed,step", [(0, 0), (11, 5), (0x5EED, 1 << 40)])
def test_hand_example_sr(seed, step):
    c = _load_case("hand_gla_int8_bdr_2x2.txt")
    codes, _, _ = _run_case(c, oracle.ROUND_SR, seed=seed, step=step)
    fl = [int(x) for x in c["fx"]["sr_floor"]]
    fr = [float(x) for x in c["fx"]["sr_frac"]]
    for e in range(4):
        i, j = divmod(e, 2)
        u = oracle.uniform(oracle.hash64(seed, step, 0, 0, i, j))
        assert codes[i, j] == fl[e] + (1 if u < fr[e] else 0)


def test_sr_draw_equal_to_fraction_rounds_down():
    """u == fraction must not round up: P(up) equals the fraction exactly."""
    fx = read_fixture("sr_boundary_step.txt")
    seed, step = int(fx["seed"][0]), int(fx["step"][0])
    assert oracle.uniform(oracle.hash64(seed, step, 0, 0, 1, 0)) == 0.5
    c = _load_case("hand_gla_int8_ties_2x2.txt")
    codes, _, _ = _run_case(c, oracle.ROUND_SR, seed=seed, step=step)
    assert codes[1, 0] == 2


def test_sr_codes_clamped_to_symmetric_range():
    fx = read_fixture("sr_clamp_steps.txt")
    seed = int(fx["seed"][0])
    c = _load_case("hand_clamp_int8_1x2.txt")
    up, down = int(fx["step_up"][0]), int(fx["step_down"][0])
    assert oracle.uniform(oracle.hash64(seed, up, 0, 0, 0, 0)) < 5 * 2.0 ** -20
    assert oracle.uniform(oracle.hash64(seed, down, 0, 0, 0, 1)) >= 1 - 5 * 2.0 ** -20
    for step in (up, down, 0):
        codes, _, _ = _run_case(c, oracle.ROUND_SR, seed=seed, step=step)
        np.testing.assert_array_equal(codes, [[127, -127]])


# ------------------------------------------------ recurrence pins (fp64) ---

def _rand_inputs(rng, T, d_k, d_v, per_key=True, delta=False):
    q = rng.standard_normal((T, d_k)).astype(F32)
    k = rng.standard_normal((T, d_k)).astype(F32)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, d_v)).astype(F32)
    if per_key:
        g = np.exp(-np.log1p(np.exp(rng.normal(-2.0, 1.0, (T, d_k))))).astype(F32)
    else:
        g = (1 / (1 + np.exp(-rng.normal(2.0, 1.0, (T, 1))))).astype(F32)
    beta = (1 / (1 + np.exp(-rng.normal(0, 1, (T, 1))))).astype(F32) if delta else None
    return q, k.astype(F32), v, g, beta


@pytest.mark.parametrize("d_k,d_v,per_key", [(4, 4, True), (8, 5, True), (6, 8, False)])
def test_gated_recurrence_matches_closed_form(d_k, d_v, per_key):
    """Unquantized gated step vs o_t = sum_s (prod decay)(q_t . k_s) v_s + decayed S0,
    read per key channel."""
    rng = np.random.default_rng(d_k * 100 + d_v)
    T = 16
    q, k, v, g, _ = _rand_inputs(rng, T, d_k, d_v, per_key=per_key)
    S0 = rng.standard_normal((d_k, d_v)).astype(F32) * F32(0.1)
    S = S0[None].copy()
    gate_kind = oracle.GATE_PER_KEY if per_key else oracle.GATE_SCALAR
    gd = np.broadcast_to(g.astype(np.float64), (T, d_k))
    for t in range(T):
        out = oracle.fp32_step(S, q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1].reshape(1, -1),
                               None, update_kind=oracle.UPDATE_GATED, gate_kind=gate_kind)[0]
        ref = np.zeros(d_v)
        for s in range(t + 1):
            decay = np.prod(gd[s + 1:t + 1], axis=0)            # [d_k]
            ref += np.sum(q[t] * decay * k[s]) * v[s].astype(np.float64)
        ref += (q[t] * np.prod(gd[:t + 1], axis=0)) @ S0.astype(np.float64)
        assert np.max(np.abs(out - ref)) <= 1e-5 * max(1.0, np.max(np.abs(ref))), t


@pytest.mark.parametrize("d_k,d_v", [(4, 4), (8, 6)])
def test_delta_recurrence_matches_matrix_brute_force(d_k, d_v):
    """Unquantized delta step vs S_t = alpha (I - beta k k^T) S + beta k v^T in fp64."""
    rng = np.random.default_rng(7 + d_k)
    T = 16
    q, k, v, a, beta = _rand_inputs(rng, T, d_k, d_v, per_key=False, delta=True)
    S0 = rng.standard_normal((d_k, d_v)).astype(F32) * F32(0.1)
    S = S0[None].copy()
    Sd = S0.astype(np.float64)
    for t in range(T):
        out = oracle.fp32_step(S, q[t:t + 1], k[t:t + 1], v[t:t + 1], a[t:t + 1], beta[t],
                               update_kind=oracle.UPDATE_DELTA, gate_kind=oracle.GATE_SCALAR)[0]
        kk = k[t].astype(np.float64)
        A = float(a[t, 0]) * (np.eye(d_k) - float(beta[t, 0]) * np.outer(kk, kk))
        Sd = A @ Sd + float(beta[t, 0]) * np.outer(kk, v[t].astype(np.float64))
        ref = Sd.T @ q[t].astype(np.float64)
        assert np.max(np.abs(out - ref)) <= 1e-5 * max(1.0, np.max(np.abs(ref))), t
        assert np.max(np.abs(S[0] - Sd)) <= 1e-5 * max(1.0, np.max(np.abs(Sd)))


def test_delta_with_zero_beta_is_scalar_gating():
    rng = np.random.default_rng(3)
    d_k, d_v = 8, 8
    S = rng.standard_normal((1, d_k, d_v)).astype(F32)
    q, k, v, a, _ = _rand_inputs(rng, 1, d_k, d_v, per_key=False)
    S1, S2 = S.copy(), S.copy()
    o1 = oracle.fp32_step(S1, q, k, v, a, np.zeros(1, F32), update_kind=oracle.UPDATE_DELTA,
                          gate_kind=oracle.GATE_SCALAR)
    o2 = oracle.fp32_step(S2, q, k, np.zeros_like(v), a, None, update_kind=oracle.UPDATE_GATED,
                          gate_kind=oracle.GATE_SCALAR)
    np.testing.assert_array_equal(S1, S2)
    np.testing.assert_array_equal(o1, o2)


def test_delta_unit_key_overwrites_row():
    """k = e_i, alpha = beta = 1: (I - e_i e_i^T) S + e_i v^T replaces row i by v.
    Values on a coarse dyadic grid keep every rounding exact."""
    rng = np.random.default_rng(5)
    d_k, d_v, row = 6, 4, 2
    S = (rng.integers(-64, 64, (1, d_k, d_v)) / 16).astype(F32)
    v = (rng.integers(-64, 64, (1, d_v)) / 16).astype(F32)
    k = np.zeros((1, d_k), F32)
    k[0, row] = 1
    q = np.ones((1, d_k), F32)
    S0 = S.copy()
    oracle.fp32_step(S, q, k, v, np.ones((1, 1), F32), np.ones(1, F32),
                     update_kind=oracle.UPDATE_DELTA, gate_kind=oracle.GATE_SCALAR)
    expect = S0.copy()
    expect[0, row] = v[0]
    np.testing.assert_array_equal(S, expect)


def test_output_is_matrix_vector_product():
    rng = np.random.default_rng(9)
    d_k, d_v = 16, 12
    S = rng.standard_normal((3, d_k, d_v)).astype(F32)
    q, k, v, g, _ = _rand_inputs(rng, 3, d_k, d_v)
    out = oracle.fp32_step(S, q, k, v, g, None, update_kind=oracle.UPDATE_GATED,
                           gate_kind=oracle.GATE_PER_KEY)
    for t in range(3):
        ref = S[t].astype(np.float64).T @ q[t].astype(np.float64)
        assert np.max(np.abs(out[t] - ref)) <= 1e-5 * np.max(np.abs(ref))


# --------------------------------------------------- quantizer pins ---

def _quant_state(rng, n, d_k, d_v, group, bits, scale=1.0):
    S0 = (rng.standard_normal((n, d_k, d_v)) * scale).astype(F32)
    pm = np.full(1, bits, np.uint8)
    codes, scales = oracle.import_fp32(S0, pm, np.zeros(n, np.int32), group=group)
    return S0, codes, scales, pm


@pytest.mark.parametrize("bits", [8, 4])
def test_dequant_is_code_times_group_scale(bits):
    rng = np.random.default_rng(bits)
    _, codes, scales, _ = _quant_state(rng, 2, 8, 6, 4, bits)
    S = oracle.dequant(codes, scales, group=4)
    expect = codes.astype(F32) * np.repeat(scales, 4, axis=1)
    np.testing.assert_array_equal(S, expect)


@pytest.mark.parametrize("bits,group", [(8, 4), (4, 2), (8, 8)])
def test_import_rtn_error_bound_and_full_range(bits, group):
    rng = np.random.default_rng(100 + bits)
    qmax = 127 if bits == 8 else 7
    S0, codes, scales, _ = _quant_state(rng, 4, 8, 8, group, bits)
    assert np.all(np.abs(codes.astype(int)) <= qmax)
    S = oracle.dequant(codes, scales, group=group).astype(np.float64)
    sc = np.repeat(scales, group, axis=1).astype(np.float64)
    assert np.all(np.abs(S - S0) <= sc * (0.5 + 1e-5))
    # the largest element of every (group, column) lands on +-qmax
    cm = np.abs(codes.astype(int)).reshape(4, 8 // group, group, 8).max(axis=2)
    assert np.all(cm == qmax)


def test_tiny_column_group_stored_as_zero():
    """Reading: a (group, column) whose absmax is below 2^-100 is stored as zero
    (scale 0, codes 0), which keeps qmax/absmax finite."""
    pm = np.full(1, 8, np.uint8)
    S0 = np.zeros((1, 2, 3), F32)
    S0[0, :, 0] = [2.0 ** -110, -2.0 ** -111]   # below the threshold
    S0[0, :, 1] = [2.0 ** -90, 0.0]             # above it: quantized normally
    S0[0, :, 2] = [2.0 ** -100, 0.0]            # at it: quantized normally
    codes, scales = oracle.import_fp32(S0, pm, [0], group=2)
    assert scales[0, 0, 0] == 0 and not codes[0, :, 0].any()
    assert codes[0, 0, 1] == 127 and scales[0, 0, 1] == F32(2.0 ** -90) / F32(127)
    assert codes[0, 0, 2] == 127


def test_zero_state_imports_to_zero():
    pm = np.full(1, 8, np.uint8)
    codes, scales = oracle.import_fp32(np.zeros((1, 4, 4), F32), pm, [0], group=2)
    assert not codes.any() and not scales.any()


@pytest.mark.parametrize("bits,group,upd,gate", [
    (8, 4, oracle.UPDATE_GATED, oracle.GATE_PER_KEY),
    (4, 8, oracle.UPDATE_GATED, oracle.GATE_SCALAR),
    (8, 16, oracle.UPDATE_DELTA, oracle.GATE_SCALAR),
    (4, 4, oracle.UPDATE_DELTA, oracle.GATE_SCALAR)])
def test_rtn_idempotent_under_identity_decay_and_zero_update(bits, group, upd, gate):
    rng = np.random.default_rng(bits * 10 + group)
    n, d_k, d_v = 8, 16, 16
    for scale in (1.0, 1e-3, 37.0):
        _, codes, scales, pm = _quant_state(rng, n, d_k, d_v, group, bits, scale)
        c0, s0 = codes.copy(), scales.copy()
        glen = d_k if gate == oracle.GATE_PER_KEY else 1
        oracle.step(codes, scales, rng.standard_normal((n, d_k)), np.zeros((n, d_k)),
                    rng.standard_normal((n, d_v)), np.ones((n, glen)), np.zeros(n),
                    pm, np.arange(n), np.zeros(n), group=group, update_kind=upd, gate_kind=gate,
                    mode=oracle.ROUND_RTN)
        np.testing.assert_array_equal(codes, c0)
        np.testing.assert_array_equal(scales, s0)


def _one_step_parts(rng, bits, mode, n=1, d_k=32, d_v=32, group=8, seed=0):
    """A quantized state plus one step's inputs, with the pre-rounding x taken
    from the unquantized step applied to the dequantized state."""
    _, codes, scales, pm = _quant_state(rng, n, d_k, d_v, group, bits)
    q, k, v, g, _ = _rand_inputs(rng, n, d_k, d_v)
    deq = oracle.dequant(codes, scales, group=group)
    x = deq.copy()
    oracle.fp32_step(x, q, k, v, g, None, update_kind=oracle.UPDATE_GATED,
                     gate_kind=oracle.GATE_PER_KEY)
    return codes, scales, pm, q, k, v, g, deq, x


@pytest.mark.parametrize("bits", [8, 4])
def test_sr_mean_over_seeds_is_unbiased(bits):
    rng = np.random.default_rng(55 + bits)
    d_k, d_v, group = 32, 32, 8
    codes, scales, pm, q, k, v, g, deq, x = _one_step_parts(rng, bits, oracle.ROUND_SR)
    N = 10_000
    acc = np.zeros((d_k, d_v))
    s_new = None
    for seed in range(N):
        c, s = codes.copy(), scales.copy()
        oracle.step(c, s, q, k, v, g, None, pm, [0], [0], group=group,
                    update_kind=oracle.UPDATE_GATED, gate_kind=oracle.GATE_PER_KEY,
                    mode=oracle.ROUND_SR, seed=seed, step=1)
        acc += c[0]
        s_new = s[0] if s_new is None else s_new
        assert np.array_equal(s[0], s_new)   # scales do not depend on the draw
    sc = np.repeat(s_new, group, axis=0).astype(np.float64)
    mean = acc / N * sc
    xd = x[0].astype(np.float64)
    inv = np.where(sc > 0, 1.0 / np.where(sc > 0, sc, 1), 0)
    y = xd * inv
    fr = y - np.floor(y)
    sigma = sc * np.sqrt(fr * (1 - fr) / N)
    exact = fr < 1e-6
    assert np.all(np.abs(mean[exact] - xd[exact]) <= 1e-5 * np.abs(xd[exact]) + 1e-30)
    ok = np.abs(mean - xd) <= 3 * sigma + 1e-6 * np.abs(xd)
    assert ok[~exact].mean() >= 0.99


@pytest.mark.parametrize("bits", [8, 4])
def test_bdr_never_moves_against_update(bits):
    rng = np.random.default_rng(77 + bits)
    group, qmax = 8, (127 if bits == 8 else 7)
    reversals = 0
    for trial in range(20):
        codes, scales, pm, q, k, v, g, deq, x = _one_step_parts(rng, bits, oracle.ROUND_BDR,
                                                                n=2, group=group)
        c_rtn, s_rtn = codes.copy(), scales.copy()
        oracle.step(c_rtn, s_rtn, q, k, v, g, None, pm, [0, 1], [0, 0], group=group,
                    update_kind=oracle.UPDATE_GATED, gate_kind=oracle.GATE_PER_KEY,
                    mode=oracle.ROUND_RTN)
        oracle.step(codes, scales, q, k, v, g, None, pm, [0, 1], [0, 0], group=group,
                    update_kind=oracle.UPDATE_GATED, gate_kind=oracle.GATE_PER_KEY,
                    mode=oracle.ROUND_BDR)
        np.testing.assert_array_equal(scales, s_rtn)
        sc = np.repeat(scales, group, axis=1)
        inv = np.where(sc > 0, F32(qmax) / np.where(sc > 0, np.repeat(
            np.abs(x).reshape(2, -1, group, x.shape[2]).max(axis=2), group, axis=1), 1), 0)
        y = x.astype(np.float64) * inv.astype(F32).astype(np.float64)   # exact product
        delta = (x - deq).astype(F32)
        moved = ((codes.astype(F32) * sc).astype(F32) - deq).astype(F32)
        bounded_up = codes == np.clip(np.ceil(y), -qmax, qmax)
        bounded_dn = codes == np.clip(np.floor(y), -qmax, qmax)
        ok = (delta == 0) | (moved * np.sign(delta) >= 0) | \
             ((delta > 0) & bounded_up) | ((delta < 0) & bounded_dn)
        assert ok.all()
        assert np.all(np.abs(codes.astype(np.float64) - y) < 1.0 + 1e-6)
        # where round-to-nearest does not reverse, BDR is round-to-nearest
        rtn_moved = ((c_rtn.astype(F32) * sc).astype(F32) - deq).astype(F32)
        no_rev = ~(((delta > 0) & (rtn_moved < 0)) | ((delta < 0) & (rtn_moved > 0)))
        np.testing.assert_array_equal(codes[no_rev], c_rtn[no_rev])
        reversals += int((~no_rev).sum())
    assert reversals > 0   # the case under test actually occurs


def test_quantized_trajectory_tracks_closed_form():
    """int8 RTN steps stay close to the exact unquantized recurrence (a loose
    pin on the whole quantized step: dequant, update, output, requant)."""
    rng = np.random.default_rng(21)
    d_k, d_v, group, T = 16, 16, 8, 16
    q, k, v, g, _ = _rand_inputs(rng, T, d_k, d_v)
    codes = np.zeros((1, d_k, d_v), np.int8)
    scales = np.zeros((1, d_k // group, d_v), F32)
    pm = np.full(1, 8, np.uint8)
    gd = g.astype(np.float64)
    for t in range(T):
        out = oracle.step(codes, scales, q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1], None,
                          pm, [0], [0], group=group, update_kind=oracle.UPDATE_GATED,
                          gate_kind=oracle.GATE_PER_KEY, mode=oracle.ROUND_RTN)[0]
        ref = np.zeros(d_v)
        for s in range(t + 1):
            ref += np.sum(q[t] * np.prod(gd[s + 1:t + 1], axis=0) * k[s]) * v[s]
        assert np.max(np.abs(out - ref)) <= 3e-2 * np.max(np.abs(ref)), t


# --------------------------------------------------- precision map ---

def test_precision_map_hand_examples():
    means = np.array([0.9, 0.95, 0.5, 0.95])
    np.testing.assert_array_equal(oracle.precision_map(means, 2), [4, 8, 4, 8])
    np.testing.assert_array_equal(oracle.precision_map(means, 1), [4, 8, 4, 4])
    np.testing.assert_array_equal(oracle.precision_map(means, 3), [8, 8, 4, 8])
    np.testing.assert_array_equal(oracle.precision_map(means, 0), [4, 4, 4, 4])
    np.testing.assert_array_equal(oracle.precision_map(means, 4), [8, 8, 8, 8])


def test_decay_means_closed_form():
    outer, H, inner = 6, 3, 5
    o = np.arange(outer)[:, None, None]
    h = np.arange(H)[None, :, None]
    c = np.arange(inner)[None, None, :]
    decay = (0.25 * h + 0.01 * o + 0.001 * c + 0.1).astype(F32)
    means = oracle.decay_means(decay)
    # arithmetic progressions: mean = 0.25 h + 0.01 (outer-1)/2 + 0.001 (inner-1)/2 + 0.1
    expect = 0.25 * np.arange(H) + 0.01 * (outer - 1) / 2 + 0.001 * (inner - 1) / 2 + 0.1
    np.testing.assert_allclose(means, expect, rtol=1e-6)
