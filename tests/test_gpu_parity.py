"""GPU parity of the fused decode step against the CPU oracle, through the C ABI.

Small cases compare every tile at every step; the full-size workloads compare
a spread sample of tiles over the whole trajectory (tiles are independent, so
a sampled tile's trajectory is exact) with the kernel launched exactly as the
benchmark launches it.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_recurrent_state_decode_b200 import inputs as I
from quantized_recurrent_state_decode_b200 import lrs
from tests import parity as P

pytestmark = pytest.mark.gpu

W = I.WORKLOADS


def _small(family, B, H, d_k, d_v, group, mode, precision, steps, frac=0.5, name=None,
           s0_std=0.02, gate_mu=None):
    mu = {"gla": -3.0, "gdn": 4.0, "mamba2": -2.0}[family] if gate_mu is None else gate_mu
    return I.Workload(name or "%s_%s_%d_%d_%dx%d_g%d_m%d" % (family, precision, B, H, d_k, d_v,
                                                           group, mode),
                      family, B, H, d_k, d_v, group, steps, mode, precision,
                      int8_fraction=frac, s0_std=s0_std, gate_mu=mu, seed_id=100 + B + H + mode)


def test_gla_rtn_int8_small_every_tile_every_step():
    stats = {}
    w = W["gla_rtn_int8_b2h2_64"]
    P.run_parity(w, w.steps, check_every=1, stats=stats)
    assert stats["exact_out_steps"] == w.steps


GRID = []
for fam in ("gla", "gdn", "mamba2"):
    for mode in (I.ROUND_RTN, I.ROUND_SR, I.ROUND_BDR):
        for prec in ("int8", "int4", "mixed"):
            GRID.append((fam, mode, prec))


@pytest.mark.parametrize("fam,mode,prec", GRID)
def test_mode_family_precision_grid(fam, mode, prec):
    # d_v=128 group 32 and d_v=64 group 16/64 shapes, ragged tile counts
    d_v = 64 if fam == "mamba2" else 128
    group = {"gla": 32, "gdn": 16, "mamba2": 64}[fam]
    w = _small(fam, 3, 5, 128, d_v, group, mode, prec, steps=6)
    P.run_parity(w, w.steps, check_every=1)


@pytest.mark.parametrize("d_k,d_v,group", [(64, 64, 64), (64, 64, 16), (128, 64, 32),
                                           (64, 128, 16), (256, 128, 32), (32, 128, 32),
                                           (16, 64, 16), (192, 64, 64)])
def test_shapes(d_k, d_v, group):
    w = _small("gla", 2, 3, d_k, d_v, group, I.ROUND_SR, "mixed", steps=4)
    P.run_parity(w, w.steps, check_every=1)


@pytest.mark.parametrize("B,H", [(1, 1), (1, 7), (37, 3), (149, 8)])
def test_ragged_tile_counts(B, H):
    # tile counts that are not multiples of the warps per CTA or of the SM count
    w = _small("gdn", B, H, 128, 128, 32, I.ROUND_BDR, "mixed", steps=3)
    P.run_parity(w, w.steps, check_every=1)


@pytest.mark.parametrize("B,H", [(1, 1), (1, 7), (37, 3), (149, 8)])
def test_ragged_tile_counts_gated_sr(B, H):
    # the gated SR launch (a one-slot ring handed to the next copy after the
    # last pair's first loop) on tile counts below and between warp multiples
    w = _small("gla", B, H, 128, 128, 32, I.ROUND_SR, "mixed", steps=3)
    P.run_parity(w, w.steps, check_every=1)


def test_zero_batch_is_a_no_op():
    w = _small("gla", 0, 4, 64, 64, 32, I.ROUND_RTN, "int8", steps=1)
    st = lrs.lrs_state_alloc(P.make_shape(w), np.full(4, 8, np.uint8))
    try:
        e = torch.empty(16, device="cuda")
        lrs.lrs_decode_step(st, e, e, e, e, e, e, e, e, e, 0, 0, 0)
        lrs.lrs_sync()
    finally:
        lrs.lrs_state_free(st)


def test_zero_and_tiny_states():
    """A zero state with zero update stays exactly zero; magnitudes below the
    2^-100 threshold are stored as zero, on both sides."""
    w = _small("gla", 2, 2, 64, 64, 32, I.ROUND_SR, "mixed", steps=1, s0_std=0.0)
    pm = np.array([8, 4], np.uint8)
    pair = P.Pair(w, pm)
    try:
        S0 = torch.zeros(2, 2, 64, 64, device="cuda")
        S0[0, 0, :4, :4] = 2.0 ** -110
        S0[1, 1, :4, :4] = 2.0 ** -90
        pair.init(S0)
        pair.compare_state("import")
        x = {n: torch.zeros_like(t) for n, t in I.step_inputs(w, 0, device="cuda").items()
             if t is not None}
        x["gates"] = torch.ones_like(x["gates"])
        x["beta"] = None
        o_gpu, o_ref = pair.step(x, 0, 7)
        pair.compare_state("after zero step")
        assert not o_gpu.any() and not o_ref.any()
        assert not pair.gpu_codes()[0].any()
    finally:
        pair.free()


def test_large_magnitudes():
    w = _small("gla", 2, 4, 128, 128, 32, I.ROUND_BDR, "mixed", steps=3, s0_std=1e30)
    P.run_parity(w, w.steps, check_every=1)


def test_gla_rtn_int8_throughput_shape_sampled():
    w = W["gla_rtn_int8_b256h32_128"]
    P.run_parity(w, w.steps, tiles="sample")


def test_gdn_sr_int8_sampled_full_trajectory():
    w = W["gdn_sr_int8_b64h16_128"]
    P.run_parity(w, w.steps, tiles="sample")


def test_mamba2_mixed_sr_sampled_full_trajectory():
    w = W["mamba2_mixed_sr_b128h64"]
    P.run_parity(w, w.steps, tiles="sample")


@pytest.mark.parametrize("mode", [I.ROUND_BDR, I.ROUND_RTN])
def test_gla_int4_sampled_full_trajectory(mode):
    w = W["gla_bdr_int4_b256h32_128"]
    P.run_parity(w, w.steps, tiles="sample", mode=mode)


@pytest.mark.parametrize("batch", [64, 256, 1024])
def test_gdn_mixed_sr_sweep_sampled(batch):
    w = W["gdn_mixed_sr_h32_128"].with_batch(batch)
    P.run_parity(w, w.steps, tiles="sample")


def test_fp32_state_kernel_matches_oracle():
    for fam, d_v in (("gla", 128), ("gdn", 128), ("mamba2", 64)):
        w = _small(fam, 5, 3, 128, d_v, 32, I.ROUND_RTN, "int8", steps=5)
        S = I.initial_state(w, device="cuda").contiguous()
        S_ref = S.cpu().numpy().reshape(-1, w.d_k, w.d_v).copy()
        out = torch.empty(w.batch, w.heads, w.d_v, device="cuda")
        shp = P.make_shape(w)
        for t in range(w.steps):
            x = I.step_inputs(w, t, device="cuda")
            lrs.lrs_fp32_decode_step(shp, S, x["q"], x["k"], x["v"], x["gates"], x["beta"], out)
            n = w.batch * w.heads
            c = lambda a: None if a is None else a.cpu().numpy().reshape(n, -1)
            o_ref = oracle.fp32_step(S_ref, c(x["q"]), c(x["k"]), c(x["v"]), c(x["gates"]),
                                     None if x["beta"] is None else c(x["beta"]).reshape(n),
                                     update_kind=w.update_kind, gate_kind=w.gate_kind)
            np.testing.assert_array_equal(out.cpu().numpy().reshape(n, -1), o_ref)
            np.testing.assert_array_equal(S.cpu().numpy().reshape(n, w.d_k, w.d_v), S_ref)


HAND = ["hand_gla_int8_rtn_4x2.txt", "hand_gla_int8_bdr_2x2.txt", "hand_gdn_int4_rtn_2x2.txt",
        "hand_gla_int8_ties_2x2.txt", "hand_clamp_int8_1x2.txt",
        "hand_exact_product_int8_2x2.txt", "hand_bdr_zero_move_int8_2x2.txt"]


@pytest.mark.parametrize("name", HAND)
@pytest.mark.parametrize("mode", [I.ROUND_RTN, I.ROUND_SR, I.ROUND_BDR])
def test_hand_fixtures_on_gpu(name, mode):
    """The hand-derived steps, embedded in a 16-row-group, 64-column tile
    (each fixture group in its own 16-row group, other rows and columns zero):
    the GPU matches the oracle on the embedded problem, and the fixture's own
    codes where it states them (RTN, BDR)."""
    from tests.conftest import read_fixture
    fx = read_fixture(name)
    dk, dv, grp = (int(fx[k][0]) for k in ("d_k", "d_v", "group"))
    bits = int(fx["bits"][0])
    G = dk // grp
    DK, DV = 16 * G, 64
    rows = np.array([(i // grp) * 16 + i % grp for i in range(dk)])
    delta = fx["update"][0] == "delta"
    perkey = fx["gate"][0] == "per_key"
    codes = np.zeros((1, 1, DK, DV), np.int8)
    codes[0, 0, rows[:, None], np.arange(dv)[None, :]] = \
        np.array([int(c) for c in fx["codes_old"]]).reshape(dk, dv)
    scales = np.zeros((1, 1, G, DV), np.float32)
    scales[0, 0, :, :dv] = np.array([float(c) for c in fx["scales_old"]]).reshape(G, dv)
    emb = lambda key, n, fill=0.0: _embed(fx, key, n, rows, fill)
    q, k = emb("q", DK), emb("k", DK)
    v = np.zeros(DV, np.float32)
    v[:dv] = [float(c) for c in fx["v"]]
    gates = emb("gates", DK, 1.0) if perkey else np.array([float(fx["gates"][0])], np.float32)
    beta = np.array([float(fx["beta"][0])], np.float32) if delta else None
    shp = lrs.shape(1, 1, DK, DV, 16, 1 if delta else 0, 1 if perkey else 0)
    pm = np.array([bits], np.uint8)
    st = lrs.lrs_state_alloc(shp, pm)
    try:
        lrs.lrs_state_import_codes(st, torch.from_numpy(codes).cuda(),
                                   torch.from_numpy(scales).cuda())
        out = torch.empty(1, 1, DV, device="cuda")
        t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()
        lrs.lrs_decode_step(st, st.state_codes, st.scales, st.prec_map, t(q), t(k), t(v),
                            t(gates), t(beta), out, 7, 3, mode)
        lrs.lrs_sync()
        got = torch.empty(1, 1, DK, DV, dtype=torch.int8, device="cuda")
        lrs.lrs_state_export_codes(st, got)
        lrs.lrs_sync()
        got = got.cpu().numpy()[0, 0]
        rc, rs = codes[0].copy(), scales[0].copy()
        ro = oracle.step(rc, rs, q[None], k[None], v[None], gates[None], beta, pm, [0], [0],
                         group=16, update_kind=1 if delta else 0, gate_kind=1 if perkey else 0,
                         mode=mode, seed=7, step=3)
        np.testing.assert_array_equal(got, rc[0])
        np.testing.assert_array_equal(out.cpu().numpy()[0, 0], ro[0])
        key = {I.ROUND_RTN: "codes_rtn", I.ROUND_BDR: "codes_bdr"}.get(mode)
        if key in fx:
            expect = np.array([int(c) for c in fx[key]]).reshape(dk, dv)
            np.testing.assert_array_equal(got[rows[:, None], np.arange(dv)[None, :]], expect)
            np.testing.assert_array_equal(out.cpu().numpy()[0, 0, :dv],
                                          np.array([float(c) for c in fx["out"]], np.float32))
    finally:
        lrs.lrs_state_free(st)


def _embed(fx, key, n, rows, fill):
    a = np.full(n, fill, np.float32)
    a[rows] = [float(c) for c in fx[key]]
    return a


_U64 = np.uint64


def _splitmix64(z):
    z = z + _U64(0x9E3779B97F4A7C15)
    z = (z ^ (z >> _U64(30))) * _U64(0xBF58476D1CE4E5B9)
    z = (z ^ (z >> _U64(27))) * _U64(0x94D049BB133111EB)
    return z ^ (z >> _U64(31))


def _column_varying_carry_seed(B, H, d_v, step):
    """The first seed for which some tile's hash key k2 = m(m(m(seed) ^ step)
    ^ (b<<32 | h)) has a low half whose sum with the golden gamma's low half
    carries for some value columns j < d_v and not for others (about one tile
    in 2^32 / d_v)."""
    bh = ((np.arange(B, dtype=np.uint64)[:, None] << _U64(32)) |
          np.arange(H, dtype=np.uint64)[None, :]).reshape(-1)
    wrap = (1 << 32) - 0x7F4A7C15
    for s0 in range(0, 1 << 22, 4096):
        seeds = np.arange(s0, s0 + 4096, dtype=np.uint64)
        k1 = _splitmix64(_splitmix64(seeds) ^ _U64(step))
        lo = _splitmix64(k1[:, None] ^ bh[None, :]) & _U64(0xFFFFFFFF)
        kmin, kmax = lo & _U64(~(d_v - 1) & 0xFFFFFFFF), lo | _U64(d_v - 1)
        hit = np.argwhere((kmin < wrap) & (kmax >= wrap))
        if len(hit):
            si, t = hit[0]
            seed = int(seeds[si])
            # the chain, recomputed by the oracle's SplitMix64
            k = oracle.splitmix64(oracle.splitmix64(oracle.splitmix64(seed) ^ step) ^
                                  int(bh[t]))
            assert (k & 0xFFFFFFFF) == int(lo[si, t])
            return seed, int(t)
    raise AssertionError("no seed found")


@pytest.mark.parametrize("d_v,prec", [(128, "int8"), (64, "int4")])
def test_sr_tile_whose_hash_carry_varies_across_columns(d_v, prec):
    # The kernel draws most tiles' numbers from a per-row table that assumes
    # the same carry in every column; a tile where it differs takes the whole
    # per-element hash. Find such a tile and compare the step with the oracle.
    w = _small("gla", 64, 16, 128, d_v, 32, I.ROUND_SR, prec, steps=1)
    step = 5
    seed, tile = _column_varying_carry_seed(w.batch, w.heads, d_v, step)
    pm = np.full(w.heads, 8 if prec == "int8" else 4, np.uint8)
    pair = P.Pair(w, pm)
    try:
        pair.init(I.initial_state(w, device="cuda"))
        x = I.step_inputs(w, 0, device="cuda")
        o_gpu, o_ref = pair.step(x, step, seed)
        P.check_out(o_gpu, o_ref, "carry tile %d" % tile)
        pair.compare_state("carry tile %d" % tile)
    finally:
        pair.free()

