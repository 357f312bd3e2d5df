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
