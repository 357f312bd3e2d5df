"""GPU parity of the decode step with a Low-Rank Bypass buffer against the
oracle's orc_lrb_step: codes, scales, outputs and both buffer factors must be
bit-identical after every step, through several merges."""
import numpy as np
import pytest
import torch

import oracle
from quantized_recurrent_state_decode_b200 import inputs as I
from quantized_recurrent_state_decode_b200 import lrs
from tests import parity as P
from tests.test_gpu_parity import _small

pytestmark = pytest.mark.gpu


def run_lrb(w, rank, steps, tiles=None, mode=None, v_scale=None, pm=None):
    mode = w.mode if mode is None else mode
    pm = P.prec_map_for(w) if pm is None else pm
    if tiles == "sample":
        tiles = P.sample_tiles(w, pm)
    pair = P.Pair(w, pm, tiles=tiles, mode=mode)
    n = len(pair.tb)
    U = torch.zeros(w.batch, w.heads, rank, w.d_k, device="cuda")
    V = torch.zeros(w.batch, w.heads, rank, w.d_v, device="cuda")
    Ur = np.zeros((n, rank, w.d_k), np.float32)
    Vr = np.zeros((n, rank, w.d_v), np.float32)
    try:
        pair.init(I.initial_state(w, device="cuda"))
        seed = I.sr_seed(w)
        for t in range(steps):
            x = I.step_inputs(w, t, device="cuda")
            if v_scale is not None:
                x["v"] = x["v"] * v_scale
            lrs.lrs_lrb_step(pair.st, pair.st.state_codes, pair.st.scales, pair.st.prec_map, rank,
                             U, V, x["q"], x["k"], x["v"], x["gates"], x["beta"], pair.out, seed, t,
                             mode)
            lrs.lrs_sync()
            sel = lambda a: None if a is None else a[pair.tb_t, pair.th_t].cpu().numpy()
            o_ref = oracle.lrb_step(pair.codes, pair.scales, Ur, Vr, sel(x["q"]), sel(x["k"]),
                                    sel(x["v"]), sel(x["gates"]).reshape(n, -1), sel(x["beta"]),
                                    pm, pair.tb, pair.th, group=w.group,
                                    update_kind=w.update_kind, gate_kind=w.gate_kind, mode=mode,
                                    rank=rank, seed=seed, step=t)
            where = "%s rank %d step %d" % (w.name, rank, t)
            np.testing.assert_array_equal(sel(pair.out), o_ref, err_msg=where)
            np.testing.assert_array_equal(U[pair.tb_t, pair.th_t].cpu().numpy(), Ur, err_msg=where)
            np.testing.assert_array_equal(V[pair.tb_t, pair.th_t].cpu().numpy(), Vr, err_msg=where)
            pair.compare_state(where)
    finally:
        pair.free()


GRID = [(fam, mode) for fam in ("gla", "gdn", "mamba2")
        for mode in (I.ROUND_RTN, I.ROUND_SR, I.ROUND_BDR)]


@pytest.mark.parametrize("fam,mode", GRID)
@pytest.mark.parametrize("prec", ["int8", "mixed"])
@pytest.mark.parametrize("rank", [4, 6])
def test_lrb_family_mode_grid(fam, mode, prec, rank):
    """Ranks up to 4 run the streaming kernel, larger ones the one-CTA-per-tile
    kernel; both must match the oracle."""
    d_v = 64 if fam == "mamba2" else 128
    group = {"gla": 32, "gdn": 16, "mamba2": 64}[fam]
    w = _small(fam, 3, 5, 128, d_v, group, mode, prec, steps=rank + 3)
    run_lrb(w, rank=rank, steps=rank + 3)


@pytest.mark.parametrize("rank", [1, 2, 3, 8])
@pytest.mark.parametrize("mode", [I.ROUND_RTN, I.ROUND_SR])
def test_lrb_ranks(rank, mode):
    """Every rank through two merge cycles, on the register (RTN) and the
    staged (SR) pair code."""
    w = _small("gla", 2, 3, 128, 128, 32, mode, "mixed", steps=2 * rank + 1)
    run_lrb(w, rank=rank, steps=2 * rank + 1)


@pytest.mark.parametrize("d_k,d_v,group", [(64, 64, 16), (64, 128, 32), (128, 64, 32)])
def test_lrb_shapes(d_k, d_v, group):
    w = _small("gdn", 2, 3, d_k, d_v, group, I.ROUND_BDR, "mixed", steps=5)
    run_lrb(w, rank=2, steps=5)


def test_lrb_small_updates_merge():
    """Values scaled down so that most single updates are below half a step
    (the case the buffer exists for): merges must still match exactly."""
    w = _small("gla", 3, 4, 128, 128, 32, I.ROUND_RTN, "int8", steps=8, s0_std=1.0)
    run_lrb(w, rank=4, steps=8, v_scale=0.01)


def test_lrb_many_tiles_per_cta_sampled():
    w = I.WORKLOADS["gdn_mixed_sr_h32_128"].with_batch(64)
    run_lrb(w, rank=4, steps=5, tiles="sample")


@pytest.mark.parametrize("rank", [4, 6])
@pytest.mark.parametrize("fam,mode", [("gla", I.ROUND_RTN), ("gla", I.ROUND_BDR),
                                      ("gdn", I.ROUND_SR), ("mamba2", I.ROUND_SR)])
def test_lrb_group_widths(fam, mode, rank):
    """One width per (head, scale group): both bypass kernels (rank 4
    streaming, rank 6 one CTA per tile) against the oracle's per-group entry,
    through a merge."""
    d_v = 64 if fam == "mamba2" else 128
    w = _small(fam, 2, 5, 128, d_v, 32, mode, "mixed", steps=rank + 2)
    rng = np.random.default_rng(rank + 3 * mode)
    pm = rng.choice(np.array([4, 8], np.uint8), size=(w.heads, w.d_k // w.group))
    run_lrb(w, rank=rank, steps=rank + 2, pm=pm)


def test_lrb_rejects_bad_rank():
    w = _small("gla", 1, 2, 128, 128, 32, I.ROUND_RTN, "int8", steps=1)
    e = torch.zeros(1 << 16, device="cuda")
    st = lrs.lrs_state_alloc(P.make_shape(w), np.full(2, 8, np.uint8))
    try:
        for r in (0, 9):
            with pytest.raises(lrs.LrsError) as ei:
                lrs.lrs_lrb_step(st, st.state_codes, st.scales, st.prec_map, r, e, e, e, e, e, e,
                                 None, e, 0, 0, 0)
            assert ei.value.status == lrs.LRS_ERR_INVALID_ARG
    finally:
        lrs.lrs_state_free(st)


@pytest.mark.parametrize("name", ["gla_rtn_int8_b256h32_128", "mamba2_mixed_sr_b128h64",
                                  "gla_bdr_int4_b256h32_128"])
def test_lrb_full_size_workloads_sampled(name):
    """The full-size workloads through two merges (every tile updated, a spread
    sample compared, buffers included)."""
    run_lrb(I.WORKLOADS[name], rank=4, steps=8, tiles="sample")
