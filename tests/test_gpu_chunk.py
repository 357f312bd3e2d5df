"""GPU parity of the multi-token (chunked) update against the oracle's chunked
update: T tokens applied in fp32 and one requantization at the end, through
the C ABI. Codes, scales and every token's outputs must be bit-identical."""
import numpy as np
import pytest
import torch

import oracle
from quantized_recurrent_state_decode_b200 import inputs as I
from quantized_recurrent_state_decode_b200 import lrs
from tests import parity as P
from tests.test_gpu_parity import _small

pytestmark = pytest.mark.gpu


def run_chunks(w, T, n_chunks=1, tiles=None, mode=None, pm=None):
    mode = w.mode if mode is None else mode
    if pm is None:
        pm = P.prec_map_for(w)
    if tiles == "sample":
        tiles = P.sample_tiles(w, pm)
    pair = P.Pair(w, pm, tiles=tiles, mode=mode)
    n = len(pair.tb)
    try:
        pair.init(I.initial_state(w, device="cuda"))
        seed = I.sr_seed(w)
        out = torch.empty(T, w.batch, w.heads, w.d_v, device="cuda")
        for c in range(n_chunks):
            x = I.chunk_inputs(w, c * T, T, device="cuda")
            lrs.lrs_chunk_step(pair.st, pair.st.state_codes, pair.st.scales, pair.st.prec_map, T,
                               x["q"], x["k"], x["v"], x["gates"], x["beta"], out, seed, c, mode)
            lrs.lrs_sync()
            sel = lambda a: None if a is None else a[:, pair.tb_t, pair.th_t].cpu().numpy()
            g = sel(x["gates"]).reshape(T, n, -1)
            o_ref = oracle.chunk_step(pair.codes, pair.scales, sel(x["q"]), sel(x["k"]),
                                      sel(x["v"]), g, sel(x["beta"]), pm, pair.tb, pair.th,
                                      group=w.group, update_kind=w.update_kind,
                                      gate_kind=w.gate_kind, mode=mode, seed=seed, step=c,
                                      nthreads=oracle.default_threads())
            o_gpu = out[:, pair.tb_t, pair.th_t].cpu().numpy()
            np.testing.assert_array_equal(o_gpu, o_ref, err_msg="%s chunk %d" % (w.name, c))
            pair.compare_state("%s after chunk %d" % (w.name, c))
    finally:
        pair.free()


GRID = [(fam, mode, prec) for fam in ("gla", "gdn", "mamba2")
        for mode in (I.ROUND_RTN, I.ROUND_SR, I.ROUND_BDR) for prec in ("int8", "int4", "mixed")]


@pytest.mark.parametrize("fam,mode,prec", GRID)
def test_chunk_mode_family_precision_grid(fam, mode, prec):
    d_v = 64 if fam == "mamba2" else 128
    group = {"gla": 32, "gdn": 16, "mamba2": 64}[fam]
    w = _small(fam, 3, 5, 128, d_v, group, mode, prec, steps=4)
    run_chunks(w, T=11, n_chunks=2)      # more tokens than ring slots, not a multiple


@pytest.mark.parametrize("T", [1, 2, 8, 9])
def test_chunk_lengths(T):
    w = _small("gdn", 2, 3, 128, 128, 32, I.ROUND_SR, "mixed", steps=2)
    run_chunks(w, T=T, n_chunks=2)


@pytest.mark.parametrize("T", [1, 2, 3, 8, 9, 17])
@pytest.mark.parametrize("fam,mode", [("gla", I.ROUND_BDR), ("mamba2", I.ROUND_SR)])
def test_chunk_lengths_gated(fam, mode, T):
    """The gated forms' kernel skews its two row halves by one token: chunks
    of one token, of fewer tokens than ring slots, and of more."""
    d_v = 64 if fam == "mamba2" else 128
    w = _small(fam, 2, 3, 128, d_v, 32, mode, "mixed", steps=2)
    run_chunks(w, T=T, n_chunks=2)


@pytest.mark.parametrize("d_k,d_v,group", [(64, 64, 16), (64, 128, 32), (128, 64, 32),
                                           (64, 64, 64)])
def test_chunk_shapes(d_k, d_v, group):
    w = _small("gla", 2, 3, d_k, d_v, group, I.ROUND_BDR, "mixed", steps=2)
    run_chunks(w, T=5)


def test_chunk_of_one_token_matches_decode_step():
    """T = 1 is the decode step: same codes, scales and output as lrs_decode_step."""
    w = _small("gla", 4, 6, 128, 128, 32, I.ROUND_SR, "mixed", steps=1)
    pm = P.prec_map_for(w)
    a, b = P.Pair(w, pm), P.Pair(w, pm)
    try:
        S0 = I.initial_state(w, device="cuda")
        a.init(S0)
        b.init(S0)
        x = I.step_inputs(w, 0, device="cuda")
        xc = I.chunk_inputs(w, 0, 1, device="cuda")
        oa = torch.empty(w.batch, w.heads, w.d_v, device="cuda")
        ob = torch.empty(1, w.batch, w.heads, w.d_v, device="cuda")
        lrs.lrs_decode_step(a.st, a.st.state_codes, a.st.scales, a.st.prec_map, x["q"], x["k"],
                            x["v"], x["gates"], x["beta"], oa, 5, 3, w.mode)
        lrs.lrs_chunk_step(b.st, b.st.state_codes, b.st.scales, b.st.prec_map, 1, xc["q"],
                           xc["k"], xc["v"], xc["gates"], xc["beta"], ob, 5, 3, w.mode)
        lrs.lrs_sync()
        assert torch.equal(oa, ob[0])
        np.testing.assert_array_equal(a.gpu_codes(), b.gpu_codes())
        np.testing.assert_array_equal(a.gpu_scales(), b.gpu_scales())
    finally:
        a.free()
        b.free()


def test_chunk_many_tiles_per_cta_sampled():
    """More tiles than resident CTAs: each CTA walks several tiles, the token
    ring's phases carry over from tile to tile."""
    w = I.WORKLOADS["gdn_mixed_sr_h32_128"].with_batch(64)
    run_chunks(w, T=6, n_chunks=2, tiles="sample")


def test_chunk_gla_throughput_shape_sampled():
    w = I.WORKLOADS["gla_rtn_int8_b256h32_128"]
    run_chunks(w, T=16, tiles="sample")


def test_chunk_zero_tokens_is_a_no_op_and_bad_shapes_rejected():
    w = _small("gla", 2, 2, 128, 128, 32, I.ROUND_RTN, "int8", steps=1)
    pm = P.prec_map_for(w)
    pair = P.Pair(w, pm)
    try:
        pair.init(I.initial_state(w, device="cuda"))
        c0 = pair.gpu_codes().copy()
        e = torch.empty(64, device="cuda")
        lrs.lrs_chunk_step(pair.st, pair.st.state_codes, pair.st.scales, pair.st.prec_map, 0,
                           e, e, e, e, None, e, 0, 0, 0)
        lrs.lrs_sync()
        np.testing.assert_array_equal(pair.gpu_codes(), c0)
        with pytest.raises(lrs.LrsError) as ei:
            lrs.lrs_chunk_step(pair.st, pair.st.state_codes, pair.st.scales, pair.st.prec_map,
                               -1, e, e, e, e, None, e, 0, 0, 0)
        assert ei.value.status == lrs.LRS_ERR_INVALID_ARG
    finally:
        pair.free()
    w2 = _small("gla", 1, 1, 256, 128, 32, I.ROUND_RTN, "int8", steps=1)
    st = lrs.lrs_state_alloc(P.make_shape(w2), np.full(1, 8, np.uint8))
    try:
        e = torch.empty(1024, device="cuda")
        with pytest.raises(lrs.LrsError) as ei:
            lrs.lrs_chunk_step(st, st.state_codes, st.scales, st.prec_map, 2, e, e, e, e, None,
                               e, 0, 0, 0)
        assert ei.value.status == lrs.LRS_ERR_UNSUPPORTED
    finally:
        lrs.lrs_state_free(st)


def test_chunk_injected_timeout_reports_and_leaves_state():
    w = _small("gdn", 2, 2, 128, 128, 32, I.ROUND_RTN, "int8", steps=1)
    pm = P.prec_map_for(w)
    pair = P.Pair(w, pm)
    try:
        pair.init(I.initial_state(w, device="cuda"))
        c0 = pair.gpu_codes().copy()
        x = I.chunk_inputs(w, 0, 3, device="cuda")
        out = torch.empty(3, w.batch, w.heads, w.d_v, device="cuda")
        lrs.lrs_debug_inject_timeout(True, 2000)
        lrs.lrs_chunk_step(pair.st, pair.st.state_codes, pair.st.scales, pair.st.prec_map, 3,
                           x["q"], x["k"], x["v"], x["gates"], x["beta"], out, 0, 0, 0)
        with pytest.raises(lrs.LrsError) as ei:
            lrs.lrs_sync()
        assert ei.value.status == lrs.LRS_ERR_DEVICE_TIMEOUT
        np.testing.assert_array_equal(pair.gpu_codes(), c0)
        # the context stays usable
        lrs.lrs_chunk_step(pair.st, pair.st.state_codes, pair.st.scales, pair.st.prec_map, 3,
                           x["q"], x["k"], x["v"], x["gates"], x["beta"], out, 0, 0, 0)
        lrs.lrs_sync()
    finally:
        pair.free()


@pytest.mark.parametrize("name,T", [("mamba2_mixed_sr_b128h64", 8), ("gla_bdr_int4_b256h32_128", 8),
                                    ("gdn_sr_int8_b64h16_128", 8)])
def test_chunk_full_size_workloads_sampled(name, T):
    """The full-size workloads (every tile updated, a spread sample compared)."""
    run_chunks(I.WORKLOADS[name], T=T, n_chunks=2, tiles="sample")
