"""GPU parity with per-channel precision: one code width per (head, scale
group), the state's tiles mixing int8 and int4 groups, against the oracle's
per-group entry points."""
import numpy as np
import pytest
import torch

from quantized_recurrent_state_decode_b200 import inputs as I
from quantized_recurrent_state_decode_b200 import lrs
from tests import parity as P
from tests.test_gpu_chunk import run_chunks
from tests.test_gpu_parity import _small

pytestmark = pytest.mark.gpu


def _random_map(w, seed):
    rng = np.random.default_rng(seed)
    return rng.choice(np.array([4, 8], np.uint8), size=(w.heads, w.d_k // w.group))


@pytest.mark.parametrize("fam", ["gla", "gdn", "mamba2"])
@pytest.mark.parametrize("mode", [I.ROUND_RTN, I.ROUND_SR, I.ROUND_BDR])
def test_random_group_widths(fam, mode):
    d_v = 64 if fam == "mamba2" else 128
    group = {"gla": 32, "gdn": 16, "mamba2": 32}[fam]
    w = _small(fam, 3, 5, 128, d_v, group, mode, "mixed", steps=4)
    P.run_parity(w, w.steps, check_every=1, pm=_random_map(w, 7 + mode))


@pytest.mark.parametrize("d_k,d_v,group", [(64, 64, 16), (256, 128, 32), (192, 64, 64)])
def test_group_widths_shapes(d_k, d_v, group):
    w = _small("gla", 2, 3, d_k, d_v, group, I.ROUND_SR, "mixed", steps=3)
    P.run_parity(w, w.steps, check_every=1, pm=_random_map(w, d_k))


def test_decay_ranked_group_map_gla_sampled():
    """GLA's decay is per key channel: rank the (head, group) blocks by their
    mean decay, half of them int8, and run the throughput shape."""
    w = I.WORKLOADS["gla_rtn_int8_b256h32_128"]
    w = I.Workload(**{**w.__dict__, "precision": "mixed", "int8_fraction": 0.5,
                      "name": "gla_group_mixed_b256h32"})
    pm = P.group_prec_map_for(w, steps=8)
    assert 0 < (pm == 8).sum() < pm.size
    P.run_parity(w, 8, tiles="sample", pm=pm)


def test_bf16_io_with_group_widths():
    w = _small("gla", 3, 4, 128, 128, 32, I.ROUND_BDR, "mixed", steps=3)
    P.run_parity(w, w.steps, check_every=1, pm=_random_map(w, 3), io="bf16")


def test_uniform_group_map_has_the_head_layout():
    """Every group at its head's width: the same bytes and offsets as the
    per-head state after the same steps."""
    w = _small("gdn", 2, 4, 128, 128, 32, I.ROUND_SR, "mixed", steps=3)
    pm_h = np.array([8, 4, 4, 8], np.uint8)
    pm_g = np.repeat(pm_h[:, None], 4, axis=1)
    shp = P.make_shape(w)
    a, b = lrs.lrs_state_alloc(shp, pm_h), lrs.lrs_state_alloc(shp, pm_g)
    try:
        assert a.batch_stride_bytes == b.batch_stride_bytes
        S0 = I.initial_state(w, device="cuda")
        out = torch.empty(w.batch, w.heads, w.d_v, device="cuda")
        for st in (a, b):
            lrs.lrs_state_import_fp32(st, S0)
            for t in range(w.steps):
                x = I.step_inputs(w, t, device="cuda")
                lrs.lrs_decode_step(st, st.state_codes, st.scales, st.prec_map, x["q"], x["k"],
                                    x["v"], x["gates"], x["beta"], out, 9, t, w.mode)
        lrs.lrs_sync()
        raw = []
        for st in (a, b):
            c = np.zeros(st.code_bytes, np.uint8)
            sc = np.zeros(st.scale_count, np.float32)
            lrs.lrs_state_copy_raw(st, c, sc, True)
            lrs.lrs_sync()
            raw.append((c, sc))
        np.testing.assert_array_equal(raw[0][0], raw[1][0])
        np.testing.assert_array_equal(raw[0][1], raw[1][1])
    finally:
        lrs.lrs_state_free(a)
        lrs.lrs_state_free(b)


@pytest.mark.parametrize("fam", ["gla", "gdn"])
def test_chunk_with_group_widths(fam):
    w = _small(fam, 3, 5, 128, 128, 32, I.ROUND_BDR, "mixed", steps=2)
    run_chunks(w, T=5, n_chunks=2, pm=_random_map(w, 21))


def test_decay_ranked_group_map_gdn_mixed_sampled():
    w = I.WORKLOADS["gdn_mixed_sr_h32_128"].with_batch(256)
    pm = P.group_prec_map_for(w, steps=8)
    assert 0 < (pm == 8).sum() < pm.size
    P.run_parity(w, 6, tiles="sample", pm=pm)
