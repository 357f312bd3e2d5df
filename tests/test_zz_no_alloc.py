"""The allocation-free host-buffer step (lrs_decode_step_host_noalloc).

Callers that must not allocate device memory when they step -- a process
whose device memory belongs to another allocator or to a fixed pool sized at
start-up, or a latency-critical path that cannot pay for a cudaMalloc --
use this entry point; its scratch is a static array in the library. This test
runs it through the C ABI next to the allocating entry point
(lrs_decode_step_host) on two states with the same start, for two calls in a
row, and requires identical outputs and states (the same bit-exact bar as the
other parity tests): round to nearest, stochastic rounding and BDR, per-head
and per-(head, scale group) widths, the gated and the delta-rule update. It
sits in a file pytest collects last and works both alone in a fresh process
and after the other tests.
"""
import numpy as np
import pytest
import torch

from quantized_recurrent_state_decode_b200 import inputs as I
from quantized_recurrent_state_decode_b200 import lrs

pytestmark = pytest.mark.gpu


def _snapshot(st):
    raw = np.zeros(st.code_bytes, np.uint8)
    sc = np.zeros(st.scale_count, np.float32)
    lrs.lrs_state_copy_raw(st, raw, sc, True)
    return raw, sc


# per-(head, scale group) widths of the 4 heads x 4 groups states
PG = [[8, 4, 4, 8], [4, 4, 8, 8], [8, 8, 8, 4], [4, 8, 4, 4]]


@pytest.mark.parametrize("family,mode,pm,d_k", [
    ("gla", I.ROUND_RTN, [8, 8, 4, 4], 128),
    ("gdn", I.ROUND_SR, [8, 4, 8, 4], 128),
    ("gla", I.ROUND_BDR, [4, 8, 8, 4], 128),
    ("gdn", I.ROUND_BDR, [8, 4, 4, 8], 64),
    ("gla", I.ROUND_SR, PG, 128),
    ("gdn", I.ROUND_BDR, PG, 128),
])
def test_noalloc_step_matches_allocating_step(family, mode, pm, d_k):
    w = I.Workload("noalloc_" + family, family, 9, 4, d_k, 128, 32, 2, mode, "mixed",
                   s0_std=0.02, gate_mu=4.0 if family == "gdn" else -4.0, seed_id=95)
    pm = np.array(pm, np.uint8)
    shp = lrs.shape(w.batch, w.heads, w.d_k, w.d_v, w.group, w.update_kind, w.gate_kind)
    a = lrs.lrs_state_alloc(shp, pm)          # [H] or [H][G] widths
    b = lrs.lrs_state_alloc(shp, pm)
    try:
        S0 = I.initial_state(w, device="cuda")
        lrs.lrs_state_import_fp32(a, S0)
        lrs.lrs_state_import_fp32(b, S0)
        lrs.lrs_sync()
        out_a = torch.empty(w.batch, w.heads, w.d_v).pin_memory()
        out_b = torch.empty(w.batch, w.heads, w.d_v).pin_memory()
        err = torch.full((1,), 7, dtype=torch.int32).pin_memory()
        for t in range(2):            # two calls in a row
            x = {n: (None if v is None else v.pin_memory())
                 for n, v in I.step_inputs(w, t).items()}
            lrs.lrs_decode_step_host(a, x["q"], x["k"], x["v"], x["gates"], x["beta"], out_a,
                                     11, t, mode)
            lrs.lrs_decode_step_host_noalloc(b, x["q"], x["k"], x["v"], x["gates"], x["beta"],
                                             out_b, err, 11, t, mode)
            torch.cuda.synchronize()
            lrs.lrs_sync()
            assert int(err[0]) == 0
            assert torch.equal(out_a, out_b), "step %d outputs differ" % t
            assert out_b.abs().max() > 0
            ra, sa = _snapshot(a)
            rb, sb = _snapshot(b)
            np.testing.assert_array_equal(ra, rb)
            np.testing.assert_array_equal(sa, sb)
    finally:
        lrs.lrs_state_free(a)
        lrs.lrs_state_free(b)


def test_noalloc_rejects_a_step_beyond_the_static_scratch():
    # 512 x 32 tiles of 128x128 with per-key gates need about 40 MiB of staging
    shp = lrs.shape(512, 32, 128, 128, 32, lrs.LRS_UPDATE_GATED, lrs.LRS_GATE_PER_KEY)
    st = lrs.lrs_state_alloc(shp, np.full(32, 4, np.uint8))
    try:
        h = torch.zeros(16).pin_memory()
        with pytest.raises(lrs.LrsError) as e:
            lrs.lrs_decode_step_host_noalloc(st, h, h, h, h, None, h, None, 0, 0,
                                             lrs.LRS_ROUND_RTN)
        assert e.value.status == lrs.LRS_ERR_UNSUPPORTED
        assert "static scratch" in lrs.lrs_last_error()
    finally:
        lrs.lrs_state_free(st)
