"""GPU tests of the state itself: the packed code layout, import/export,
checkpoint and resume, the host-buffer step, and the device error paths
(precision-map mismatch, timed-out waits) -- all through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from quantized_recurrent_state_decode_b200 import inputs as I
from quantized_recurrent_state_decode_b200 import lrs
from tests import parity as P

pytestmark = pytest.mark.gpu


def pack_tile_reference(codes, bits, group):
    """Packed bytes of one tile, written from the layout documented in lrs.h:
    lane t owns columns [t*C, t*C+C); its codes, ordered by scale group, column
    pair, key row, column within the pair, form a byte stream (offset binary;
    int4: byte n of each 32-bit word holds elements n and n+4) cut into
    16-byte units, unit u of lane t at (u*32+t)*16."""
    d_k, d_v = codes.shape
    C = d_v // 32
    tile = np.zeros(d_k * d_v * bits // 8, np.uint8)
    for t in range(32):
        elems = []
        for g in range(d_k // group):
            for p in range(C // 2):
                cols = codes[g * group:(g + 1) * group, t * C + 2 * p: t * C + 2 * p + 2]
                elems.append(cols.reshape(-1))
        elems = np.concatenate(elems).astype(np.int64)
        if bits == 8:
            stream = (elems + 128).astype(np.uint8)
        else:
            e = (elems + 8).reshape(-1, 8)
            stream = (e[:, :4] | (e[:, 4:] << 4)).astype(np.uint8).reshape(-1)
        units = stream.reshape(-1, 16)
        for u in range(units.shape[0]):
            tile[(u * 32 + t) * 16:(u * 32 + t + 1) * 16] = units[u]
    return tile


def _state(B, H, d_k, d_v, group, pm, upd=0, gate=1):
    shp = lrs.shape(B, H, d_k, d_v, group, upd, gate)
    return shp, lrs.lrs_state_alloc(shp, np.asarray(pm, np.uint8))


@pytest.mark.parametrize("d_k,d_v,group", [(128, 128, 32), (64, 64, 16), (128, 64, 64)])
def test_packed_layout_and_code_round_trip(d_k, d_v, group):
    pm = np.array([8, 4, 4, 8, 4], np.uint8)
    B, H = 3, len(pm)
    shp, st = _state(B, H, d_k, d_v, group, pm)
    try:
        rng = np.random.default_rng(d_k + d_v)
        qmax = np.where(pm == 8, 127, 7)[None, :, None, None]
        codes = rng.integers(-128, 128, (B, H, d_k, d_v)).clip(-qmax, qmax).astype(np.int8)
        scales = rng.random((B, H, d_k // group, d_v)).astype(np.float32)
        lrs.lrs_state_import_codes(st, torch.from_numpy(codes).cuda(),
                                   torch.from_numpy(scales).cuda())
        lrs.lrs_sync()
        raw = np.zeros(st.code_bytes, np.uint8)
        sc = np.zeros(st.scale_count, np.float32)
        lrs.lrs_state_copy_raw(st, raw, sc, True)
        np.testing.assert_array_equal(sc, scales.reshape(-1))
        offs, stride, _ = lrs.lrs_layout_query(shp, pm)
        for b in range(B):
            for h in range(H):
                n = d_k * d_v * int(pm[h]) // 8
                got = raw[b * stride + offs[h]: b * stride + offs[h] + n]
                np.testing.assert_array_equal(got, pack_tile_reference(codes[b, h], int(pm[h]),
                                                                          group))
        back = torch.empty(B, H, d_k, d_v, dtype=torch.int8, device="cuda")
        lrs.lrs_state_export_codes(st, back)
        np.testing.assert_array_equal(back.cpu().numpy(), codes)
        S = torch.empty(B, H, d_k, d_v, device="cuda")
        lrs.lrs_state_export_fp32(st, S)
        np.testing.assert_array_equal(S.cpu().numpy().reshape(-1, d_k, d_v),
                                      oracle.dequant(codes.reshape(-1, d_k, d_v),
                                                     scales.reshape(-1, d_k // group, d_v),
                                                     group=group))
    finally:
        lrs.lrs_state_free(st)


def test_every_nibble_value_in_every_position():
    pm = np.array([4], np.uint8)
    shp, st = _state(1, 1, 64, 64, 16, pm)
    try:
        codes = np.zeros((1, 1, 64, 64), np.int8)
        vals = np.arange(-7, 8)
        for i in range(64):
            codes[0, 0, i] = np.roll(np.resize(vals, 64), i)
        lrs.lrs_state_import_codes(st, torch.from_numpy(codes).cuda(),
                                   torch.ones(1, 1, 4, 64, device="cuda"))
        back = torch.empty_like(torch.from_numpy(codes)).cuda()
        lrs.lrs_state_export_codes(st, back)
        lrs.lrs_sync()
        np.testing.assert_array_equal(back.cpu().numpy(), codes)
    finally:
        lrs.lrs_state_free(st)


def test_out_of_range_codes_are_clamped_and_reported():
    pm = np.array([4, 8], np.uint8)
    shp, st = _state(1, 2, 64, 64, 32, pm)
    try:
        codes = np.zeros((1, 2, 64, 64), np.int8)
        codes[0, 0, 0, 0] = 9
        codes[0, 1, 1, 1] = -128
        lrs.lrs_state_import_codes(st, torch.from_numpy(codes).cuda(),
                                   torch.ones(1, 2, 2, 64, device="cuda"))
        with pytest.raises(lrs.LrsError) as e:
            lrs.lrs_sync()
        assert e.value.status == lrs.LRS_ERR_DEVICE_RANGE
        back = torch.empty(1, 2, 64, 64, dtype=torch.int8, device="cuda")
        lrs.lrs_state_export_codes(st, back)
        lrs.lrs_sync()
        b = back.cpu().numpy()
        assert b[0, 0, 0, 0] == 7 and b[0, 1, 1, 1] == -127
    finally:
        lrs.lrs_state_free(st)


def _run(st, w, t0, t1, out, seed=3, codes=None, scales=None):
    for t in range(t0, t1):
        x = I.step_inputs(w, t, device="cuda")
        lrs.lrs_decode_step(st, codes or st.state_codes, scales or st.scales, st.prec_map,
                            x["q"], x["k"], x["v"], x["gates"], x["beta"], out, seed, t, w.mode)
    lrs.lrs_sync()


def _snapshot(st):
    raw = np.zeros(st.code_bytes, np.uint8)
    sc = np.zeros(st.scale_count, np.float32)
    lrs.lrs_state_copy_raw(st, raw, sc, True)
    return raw, sc


def test_checkpoint_and_resume_is_bit_exact():
    w = I.Workload("ckpt", "gdn", 6, 4, 128, 128, 32, 10, I.ROUND_SR, "mixed", s0_std=0.02,
                   gate_mu=4.0, seed_id=77)
    pm = np.array([8, 4, 8, 4], np.uint8)
    shp = P.make_shape(w)
    a = lrs.lrs_state_alloc(shp, pm)
    b = lrs.lrs_state_alloc(shp, pm)
    try:
        lrs.lrs_state_import_fp32(a, I.initial_state(w, device="cuda"))
        oa = torch.empty(w.batch, w.heads, w.d_v, device="cuda")
        ob = torch.empty_like(oa)
        _run(a, w, 0, 5, oa)
        raw, sc = _snapshot(a)
        lrs.lrs_state_copy_raw(b, raw, sc, False)
        _run(a, w, 5, 10, oa)
        _run(b, w, 5, 10, ob)
        assert torch.equal(oa, ob)
        ra, sa = _snapshot(a)
        rb, sb = _snapshot(b)
        np.testing.assert_array_equal(ra, rb)
        np.testing.assert_array_equal(sa, sb)
    finally:
        lrs.lrs_state_free(a)
        lrs.lrs_state_free(b)


def test_step_on_another_states_buffers():
    """One lrs_state describes the layout; the buffers of another state with
    the same shape and precision map (another layer) are stepped in place."""
    w = I.Workload("layers", "gla", 4, 4, 128, 128, 32, 3, I.ROUND_RTN, "mixed", s0_std=0.02,
                   gate_mu=-4.0, seed_id=78)
    pm = np.array([8, 8, 4, 4], np.uint8)
    shp = P.make_shape(w)
    a = lrs.lrs_state_alloc(shp, pm)
    b = lrs.lrs_state_alloc(shp, pm)
    c = lrs.lrs_state_alloc(shp, pm)
    try:
        S0 = I.initial_state(w, device="cuda")
        for s in (a, b, c):
            lrs.lrs_state_import_fp32(s, S0)
        o1 = torch.empty(w.batch, w.heads, w.d_v, device="cuda")
        o2 = torch.empty_like(o1)
        _run(b, w, 0, 3, o1)
        _run(a, w, 0, 3, o2, codes=c.state_codes, scales=c.scales)   # steps c through a
        assert torch.equal(o1, o2)
        np.testing.assert_array_equal(_snapshot(b)[0], _snapshot(c)[0])
        np.testing.assert_array_equal(_snapshot(b)[1], _snapshot(c)[1])
    finally:
        for s in (a, b, c):
            lrs.lrs_state_free(s)


def test_host_buffer_step_matches_device_step():
    w = I.Workload("host", "gdn", 5, 6, 128, 128, 32, 3, I.ROUND_SR, "mixed", s0_std=0.02,
                   gate_mu=4.0, seed_id=79)
    pm = np.array([8, 4, 8, 4, 8, 4], np.uint8)
    shp = P.make_shape(w)
    a = lrs.lrs_state_alloc(shp, pm)
    b = lrs.lrs_state_alloc(shp, pm)
    try:
        S0 = I.initial_state(w, device="cuda")
        lrs.lrs_state_import_fp32(a, S0)
        lrs.lrs_state_import_fp32(b, S0)
        out_d = torch.empty(w.batch, w.heads, w.d_v, device="cuda")
        out_h = torch.empty(w.batch, w.heads, w.d_v).pin_memory()
        for t in range(w.steps):
            x = I.step_inputs(w, t, device="cuda")
            lrs.lrs_decode_step(a, a.state_codes, a.scales, a.prec_map, x["q"], x["k"], x["v"],
                                x["gates"], x["beta"], out_d, 5, t, w.mode)
            xh = {n: (None if v is None else v.cpu().pin_memory()) for n, v in x.items()}
            lrs.lrs_decode_step_host(b, xh["q"], xh["k"], xh["v"], xh["gates"], xh["beta"],
                                     out_h, 5, t, w.mode)
            lrs.lrs_sync()
            assert torch.equal(out_d.cpu(), out_h)
        np.testing.assert_array_equal(_snapshot(a)[0], _snapshot(b)[0])
    finally:
        lrs.lrs_state_free(a)
        lrs.lrs_state_free(b)


def test_host_buffer_steps_back_to_back():
    """Consecutive host-buffer steps with no synchronization between them (the
    input copies of one step overlap the previous step): every step's output
    and the final state equal the device-buffer steps'."""
    w = I.Workload("host_pipe", "gla", 6, 5, 128, 128, 32, 7, I.ROUND_BDR, "mixed", s0_std=0.02,
                   gate_mu=-3.0, seed_id=81)
    pm = np.array([8, 4, 8, 4, 8], np.uint8)
    shp = P.make_shape(w)
    a = lrs.lrs_state_alloc(shp, pm)
    b = lrs.lrs_state_alloc(shp, pm)
    try:
        S0 = I.initial_state(w, device="cuda")
        lrs.lrs_state_import_fp32(a, S0)
        lrs.lrs_state_import_fp32(b, S0)
        xs = [I.step_inputs(w, t, device="cuda") for t in range(w.steps)]
        xh = [{n: (None if v is None else v.cpu().pin_memory()) for n, v in x.items()} for x in xs]
        outs_h = [torch.empty(w.batch, w.heads, w.d_v).pin_memory() for _ in range(w.steps)]
        torch.cuda.synchronize()
        for t in range(w.steps):
            x = xh[t]
            lrs.lrs_decode_step_host(b, x["q"], x["k"], x["v"], x["gates"], x["beta"], outs_h[t],
                                     5, t, w.mode)
        lrs.lrs_sync()
        out_d = torch.empty(w.batch, w.heads, w.d_v, device="cuda")
        for t in range(w.steps):
            x = xs[t]
            lrs.lrs_decode_step(a, a.state_codes, a.scales, a.prec_map, x["q"], x["k"], x["v"],
                                x["gates"], x["beta"], out_d, 5, t, w.mode)
            lrs.lrs_sync()
            assert torch.equal(out_d.cpu(), outs_h[t]), t
        np.testing.assert_array_equal(_snapshot(a)[0], _snapshot(b)[0])
        np.testing.assert_array_equal(_snapshot(a)[1], _snapshot(b)[1])
    finally:
        lrs.lrs_state_free(a)
        lrs.lrs_state_free(b)


def test_precision_map_mismatch_is_detected_and_skipped():
    w = I.Workload("mismatch", "gla", 4, 2, 128, 128, 32, 1, I.ROUND_RTN, "mixed", s0_std=0.02,
                   gate_mu=-4.0, seed_id=80)
    pm = np.array([8, 4], np.uint8)
    shp = P.make_shape(w)
    st = lrs.lrs_state_alloc(shp, pm)
    try:
        lrs.lrs_state_import_fp32(st, I.initial_state(w, device="cuda"))
        before = _snapshot(st)
        wrong = torch.tensor([8, 8], dtype=torch.uint8, device="cuda")
        x = I.step_inputs(w, 0, device="cuda")
        out = torch.empty(w.batch, w.heads, w.d_v, device="cuda")
        lrs.lrs_decode_step(st, st.state_codes, st.scales, wrong, x["q"], x["k"], x["v"],
                            x["gates"], None, out, 0, 0, w.mode)
        with pytest.raises(lrs.LrsError) as e:
            lrs.lrs_sync()
        assert e.value.status == lrs.LRS_ERR_DEVICE_LAYOUT
        after = _snapshot(st)
        _, stride, _ = lrs.lrs_layout_query(shp, pm)
        for b in range(w.batch):   # head 1 (int4, misdeclared as int8) untouched
            np.testing.assert_array_equal(after[0][b * stride + 16384:(b + 1) * stride],
                                          before[0][b * stride + 16384:(b + 1) * stride])
        lrs.lrs_sync()   # the error was consumed
    finally:
        lrs.lrs_state_free(st)


def test_timed_out_wait_reports_and_leaves_state_untouched():
    w = I.Workload("timeout", "gla", 8, 4, 128, 128, 32, 2, I.ROUND_RTN, "int8", s0_std=0.02,
                   gate_mu=-4.0, seed_id=81)
    pm = np.full(4, 8, np.uint8)
    pair = P.Pair(w, pm)
    try:
        pair.init(I.initial_state(w, device="cuda"))
        before = _snapshot(pair.st)
        x = I.step_inputs(w, 0, device="cuda")
        lrs.lrs_debug_inject_timeout(True, 2000)   # waits give up after 2 ms
        lrs.lrs_decode_step(pair.st, pair.st.state_codes, pair.st.scales, pair.st.prec_map,
                            x["q"], x["k"], x["v"], x["gates"], None, pair.out, 0, 0, w.mode)
        with pytest.raises(lrs.LrsError) as e:
            lrs.lrs_sync()
        assert e.value.status == lrs.LRS_ERR_DEVICE_TIMEOUT
        after = _snapshot(pair.st)
        np.testing.assert_array_equal(before[0], after[0])
        np.testing.assert_array_equal(before[1], after[1])
        # the context is still usable and the next step is exact
        o_gpu, o_ref = pair.step(x, 0, 0)
        P.check_out(o_gpu, o_ref, "after timeout")
        pair.compare_state("after timeout")
    finally:
        pair.free()


def test_timeout_on_a_later_group_leaves_a_partial_tile_and_checkpoint_restores():
    # Each warp copies in only its first (tile, group) item, so its wait for
    # the second one runs out after the first group of its first tile was
    # written: the documented partial state. Restoring the checkpoint makes
    # the next step exact again.
    w = I.Workload("timeout_after", "gla", 8, 4, 128, 128, 32, 2, I.ROUND_RTN, "int8",
                   s0_std=0.02, gate_mu=-4.0, seed_id=82)
    pm = np.full(4, 8, np.uint8)
    pair = P.Pair(w, pm)
    G = w.d_k // w.group
    gbytes = w.group * w.d_v                  # one int8 group block of a tile
    try:
        pair.init(I.initial_state(w, device="cuda"))
        raw0, sc0 = _snapshot(pair.st)
        x = I.step_inputs(w, 0, device="cuda")
        lrs.lrs_debug_inject_timeout_after(1, 2000)      # waits give up after 2 ms
        lrs.lrs_decode_step(pair.st, pair.st.state_codes, pair.st.scales, pair.st.prec_map,
                            x["q"], x["k"], x["v"], x["gates"], None, pair.out, 0, 0, w.mode)
        with pytest.raises(lrs.LrsError) as e:
            lrs.lrs_sync()
        assert e.value.status == lrs.LRS_ERR_DEVICE_TIMEOUT
        raw1, sc1 = _snapshot(pair.st)
        s0 = sc0.reshape(w.batch * w.heads, G, w.d_v)
        s1 = sc1.reshape(w.batch * w.heads, G, w.d_v)
        c0 = raw0.reshape(w.batch * w.heads, G, gbytes)
        c1 = raw1.reshape(w.batch * w.heads, G, gbytes)
        # 32 tiles, one per warp: every tile got its first group and no other
        np.testing.assert_array_equal(s1[:, 1:], s0[:, 1:])
        np.testing.assert_array_equal(c1[:, 1:], c0[:, 1:])
        assert not np.array_equal(s1[:, 0], s0[:, 0])
        assert not np.array_equal(c1[:, 0], c0[:, 0])
        # restore the checkpoint; the context works and the step is exact
        lrs.lrs_state_copy_raw(pair.st, raw0, sc0, False)
        o_gpu, o_ref = pair.step(x, 0, 0)
        P.check_out(o_gpu, o_ref, "after restore")
        pair.compare_state("after restore")
    finally:
        lrs.lrs_debug_inject_timeout_after(-1, 0)
        pair.free()


def test_decay_means_and_precision_map_match_oracle():
    for name in ("mamba2_mixed_sr_b128h64", "gdn_mixed_sr_h32_128"):
        w = I.WORKLOADS[name]
        pm = P.prec_map_for(w, steps=32)
        assert int((pm == 8).sum()) == I.n_int8_heads(w)
