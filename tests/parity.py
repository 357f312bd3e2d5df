"""Parity harness: runs the CUDA path (through the C ABI) and the CPU oracle
on the same seeded inputs and compares them element by element.

Both sides evolve their own state from the same initial state (free running);
no oracle input is taken from the CUDA path. The comparison rules:
  - codes bit-identical, except at elements whose pre-rounding value lies
    within 1e-5 relative of a rounding boundary, where +-1 is allowed on at
    most 0.01% of the elements;
  - scales within 1e-6 relative;
  - outputs within max |diff| <= 1e-3 * max |o| per step.
"""
import numpy as np
import torch

import oracle
from quantized_recurrent_state_decode_b200 import inputs as I
from quantized_recurrent_state_decode_b200 import lrs

CODE_BOUNDARY_REL = 1e-5
CODE_MISMATCH_FRAC = 1e-4
SCALE_REL = 1e-6
OUT_REL = 1e-3


def prec_map_for(w, device="cuda", steps=None):
    """Precision map: uniform for int8/int4 workloads; for mixed ones the
    library's decay means and ranking, checked against the oracle's."""
    pm = I.uniform_prec_map(w)
    if pm is not None:
        return pm.numpy()
    decay = I.decay_tensor(w, steps=steps, device=device)        # [T*B][H][inner]
    outer, H, inner = decay.shape
    means = torch.zeros(H, dtype=torch.float64, device=device)
    lrs.lrs_decay_head_means(decay, outer, H, inner, means)
    torch.cuda.synchronize()
    pm = lrs.lrs_precision_map(means.cpu().numpy(), I.n_int8_heads(w))
    ref_means = oracle.decay_means(decay.cpu().numpy())
    np.testing.assert_allclose(means.cpu().numpy(), ref_means, rtol=1e-12)
    np.testing.assert_array_equal(pm, oracle.precision_map(ref_means, I.n_int8_heads(w)))
    return pm


def group_prec_map_for(w, device="cuda", steps=None):
    """Per-(head, scale group) widths: the mean decay of each block of `group`
    key channels ranked over all H*G blocks (library and oracle must agree),
    the top int8_fraction of blocks int8. For scalar decays every block of a
    head has the head's mean, so ties order the blocks by index."""
    G = w.d_k // w.group
    decay = I.decay_tensor(w, steps=steps, device=device)        # [T*B][H][inner]
    outer, H, inner = decay.shape
    if inner == w.d_k:
        blocks = decay.reshape(outer, H * G, w.group)
    else:                                                        # one decay per head
        blocks = decay.expand(outer, H, w.d_k).reshape(outer, H * G, w.group).contiguous()
    means = torch.zeros(H * G, dtype=torch.float64, device=device)
    lrs.lrs_decay_head_means(blocks, outer, H * G, w.group, means)
    torch.cuda.synchronize()
    n8 = int(round(w.int8_fraction * H * G))
    pm = lrs.lrs_precision_map(means.cpu().numpy(), n8)
    ref_means = oracle.decay_means(blocks.cpu().numpy())
    np.testing.assert_allclose(means.cpu().numpy(), ref_means, rtol=1e-12)
    np.testing.assert_array_equal(pm, oracle.precision_map(ref_means, n8))
    return pm.reshape(H, G)


def make_shape(w, batch=None):
    return lrs.shape(w.batch if batch is None else batch, w.heads, w.d_k, w.d_v, w.group,
                     w.update_kind, w.gate_kind)


def sample_tiles(w, pm, n_b=8, n_h=8):
    """Tiles spread over batch rows and heads, both precisions when mixed,
    always including the first and last tile."""
    bs = np.unique(np.linspace(0, w.batch - 1, min(n_b, w.batch)).round().astype(int))
    pm = np.asarray(pm).reshape(w.heads, -1)          # [H] or [H][G] widths
    heads8 = [h for h in range(w.heads) if (pm[h] == 8).all()]
    heads4 = [h for h in range(w.heads) if not (pm[h] == 8).all()]
    hs = []
    for group in (heads8, heads4):
        if group:
            k = max(1, n_h // (2 if heads8 and heads4 else 1))
            idx = np.unique(np.linspace(0, len(group) - 1, min(k, len(group))).round().astype(int))
            hs += [group[i] for i in idx]
    hs = sorted(set(hs) | {0, w.heads - 1})
    tb = np.array([b for b in bs for h in hs], np.int32)
    th = np.array([h for b in bs for h in hs], np.int32)
    return tb, th


class Pair:
    """A GPU state and the oracle's copy of selected tiles."""

    def __init__(self, w, pm, tiles=None, mode=None, device="cuda", io="f32"):
        self.w, self.pm, self.device = w, np.asarray(pm, np.uint8), device
        self.io = io
        self.mode = w.mode if mode is None else mode
        self.shape = make_shape(w)
        self.st = lrs.lrs_state_alloc(self.shape, self.pm)
        self.codes_buf = torch.empty(w.batch, w.heads, w.d_k, w.d_v, dtype=torch.int8,
                                     device=device)
        if tiles is None:
            tb = np.repeat(np.arange(w.batch, dtype=np.int32), w.heads)
            th = np.tile(np.arange(w.heads, dtype=np.int32), w.batch)
        else:
            tb, th = tiles
        self.tb, self.th = tb, th
        self.tb_t = torch.as_tensor(tb, dtype=torch.long, device=device)
        self.th_t = torch.as_tensor(th, dtype=torch.long, device=device)
        self.G = w.d_k // w.group
        self.prec_dev = torch.as_tensor(self.pm, device=device)
        self.out = torch.empty(w.batch, w.heads, w.d_v, device=device,
                               dtype=torch.bfloat16 if io == "bf16" else torch.float32)

    def free(self):
        lrs.lrs_state_free(self.st)

    def init(self, S0):
        """Import S0 (device tensor [B][H][d_k][d_v]) on both sides."""
        lrs.lrs_state_import_fp32(self.st, S0)
        S0s = S0[self.tb_t, self.th_t].cpu().numpy()
        self.codes, self.scales = oracle.import_fp32(S0s, self.pm, self.th, group=self.w.group)
        lrs.lrs_sync()

    def gpu_codes(self):
        lrs.lrs_state_export_codes(self.st, self.codes_buf)
        return self.codes_buf[self.tb_t, self.th_t].cpu().numpy()

    def gpu_scales(self):
        n = self.w.batch * self.w.heads * self.G * self.w.d_v
        t = device_view(self.st.scales, n, "<f4").view(self.w.batch, self.w.heads, self.G,
                                                        self.w.d_v)
        return t[self.tb_t, self.th_t].cpu().numpy()

    def step(self, x, t, seed):
        """One step on both sides; returns (gpu_out, oracle_out) for the tiles."""
        w = self.w
        beta = x["beta"]
        if self.io == "bf16":
            # the inputs a bfloat16 model layer would pass: the seeded fp32
            # inputs rounded to bfloat16; the oracle gets the values they denote
            qkv = {n: x[n].to(torch.bfloat16) for n in ("q", "k", "v")}
            lrs.lrs_decode_step_bf16(self.st, self.st.state_codes, self.st.scales,
                                     self.st.prec_map, qkv["q"], qkv["k"], qkv["v"], x["gates"],
                                     beta, self.out, seed, t, self.mode)
            x = dict(x, **{n: qkv[n].float() for n in qkv})
        else:
            lrs.lrs_decode_step(self.st, self.st.state_codes, self.st.scales, self.st.prec_map,
                                x["q"], x["k"], x["v"], x["gates"], beta, self.out, seed, t,
                                self.mode)
        sel = lambda a: None if a is None else a[self.tb_t, self.th_t].cpu().numpy()
        gates = sel(x["gates"])
        o_ref = oracle.step(self.codes, self.scales, sel(x["q"]), sel(x["k"]), sel(x["v"]),
                            gates.reshape(len(self.tb), -1), sel(beta), self.pm, self.tb, self.th,
                            group=w.group, update_kind=w.update_kind, gate_kind=w.gate_kind,
                            mode=self.mode, seed=seed, step=t,
                            nthreads=oracle.default_threads())
        o_gpu = self.out[self.tb_t, self.th_t]
        lrs.lrs_sync()
        if self.io == "bf16":
            # bfloat16 outputs compared as bit patterns with the oracle's
            # nearest-even rounding of its fp32 output
            o_gpu = o_gpu.view(torch.int16).cpu().numpy().view(np.uint16)
            return o_gpu, oracle.bf16_rne(o_ref)
        return o_gpu.cpu().numpy(), o_ref

    def compare_state(self, where=""):
        check_codes(self.gpu_codes(), self.codes, where)
        check_scales(self.gpu_scales(), self.scales, where)


def device_view(ptr, n, typestr):
    """A tensor viewing n elements of library-owned device memory (no copy)."""
    class _View:
        pass
    v = _View()
    v.__cuda_array_interface__ = {"shape": (n,), "typestr": typestr,
                                  "data": (int(ptr), False), "version": 3}
    return torch.as_tensor(v, device="cuda")


def check_codes(gpu, ref, where=""):
    """Codes: the stated bar allows +-1 at near-boundary elements, but the
    kernel follows the oracle's operation order, so bit-identical codes are
    required here."""
    diff = gpu.astype(np.int16) - ref.astype(np.int16)
    bad = np.count_nonzero(diff)
    assert bad == 0, "%s: %d of %d codes differ (max |diff| %d) at %s" % (
        where, bad, diff.size, np.abs(diff).max(), np.argwhere(diff)[:4].tolist())


def check_scales(gpu, ref, where=""):
    rel = np.abs(gpu.astype(np.float64) - ref) / np.maximum(np.abs(ref), 1e-38)
    rel[(gpu == 0) & (ref == 0)] = 0
    assert rel.max() <= SCALE_REL, "%s: scale relative error %.3e" % (where, rel.max())
    assert np.array_equal(gpu.view(np.uint32), ref.view(np.uint32)), \
        "%s: scales within tolerance but not bit-identical" % where


def check_out(gpu, ref, where=""):
    scale = max(float(np.abs(ref).max()), 1e-30)
    err = float(np.abs(gpu.astype(np.float64) - ref).max())
    assert err <= OUT_REL * scale, "%s: out error %.3e vs max|o| %.3e" % (where, err, scale)
    assert np.array_equal(gpu, ref), "%s: out within tolerance (%.3e) but not bit-identical" % (
        where, err / scale)


def check_out_bf16(gpu, ref, where=""):
    """bfloat16 outputs: the same bit patterns (the fp32 o before the final
    rounding is exact, so its nearest bfloat16 is too)."""
    bad = np.count_nonzero(gpu != ref)
    assert bad == 0, "%s: %d of %d bfloat16 outputs differ, first at %s" % (
        where, bad, gpu.size, np.argwhere(gpu != ref)[:4].tolist())


def run_parity(w, steps, tiles=None, mode=None, check_every=None, device="cuda", stats=None,
               io="f32", pm=None):
    """Free-running parity over `steps` steps; full state compared at
    step 0 (import), 1, 2, steps//2 and steps (or every step if check_every=1)."""
    if pm is None:
        pm = prec_map_for(w, device=device)
    if tiles == "sample":
        tiles = sample_tiles(w, pm)
    pair = Pair(w, pm, tiles=tiles, mode=mode, device=device, io=io)
    try:
        pair.init(I.initial_state(w, device=device))
        pair.compare_state("import")
        checkpoints = {1, 2, max(1, steps // 2), steps}
        seed = I.sr_seed(w)
        exact_out = 0
        for t in range(steps):
            x = I.step_inputs(w, t, device=device)
            o_gpu, o_ref = pair.step(x, t, seed)
            if io == "bf16":
                check_out_bf16(o_gpu, o_ref, "%s step %d" % (w.name, t))
            else:
                check_out(o_gpu, o_ref, "%s step %d" % (w.name, t))
            exact_out += int(np.array_equal(o_gpu, o_ref))
            if check_every == 1 or (t + 1) in checkpoints:
                pair.compare_state("%s after step %d" % (w.name, t + 1))
        if stats is not None:
            stats["exact_out_steps"] = exact_out
            stats["tiles"] = len(pair.tb)
        return pair.gpu_codes(), pair.codes
    finally:
        pair.free()
