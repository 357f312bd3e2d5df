"""Host-side parts of bench.py: the oracle sampler that both CPU legs time
(`--impl reference` and the GPU arm's `cpu_baseline`), and the reference
arm's JSON line. No GPU."""
import json
import subprocess
import sys

import numpy as np

import bench
import oracle
from quantized_recurrent_state_decode_b200 import inputs as I

ROOT = bench.ROOT


def test_sampler_slices_match_one_oracle_call():
    # The pool hands each thread a slice of the sample; the result must be
    # the same as one call over every sampled tile.
    w = I.WORKLOADS["gdn_mixed_sr_h32_128"].with_batch(2)
    smp = bench.OracleSampler(w, I.ROUND_SR, ntiles=24, seed=3)
    codes, scales = smp.codes.copy(), smp.scales.copy()
    x = smp.xs[0]
    oracle.step(codes, scales, x["q"], x["k"], x["v"], x["gates"], x["beta"].reshape(-1), smp.pm,
                smp.tb, smp.th, group=w.group, update_kind=w.update_kind, gate_kind=w.gate_kind,
                mode=I.ROUND_SR, seed=1, step=0, nthreads=1)
    el = smp.step(0)
    smp.close()
    assert el > 0
    np.testing.assert_array_equal(smp.codes, codes)
    np.testing.assert_array_equal(smp.scales.view(np.uint32), scales.view(np.uint32))
    assert 1 <= len(smp.slices) <= oracle.default_threads()
    assert sum(sl.stop - sl.start for sl in smp.slices) == smp.n == 24


def test_reference_arm_prints_one_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload",
                        "gla_rtn_int8_b2h2_64", "--steps", "2", "--warmup", "3"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "steps/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["workload"] == "gla_rtn_int8_b2h2_64"
