"""Output drift of the two readings of Bounded Directional Rounding, on the
CPU oracle.

"Preserving Updates in Low-Bit Recurrent State Quantization" (abstract) says
a requantized element can move opposite to its update and that BDR rounds
such elements toward the update. The library reads "its update" as the
element's whole change this step, x - deq (decay included); the other
reading is the additive term k_i w_j alone. This script runs the int4 GLA
workload's distributions (per-key decay exp(-softplus(N(-4, 1))), q, k, v
N(0, 1) with k L2-normalised, S0 = 0, group 32) at a small batch through
round to nearest, BDR as the library reads it, BDR with the additive update,
and the unquantized fp32 state, all on the same seeded inputs, and prints the
drift e_t = ||o_q - o_fp32||_2 / ||o_fp32||_2 over every (b, h, j) of step t
at t = 1, 2, 4, ... as one JSON line.

    python -m oracle.bdr_reading_study [--batch 8] [--steps 1024]

TEST INFRASTRUCTURE ONLY: it uses the oracle, not the library.
"""
import argparse
import concurrent.futures as cf
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from quantized_recurrent_state_decode_b200 import inputs as I  # noqa: E402


def run(batch=8, steps=1024, workload="gla_bdr_int4_b256h32_128"):
    w = I.WORKLOADS[workload].with_batch(batch)
    assert w.family == "gla" and w.precision == "int4"
    n = w.batch * w.heads
    qmax = 7
    pm = np.full(w.heads, 4, np.uint8)
    tb = np.repeat(np.arange(w.batch, dtype=np.int32), w.heads)
    th = np.tile(np.arange(w.heads, dtype=np.int32), w.batch)
    S0 = I.initial_state(w).numpy().reshape(n, w.d_k, w.d_v)
    S = S0.copy()
    st = {name: oracle.import_fp32(S0, pm, th, group=w.group) for name in ("rtn", "bdr",
                                                                          "bdr_additive")}
    threads = oracle.default_threads()
    slices = [slice(n * i // threads, n * (i + 1) // threads) for i in range(threads)]
    pool = cf.ThreadPoolExecutor(threads)
    samples = [1 << i for i in range(steps.bit_length()) if (1 << i) <= steps]
    series = {name: [] for name in st}
    for t in range(steps):
        x = {k: (None if v is None else v.numpy().reshape(n, -1)) for k, v in
             I.step_inputs(w, t).items()}
        o_f = oracle.fp32_step(S, x["q"], x["k"], x["v"], x["gates"], None, update_kind=0,
                               gate_kind=1, nthreads=threads)
        outs = {}
        for name, mode in (("rtn", oracle.ROUND_RTN), ("bdr", oracle.ROUND_BDR)):
            c, s = st[name]
            outs[name] = oracle.step(c, s, x["q"], x["k"], x["v"], x["gates"], None, pm, tb, th,
                                     group=w.group, update_kind=0, gate_kind=1, mode=mode,
                                     nthreads=threads)
        c, s = st["bdr_additive"]
        o = np.zeros((n, w.d_v), np.float32)

        def part(sl):
            o[sl] = oracle.bdr_additive_step(c[sl], s[sl], x["q"][sl], x["k"][sl], x["v"][sl],
                                             x["gates"][sl], group=w.group, qmax=qmax)
        list(pool.map(part, slices))
        outs["bdr_additive"] = o
        if t + 1 in samples:
            ref = np.linalg.norm(o_f.astype(np.float64))
            for name in st:
                series[name].append(float(np.linalg.norm(outs[name].astype(np.float64) -
                                                         o_f) / ref))
    pool.shutdown()
    return {"workload": w.name, "batch": w.batch, "heads": w.heads, "state": "int4",
            "group": w.group, "t": samples, "measure": "||o_q - o_fp32||_2 / ||o_fp32||_2",
            "readings": {"bdr": "update = x - deq (the library's)",
                         "bdr_additive": "update = k_i w_j"}, **series}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--batch", type=int, default=8)
    ap.add_argument("--steps", type=int, default=1024)
    a = ap.parse_args()
    print(json.dumps(run(a.batch, a.steps)))


if __name__ == "__main__":
    main()
