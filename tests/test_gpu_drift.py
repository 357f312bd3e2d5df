"""The output-drift series that bench.py reports for the int4 GLA workload
(RTN, BDR, SR and the rank-4 Low-Rank Bypass against the fp32-state kernel on
the same inputs), on a small batch.

The workload starts from S0 = 0, which fixes two values exactly: the first
step's output reads the unrounded x = k vᵀ in every quantized variant without
the bypass, so it equals the fp32 kernel's output bit for bit (e_1 = 0); and
BDR cannot reverse a first-step update (the old value is 0, so the move
c·s' has the sign of the update or is 0), so RTN and BDR hold the same codes
after step 1 and e_2 agrees between them.
"""
import math

import pytest

pytestmark = pytest.mark.gpu


def test_drift_series_small_batch():
    import torch

    import bench
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream()
    res = bench.run_drift(dev, stream, steps=16, batch=4)
    assert res["t"] == [1, 2, 4, 8, 16]
    names = ("rtn", "bdr", "sr", "lrb4_rtn", "lrb4_bdr")
    for n in names:
        assert len(res[n]) == 5
        assert all(math.isfinite(e) and 0.0 <= e < 1.0 for e in res[n]), (n, res[n])
    for n in ("rtn", "bdr", "sr"):
        assert res[n][0] == 0.0, (n, res[n])
    assert res["rtn"][1] == res["bdr"][1]
    # int4 requantization leaves a visible error once the state has been rounded
    assert res["rtn"][1] > 0.0 and res["sr"][1] > 0.0
    # S0 = 0: with the bypass the quantized part stays zero until the first
    # merge (after step `rank`, whose output is read before the merge), so up
    # to t = rank = 4 the output differs from the fp32 state's only by the
    # order of fp32 roundings
    for n in ("lrb4_rtn", "lrb4_bdr"):
        assert max(res[n][:3]) <= 1e-6, (n, res[n])
        assert res[n][3] > 1e-3, (n, res[n])        # merged and rounded from t = 8 on
