"""GPU parity of the bfloat16-I/O decode step (q, k, v and out in bfloat16)
against the oracle run on the values the bfloat16 inputs denote, with its
fp32 output rounded to the nearest bfloat16 (ties to even)."""
import pytest

from quantized_recurrent_state_decode_b200 import inputs as I
from tests import parity as P
from tests.test_gpu_parity import _small

pytestmark = pytest.mark.gpu

GRID = [(fam, mode, prec) for fam in ("gla", "gdn", "mamba2")
        for mode in (I.ROUND_RTN, I.ROUND_SR, I.ROUND_BDR) for prec in ("int8", "int4", "mixed")]


@pytest.mark.parametrize("fam,mode,prec", GRID)
def test_bf16_mode_family_precision_grid(fam, mode, prec):
    d_v = 64 if fam == "mamba2" else 128
    group = {"gla": 32, "gdn": 16, "mamba2": 64}[fam]
    w = _small(fam, 3, 5, 128, d_v, group, mode, prec, steps=5)
    P.run_parity(w, w.steps, check_every=1, io="bf16")


@pytest.mark.parametrize("d_k,d_v,group", [(16, 64, 16), (256, 128, 32), (64, 64, 16)])
def test_bf16_shapes(d_k, d_v, group):
    w = _small("gdn", 2, 3, d_k, d_v, group, I.ROUND_SR, "mixed", steps=3)
    P.run_parity(w, w.steps, check_every=1, io="bf16")


def test_bf16_throughput_shape_sampled():
    w = I.WORKLOADS["gla_rtn_int8_b256h32_128"]
    P.run_parity(w, 16, tiles="sample", io="bf16")


def test_bf16_gdn_mixed_sr_sampled():
    w = I.WORKLOADS["gdn_mixed_sr_h32_128"].with_batch(256)
    P.run_parity(w, 16, tiles="sample", io="bf16")
