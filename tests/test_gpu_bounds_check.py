"""The bounds-checked debug build (liblrs_checked.so, LRS_BOUNDS_CHECK).

Its step kernel checks, before each access, that the tile's codes and scales,
each scale group's bulk copies (shared-memory slot and tile-input buffer, and
the global ranges they read), each column pair's units and scales, and the
output row lie inside their buffers; a failed check records
LRS_ERR_DEVICE_BOUNDS and skips the access (it never traps). Run in a child
process, which loads that build instead of liblrs.so:

- the small parity cases give the oracle's results exactly, with no error;
- a state whose declared code size is below what its tiles need (the buffer
  itself is full size, so nothing is touched out of range) makes the checks
  fire: LRS_ERR_DEVICE_BOUNDS.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import ctypes, sys
import numpy as np
sys.path.insert(0, ROOT)
from quantized_recurrent_state_decode_b200 import build as B, lrs
lrs.use_library(B.build_checked())
from quantized_recurrent_state_decode_b200 import inputs as I
from tests import parity as P
from tests.test_gpu_parity import _small

cases = [_small("gla", 3, 5, 128, 128, 32, I.ROUND_RTN, "mixed", steps=3),
         _small("gdn", 3, 5, 128, 128, 16, I.ROUND_SR, "mixed", steps=3),
         _small("mamba2", 3, 5, 128, 64, 64, I.ROUND_BDR, "mixed", steps=3),
         _small("gla", 37, 3, 64, 128, 16, I.ROUND_BDR, "int4", steps=2),
         _small("gdn", 149, 8, 128, 128, 32, I.ROUND_SR, "int8", steps=2)]
for w in cases:
    P.run_parity(w, w.steps, check_every=1)
lrs.lrs_sync()

# understate the code buffer's size: every tile past the declared end fails
# its check and is skipped
w = cases[0]
pm = np.array([8, 4, 8, 4, 8], np.uint8)
st = lrs.lrs_state_alloc(P.make_shape(w), pm)
fake = lrs.lrs_state()
ctypes.memmove(ctypes.addressof(fake), ctypes.addressof(st), ctypes.sizeof(st))
fake.code_bytes = st.code_bytes // 2
x = I.step_inputs(w, 0, device="cuda")
import torch
out = torch.empty(w.batch, w.heads, w.d_v, device="cuda")
lrs.lrs_decode_step(fake, st.state_codes, st.scales, st.prec_map, x["q"], x["k"], x["v"],
                    x["gates"], None, out, 0, 0, w.mode)
try:
    lrs.lrs_sync()
    raise SystemExit("the bounds checks did not fire")
except lrs.LrsError as e:
    assert e.status == lrs.LRS_ERR_DEVICE_BOUNDS, e
lrs.lrs_sync()
lrs.lrs_state_free(st)
print("bounds-checked build ok")
"""


def test_bounds_checked_build():
    r = subprocess.run([sys.executable, "-c", CHILD.replace("ROOT", repr(ROOT))], cwd=ROOT,
                       capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "bounds-checked build ok" in r.stdout
