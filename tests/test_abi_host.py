"""The C ABI without a GPU: the library loads, exports every function that
include/lrs.h declares, and validates arguments on the host."""
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
from quantized_recurrent_state_decode_b200 import build as B
from quantized_recurrent_state_decode_b200 import lrs

HEADER = os.path.join(B.ROOT, "include", "lrs.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lrs_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_function():
    names = declared_functions()
    assert len(names) >= 18
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (lrs_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    L = lrs.lib()
    for n in names:
        assert hasattr(L, n)


def test_version_and_status_names():
    assert lrs.lrs_version() == 2
    assert lrs.lrs_status_string(lrs.LRS_ERR_DEVICE_TIMEOUT) == "LRS_ERR_DEVICE_TIMEOUT"
    assert lrs.lrs_status_string(99) == "LRS_ERR_UNKNOWN"


def test_layout_offsets_are_prefix_sums():
    pm = np.array([8, 4, 4, 8, 4], np.uint8)
    shp = lrs.shape(3, 5, 128, 64, 32, lrs.LRS_UPDATE_GATED, lrs.LRS_GATE_SCALAR)
    offs, stride, nsc = lrs.lrs_layout_query(shp, pm)
    sizes = 128 * 64 * pm.astype(np.int64) // 8
    np.testing.assert_array_equal(offs, np.concatenate([[0], np.cumsum(sizes)[:-1]]))
    assert stride == sizes.sum()
    assert nsc == 3 * 5 * (128 // 32) * 64


def test_group_layout_offsets_are_prefix_sums():
    pm = np.array([[8, 4, 4, 8], [4, 4, 4, 4], [8, 8, 8, 4]], np.uint8)
    shp = lrs.shape(2, 3, 128, 64, 32, lrs.LRS_UPDATE_GATED, lrs.LRS_GATE_SCALAR)
    offs, stride, nsc = lrs.lrs_layout_query_groups(shp, pm)
    sizes = (32 * 64 * pm.astype(np.int64) // 8).sum(axis=1)
    np.testing.assert_array_equal(offs, np.concatenate([[0], np.cumsum(sizes)[:-1]]))
    assert stride == sizes.sum()
    assert nsc == 2 * 3 * 4 * 64
    # a uniform group map is the head map's layout
    o2, s2, _ = lrs.lrs_layout_query(shp, pm[:, 0].copy())
    o3, s3, _ = lrs.lrs_layout_query_groups(shp, np.repeat(pm[:, :1], 4, axis=1))
    np.testing.assert_array_equal(o2, o3)
    assert s2 == s3
    with pytest.raises(lrs.LrsError) as ei:
        lrs.lrs_layout_query_groups(shp, np.full((3, 4), 6, np.uint8))
    assert ei.value.status == lrs.LRS_ERR_INVALID_ARG


@pytest.mark.parametrize("args,status", [
    ((2, 2, 128, 96, 32, 0, 1), lrs.LRS_ERR_UNSUPPORTED),   # d_v
    ((2, 2, 128, 128, 64, 0, 1), lrs.LRS_ERR_UNSUPPORTED),  # group*d_v too large
    ((2, 2, 100, 128, 32, 0, 1), lrs.LRS_ERR_UNSUPPORTED),  # group does not divide d_k
    ((2, 2, 512, 128, 32, 0, 1), lrs.LRS_ERR_UNSUPPORTED),  # d_k too large
    ((2, 2, 128, 128, 24, 0, 1), lrs.LRS_ERR_UNSUPPORTED),  # group size
    ((2, 2, 128, 128, 32, 1, 1), lrs.LRS_ERR_UNSUPPORTED),  # delta with per-key decay
    ((2, 2, 128, 128, 32, 2, 1), lrs.LRS_ERR_INVALID_ARG),  # update kind
    ((2, 2, 128, 128, 32, 0, 3), lrs.LRS_ERR_INVALID_ARG),  # gate kind
    ((-1, 2, 128, 128, 32, 0, 1), lrs.LRS_ERR_INVALID_ARG),
    ((2, 0, 128, 128, 32, 0, 1), lrs.LRS_ERR_INVALID_ARG),
])
def test_invalid_shapes_rejected(args, status):
    with pytest.raises(lrs.LrsError) as e:
        lrs.lrs_layout_query(lrs.shape(*args), np.full(max(args[1], 1), 8, np.uint8))
    assert e.value.status == status
    assert lrs.lrs_last_error().startswith(lrs.lrs_status_string(status))


def test_invalid_precision_rejected():
    with pytest.raises(lrs.LrsError) as e:
        lrs.lrs_layout_query(lrs.shape(1, 3, 64, 64, 32, 0, 0), np.array([8, 5, 4], np.uint8))
    assert e.value.status == lrs.LRS_ERR_INVALID_ARG


def test_step_on_unallocated_state_is_rejected_before_any_launch():
    st = lrs.lrs_state()
    with pytest.raises(lrs.LrsError) as e:
        lrs.lrs_decode_step(st, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, stream=0)
    assert e.value.status == lrs.LRS_ERR_INVALID_ARG


def test_free_of_unallocated_state_is_a_no_op():
    lrs.lrs_state_free(lrs.lrs_state())


def test_fault_injection_arguments():
    with pytest.raises(lrs.LrsError):
        lrs.lrs_debug_inject_timeout(True, 0)
    lrs.lrs_debug_inject_timeout(False, 0)


def test_precision_map_matches_oracle():
    rng = np.random.default_rng(0)
    for H in (1, 7, 32, 64):
        means = rng.random(H)
        means[rng.integers(0, H, H // 3)] = 0.5      # ties
        for n8 in {0, H // 4, H // 2, H}:
            np.testing.assert_array_equal(lrs.lrs_precision_map(means, n8),
                                          oracle.precision_map(means, n8))
    with pytest.raises(lrs.LrsError):
        lrs.lrs_precision_map(np.zeros(4), 5)
