"""The bounds-checked build (libmr_checked.so, -DMR_CHECKED) on small, odd shapes.

It runs a selection of the GPU parity and canary tests in a child process with MR_LIBRARY=checked:
ragged lengths, both block sizes, query-block ranges, fp8 maps, paged values and the dense path.
Every global store of the tensor-core kernels is then checked against its extent on the device,
and any miss would surface as MR_ERR_DEVICE_CHECK in the status words those tests assert to be OK.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SELECTION = [
    "tests/test_abi.py::test_library_variant_matches_environment",
    "tests/test_gpu_parity.py::test_tiny_lengths",
    "tests/test_gpu_parity.py::test_block_ranges_reassemble_the_full_call",
    "tests/test_gpu_parity.py::test_dense_tensor_core_ragged_with_key_block_bias",
    "tests/test_gpu_parity.py::test_fp8_maps_against_the_oracle",
    "tests/test_gpu_parity.py::test_paged_values",
    "tests/test_gpu_parity.py::test_capacity_overflow_is_reported",
    "tests/test_gpu_canary.py",
]


def test_parity_selection_under_the_checked_build():
    env = dict(os.environ, MR_LIBRARY="checked")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", *SELECTION],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-25:])
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout, tail
