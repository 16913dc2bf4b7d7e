"""The bounds-checked build on the GPU.

libdyra_debug.so is the same sources compiled with DYRA_DEBUG: every direct
global load or store of the kernels (the epilogues' row stores, the solves'
rows, the factor records) is checked against the extent of its buffer, and
an access outside it is skipped and raises DYRA_STATUS_BOUNDS instead of
touching memory. Copies through tensor maps are bounded by the hardware.
This stands in for a memory checker: a subset of the parity tests runs
against that library in a child process, and every one of them asserts a
clear status word, so any index outside its buffer fails the run.
"""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SUBSET = " or ".join([
    "test_edge_shapes",
    "test_config_parity and (tiny_f32 or vit_fc1 or whisper_fc1 or llama_up_1 or llama_up_128)",
    "test_als_iterations",
    "test_newton_schulz_solver",
    "test_bias_and_alpha",
    "test_compensated_correction",
    "test_projection_split_k",
    "test_factor_placements_agree",
])


def test_parity_subset_passes_under_the_bounds_checked_library():
    from rank_structured_matmul_b200 import dyra
    from rank_structured_matmul_b200.build import build
    build(debug=True)  # incremental: rebuilt only when a source is newer
    env = dict(os.environ, DYRA_DEBUG_LIB="1")
    out = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_parity.py"),
                          "-m", "gpu", "-q", "-x", "-p", "no:cacheprovider", "-k", SUBSET],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    tail = (out.stdout + out.stderr)[-3000:]
    assert out.returncode == 0, tail
    assert " passed" in out.stdout and "error" not in out.stdout.lower().split("passed")[-1], tail
