"""The grouped GEMM variants the library picks only for some layer shapes,
forced on every small parity case against the oracle:

* the two-SM kernel (clusters of two CTAs, M = 256 MMAs), chosen for large
  tensor-bound layers; MOE_GG_PAIR=1 forces it for every grouped GEMM
  (gathered and contiguous operands, gate/up and down, fp32 (tf32) and bf16,
  partial 256-row tiles, the shared expert, 128-wide tiles);
* 64-row down tiles with 64-row A stages, chosen when experts average at most
  64 rows; MOE_GG_HALF=1 forces them;
* the fused expert kernel (gate/up, SwiGLU, down and combine in one pass),
  chosen when experts average at most one 128-row tile; MOE_FUSED=1 forces it
  wherever the hidden width is a multiple of 128 (experts with several row
  tiles included).

The switches are read once per process, so each run is a child process."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_small_cases(**switches):
    env = dict(os.environ, **switches)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_gpu_parity.py"),
                        "-k", "forward_small or one_expert or stage_entry"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert " passed" in r.stdout


@pytest.mark.gpu
def test_forward_small_with_two_sm_tiles():
    run_small_cases(MOE_GG_PAIR="1")


@pytest.mark.gpu
def test_forward_small_with_half_height_down_tiles():
    run_small_cases(MOE_GG_PAIR="0", MOE_GG_HALF="1")


@pytest.mark.gpu
def test_forward_small_with_fused_expert_kernel():
    run_small_cases(MOE_FUSED="1")
