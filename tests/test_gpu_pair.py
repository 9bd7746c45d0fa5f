"""The GEMM variants the library picks only for some layer shapes, forced on
the small parity cases against the oracle:

* the two-SM kernel (clusters of two CTAs, M = 256 MMAs), chosen for large
  tensor-bound layers; MOE_GG_PAIR=1 forces it for every grouped GEMM
  (gathered and contiguous operands, gate/up and down, fp32 (tf32) and bf16,
  partial 256-row tiles, the shared expert, 128-wide tiles);
* 64-row down tiles with 64-row A stages, chosen when experts average at most
  64 rows; MOE_GG_HALF=1 forces them;
* the fused expert kernel (gate/up, SwiGLU, down and combine in one pass),
  opt-in; MOE_FUSED=1 forces it wherever the hidden width is a multiple of 64
  (experts with several row tiles included);
* the routed down GEMM's column tiles in consecutive groups (chosen when
  the combine accumulator is large): MOE_DOWN_GROUPS=3 forces three;
* the warp-per-output batch-1 down kernel, which the library keeps for
  layers with a shared expert or fp32 weights: MOE_DOWN_TMA=0 forces it on
  the bf16 decode cases instead of the TMA-ring kernel;
* the backward GEMMs on two-SM tiles (chosen when groups average at least 512
  rows, or a weight gradient has at least 512 rows): MOE_BWD_PAIR=1 forces
  them on the small training cases, MOE_BWD_PAIR=0 forces one-SM tiles on the
  cases sized for them.

The switches are read once per process, so each run is a child process."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_small_cases(test_file="test_gpu_parity.py", select="forward_small or one_expert or stage_entry",
                    **switches):
    env = dict(os.environ, **switches)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", test_file), "-k", select],
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


@pytest.mark.gpu
def test_forward_small_with_down_column_groups():
    """The down GEMM's column tiles in three consecutive groups (one-SM and two-SM tiles)."""
    run_small_cases(MOE_DOWN_GROUPS="3")
    run_small_cases(MOE_DOWN_GROUPS="3", MOE_GG_PAIR="1")


@pytest.mark.gpu
def test_decode_small_with_warp_per_output_down():
    run_small_cases(select="decode", MOE_DOWN_TMA="0")


@pytest.mark.gpu
def test_backward_small_with_two_sm_tiles():
    """Every backward GEMM of the small training cases on two-SM tiles."""
    run_small_cases("test_gpu_backward.py", "backward_small or balance_bias or zero_rows", MOE_BWD_PAIR="1")


@pytest.mark.gpu
def test_backward_pair_sized_cases_with_one_sm_tiles():
    """The cases sized for two-SM tiles, on one-SM tiles."""
    run_small_cases("test_gpu_backward.py", "pair_tiles or pair_ragged", MOE_BWD_PAIR="0")

