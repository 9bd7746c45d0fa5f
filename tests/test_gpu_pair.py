"""The two-SM grouped GEMM (clusters of two CTAs, M = 256 MMAs) against the
oracle on every small case, whatever the layer shape.

The library picks the two-SM kernel only for large tensor-bound layers; the
MOE_GG_PAIR=1 switch (read once per process) forces it for every grouped GEMM,
so the small parity cases run again in a child process with it set.  This
covers gathered and contiguous operands, gate/up and down, fp32 (tf32) and
bf16, partial 256-row tiles, the shared expert and 128-wide tiles."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_forward_small_with_two_sm_tiles():
    env = dict(os.environ, MOE_GG_PAIR="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_gpu_parity.py"),
                        "-k", "forward_small or one_expert or stage_entry"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert " passed" in r.stdout
