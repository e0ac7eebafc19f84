"""The fused GEMM has two variants: CTA pairs running cta_group::2 MMAs (the
default whenever a GEMM has two or more 128-feature tiles) and single CTAs
(LSQ_GEMM_PAIR=0, and every GEMM with one feature tile).  The rest of the GPU
suite runs the default; this file reruns the linear and layer parity tests in
a fresh process with the single-CTA kernel, so both stay checked against the
oracle."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_linear_and_layer_parity_with_single_cta_gemm():
    env = dict(os.environ, LSQ_GEMM_PAIR="0")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_gpu_linear.py"),
                        os.path.join(HERE, "test_gpu_layer.py")],
                       env=env, cwd=os.path.dirname(HERE), capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
