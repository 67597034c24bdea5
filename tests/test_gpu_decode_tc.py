"""Parity of the opt-in decode-regime tcgen05 residual GEMM (gemm_dq.cu).

The planner selects that kernel only when TILEQ_DECODE_TC=1 is set when the
library makes its first plan, so these cases run the decode parity tests of
test_gpu_parity.py again in a child process with the variable set: tiny layers
with ragged tiles and every supported group, and the Mixtral-, Qwen- and
64-expert-shaped layers at their decode batches (prefill batches take the
wide-tile kernels either way)."""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.gpu
def test_decode_tc_kernel_parity():
    env = dict(os.environ, TILEQ_DECODE_TC="1")
    sel = "tiny_layers or mixtral_shaped_decode_and_prefill or qwen15moe_shaped or finegrained_64e or nonfinite or range_error"
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(HERE, "test_gpu_parity.py"), "-m", "gpu", "-x", "-q",
                        "-k", sel, "-p", "no:cacheprovider"], env=env, capture_output=True, text=True, timeout=1500)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-25:])
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail
