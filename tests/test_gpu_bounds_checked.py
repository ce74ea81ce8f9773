"""The bounds-checking build (liblfwd_checked.so, -DLLM_BOUNDS_CHECK) on the GPU.

In a child process that loads the checked library (LLM_LIB_VARIANT=checked):
small cases of the GEMV, the tensor-core GEMM, the three attention kernels and
of bf16 and fp32 models agree with the oracle and leave the device error word at
zero; an out-of-range token id is reported as LLM_ERR_DEVICE_BOUNDS (naming the
check) and the model keeps working afterwards.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_checked_build_runs_clean_and_reports_a_bad_token(lib):
    from llama_decoder_forward_fwd_b200 import build as B
    B.build()
    env = dict(os.environ, LLM_LIB_VARIANT="checked")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "checked_lib_run.py")], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "CHECKED OK" in r.stdout
