"""GPU parity of the transposed tcgen05 kernel (attn_tct_kernel: S^T = K Q^T and O^T += V^T P^T
with M = 128 keys / head dims and N = 32 rows) for units of at most 32 rows, bf16 and fp8 KV.

The kernel is selected per process by WMTP_TCT (read once when the library first launches an
attention call), so the bf16 and fp8 attention parity suites run again in a child process with
WMTP_TCT=all: every unit of at most 32 rows, including the one-query draft calls, the windowed
ring calls, ragged batches, empty and short requests, a planted bad page id and the tree verify,
then goes through this kernel and is compared with the fp64 oracle.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_attention_suites_pass_on_the_transposed_kernel():
    env = dict(os.environ, WMTP_TCT="all")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        "tests/test_gpu_attention.py", "tests/test_gpu_fp8.py"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
