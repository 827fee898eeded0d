"""The debug build (libkda_debug.so, compiled with KDA_DEBUG=1) checks every global index of the
prefill, scan, single-kernel, fp32 and backward kernels against its buffer and records
KDA_ERR_BOUNDS in the status word instead of making a bad access: the library's stand-in for a
memory checker. This runs the small GPU parity cases (ragged and packed lengths, empty sequences,
fp32 and bf16 inputs, the two passes, the backward) in a child process that loads the debug
build; every case must match the oracle with a clean status word."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_small_parity_cases_on_the_debug_build():
    from kimi_delta_attention_25_b200 import build
    build.build()
    lib = build.build(debug=True)
    env = dict(os.environ, KDA_LIBRARY=lib)
    sel = ("ragged or varlen or fp32_t256 or two_pass or zero_initial or causality or "
           "fast_forgetting or beta_zero or deltanet or one_hot")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu and not slow", "-k", sel,
                        "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_gpu_parity.py"),
                        os.path.join(ROOT, "tests", "test_gpu_backward.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail
