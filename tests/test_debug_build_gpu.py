"""The bounds-checking build (libfp4q_debug.so, FP4Q_DEBUG=1) on the odd-shape suites.

That library checks every global-memory access its kernels make by hand
against the extent the call's arguments give the buffer; an access outside it
is skipped and recorded in the device error word (with its site and offset).
Here the parity suites -- ragged tails, single rows, strided rows, column
counts that are not a multiple of 32, empty and all-zero tensors, extreme
magnitudes, batches, outliers, the operand form and the product -- run against
that library in a child process (the binding picks it up from
FP4Q_DEBUG_LIBRARY=1), and afterwards the error word must be clear: no access
left its buffer.
"""
from __future__ import annotations

import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUITES = ["tests/test_parity_gpu.py", "tests/test_batch_gpu.py", "tests/test_outliers_gpu.py",
          "tests/test_gemm_gpu.py"]
CHECK = """
import sys
sys.path.insert(0, {root!r})
from activation_quantization_block_b200 import fp4q
assert fp4q.fp4q_debug_build() == 1, "not the bounds-checking library"
st, bits = fp4q.fp4q_device_errors()
st2, site, off = fp4q.fp4q_device_error_site()
assert st == 0 and st2 == 0
assert bits == 0 and site == 0, f"device error word {{bits:#x}}, first out-of-bounds access at site {{site}}, offset {{off}}"
print("debug build: error word clear")
"""


def test_odd_shape_suites_on_the_bounds_checking_build_leave_the_error_word_clear():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, FP4Q_DEBUG_LIBRARY="1")
    # the suites and the final check share one process, so that the check reads the
    # error word the suites' kernels wrote
    runner = (
        "import sys, pytest\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        f"rc = pytest.main(['-x', '-q', '-m', 'gpu', '-p', 'no:cacheprovider', *{SUITES!r}])\n"
        "if rc != 0:\n"
        "    sys.exit(int(rc))\n"
        + CHECK.format(root=ROOT)
    )
    r = subprocess.run([sys.executable, "-c", runner], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=1200)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert "debug build: error word clear" in r.stdout, tail
