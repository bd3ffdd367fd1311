"""The bounds-checked build (libqlora_b200_debug.so, compiled with
QLORA_DEBUG): its kernels check every computed index of a raw pointer access
against the extent of the buffer it indexes and record the first failure
instead of faulting.  These tests run it in child processes: the record and
report path on a check that touches no memory, then the parity suites of the
codec, decode, linear variants, block and optimizer under the checked build,
where conftest asserts after every test that no check failed."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ENV = dict(os.environ, QLORA_B200_BUILD="debug")


def run(args, timeout):
    return subprocess.run(args, cwd=ROOT, env=ENV, capture_output=True, text=True, timeout=timeout)


def test_bounds_record_and_report():
    code = (
        "import torch, bit_nf4_quantized_16_b200 as q\n"
        "torch.cuda.init()\n"
        "assert q.LIB_PATH.endswith('libqlora_b200_debug.so')\n"
        "assert q.qlora_debug_bounds() == (0, '')\n"
        "q.qlora_debug_bounds_selftest()\n"
        "line, unit = q.qlora_debug_bounds()\n"
        "assert line > 0 and unit == 'api.cu', (line, unit)\n"
        "assert q.qlora_debug_bounds() == (0, '')\n"
        "print('ok')\n")
    r = run([sys.executable, "-c", code], 300)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr


def test_parity_suites_under_the_checked_build():
    r = run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "gpu",
             "tests/test_gpu_codec.py", "tests/test_gpu_decode.py", "tests/test_gpu_block.py",
             "tests/test_gpu_optim.py", "tests/test_gpu_linear.py",
             "-k", "not llama7b and not llama65b and not 7b_gate"], 1500)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
