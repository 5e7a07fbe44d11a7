"""The bounds-checked build of the library (build.py --checked,
-DFP4ATTN_BOUNDS_CHECK): every kernel checks its global stores, atomics and
tile coordinates against the sizes of their buffers and records
FP4ATTN_ERR_RANGE instead of making an out-of-range access.

On the CPU: it builds, loads and exports every symbol the header declares.
On the GPU: the tiny parity tests run against it in a fresh process
(FP4ATTN_BOUNDS_CHECK=1 selects it) and pass unchanged -- the checks raise no
false alarm and change no result."""
import ctypes
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_checked_build_loads_and_exports_every_declared_symbol():
    from nvfp4_precision_b200 import build
    path = build.build(checked=True)
    lib = ctypes.CDLL(path)
    from test_abi_cpu import declared_functions
    for name in sorted(declared_functions()):
        assert hasattr(lib, name), name


@pytest.mark.gpu
def test_tiny_parity_against_the_checked_build():
    from nvfp4_precision_b200 import build
    build.build(checked=True)
    env = dict(os.environ, FP4ATTN_BOUNDS_CHECK="1")
    tests = ["tests/test_gpu_attention.py::test_attention_tiny_full",
             "tests/test_gpu_attention.py::test_attention_ragged_lengths",
             "tests/test_gpu_attention.py::test_end_to_end_prologue_then_attention_tiny",
             "tests/test_gpu_prologue.py::test_prologue_bit_exact_tiny_all_flags",
             "tests/test_gpu_prologue.py::test_prologue_bit_exact_small",
             "tests/test_gpu_toy.py::test_toy_prologue_bit_exact",
             "tests/test_gpu_degenerate.py::test_empty_shapes_through_the_general_entry_points"]
    code = ("import sys, pytest\n"
            "from nvfp4_precision_b200 import fp4attn\n"
            "assert fp4attn.LIB_PATH.endswith('libfp4attn_checked.so'), fp4attn.LIB_PATH\n"
            f"sys.exit(pytest.main({tests!r} + ['-q', '-m', 'gpu', '-p', 'no:cacheprovider']))\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
