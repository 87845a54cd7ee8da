"""The debug build of the library (Q4_DEBUG defined: index checks in the
decode and tensor-core kernels that flag Q4_DEVERR_DEBUG_CHECK and skip the
access instead of touching memory outside a buffer) compiles for sm_100a, and
the library it links exports every entry point the header declares.  Its
kernels run on the GPU in tests/test_gpu_debug_build.py."""
import ctypes
import importlib.util
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _builder():
    spec = importlib.util.spec_from_file_location("q4_0_b200_build", os.path.join(ROOT, "bit_weight_only_matmul_b200",
                                                                                  "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_debug_build_compiles_and_exports_the_abi():
    lib_path = _builder().build(debug=True)
    assert lib_path.endswith("libq4_0_b200_debug.so") and os.path.exists(lib_path)
    header = open(os.path.join(ROOT, "include", "q4_0.h")).read()
    names = re.findall(r"Q4_0_API\s+[\w\s\*]+?\b(q4_0_\w+)\s*\(", header)
    assert len(names) >= 18
    lib = ctypes.CDLL(lib_path)
    for n in names:
        assert hasattr(lib, n), n
    # host-side argument checks run without a GPU
    lib.q4_0_gemm.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 3 + [ctypes.c_void_p]
    assert lib.q4_0_gemm(1 << 20, 1 << 20, 1 << 20, 2, 64, 100, None) == 1   # K % 32 != 0
