"""The C-ABI library loads and exports every symbol include/q4_0.h declares,
and its host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "q4_0.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"Q4_0_API\s+[\w\s\*]*?\b(q4_0_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def q4():
    import bit_weight_only_matmul_b200 as q4
    return q4


def test_header_lists_the_entry_points():
    syms = declared_symbols()
    assert "q4_0_gemm" in syms and "q4_0_pack" in syms and "q4_0_dequant" in syms
    assert "q4_0_gemm_grouped" in syms


def test_every_declared_symbol_is_exported(q4):
    lib = ctypes.CDLL(q4.LIB_PATH)
    missing = [s for s in declared_symbols() if not hasattr(lib, s)]
    assert not missing, missing
    assert sorted(q4.EXPORTS) == declared_symbols()


def test_status_strings(q4):
    for st in range(5):
        assert q4.lib.q4_0_status_string(st)
    assert b"unknown" in q4.lib.q4_0_status_string(99)


def test_bytes(q4):
    assert q4.q4_0_bytes(3072, 3072) == 5308416
    assert q4.q4_0_bytes(1, 32) == 18
    assert q4.q4_0_bytes(0, 64) == 0
    assert q4.q4_0_bytes(4, 33) == -1
    assert q4.q4_0_bytes(-1, 32) == -1


def test_force_path_range(q4):
    assert q4.lib.q4_0_force_path(7) == q4.Q4_ERR_INVALID_ARG
    assert q4.lib.q4_0_force_path(6) == q4.Q4_OK
    assert q4.lib.q4_0_force_path(-1) == q4.Q4_ERR_INVALID_ARG
    assert q4.lib.q4_0_force_path(0) == q4.Q4_OK


# argument checks happen before any CUDA call, so they work without a GPU
A = 1 << 20   # a fake, 16-byte aligned address that is never dereferenced


def test_gemm_argument_checks(q4):
    g = q4.lib.q4_0_gemm
    assert g(A, A, A, 1, 8, 48, None) == q4.Q4_ERR_INVALID_ARG       # K % 32
    assert g(A, A, A, -1, 8, 64, None) == q4.Q4_ERR_INVALID_ARG      # M < 0
    assert g(A, A, A, 1, -8, 64, None) == q4.Q4_ERR_INVALID_ARG      # N < 0
    assert g(A, A, A, 1, 8, 1 << 31, None) == q4.Q4_ERR_INVALID_ARG  # K too large
    assert g(None, A, A, 1, 8, 64, None) == q4.Q4_ERR_INVALID_ARG
    assert g(A, None, A, 1, 8, 64, None) == q4.Q4_ERR_INVALID_ARG
    assert g(A, A, None, 1, 8, 64, None) == q4.Q4_ERR_INVALID_ARG
    assert g(A + 2, A, A, 1, 8, 64, None) == q4.Q4_ERR_MISALIGNED
    assert g(A, A + 8, A, 1, 8, 64, None) == q4.Q4_ERR_MISALIGNED
    assert g(A, A, A + 4, 1, 8, 64, None) == q4.Q4_ERR_MISALIGNED
    # empty problems are valid no-ops and need no device
    assert g(None, None, None, 0, 8, 64, None) == q4.Q4_OK
    assert g(None, None, None, 4, 0, 64, None) == q4.Q4_OK


def test_pack_dequant_argument_checks(q4):
    p, d = q4.lib.q4_0_pack, q4.lib.q4_0_dequant
    assert p(A, A, A, 4, 40, None) == q4.Q4_ERR_INVALID_ARG
    assert p(None, A, A, 4, 64, None) == q4.Q4_ERR_INVALID_ARG
    assert p(A + 1, A, A, 4, 64, None) == q4.Q4_ERR_MISALIGNED
    assert p(A, A, A + 2, 4, 64, None) == q4.Q4_ERR_MISALIGNED
    assert p(None, None, None, 0, 64, None) == q4.Q4_OK
    assert p(None, None, None, 4, 0, None) == q4.Q4_OK
    assert d(A, A, 4, 31, None) == q4.Q4_ERR_INVALID_ARG
    assert d(A, None, 4, 64, None) == q4.Q4_ERR_INVALID_ARG
    assert d(A, A + 8, 4, 64, None) == q4.Q4_ERR_MISALIGNED
    assert d(None, None, 0, 64, None) == q4.Q4_OK


def test_grouped_argument_checks(q4):
    gg = q4.lib.q4_0_gemm_grouped
    probs = q4.make_problems([(A, A, A, 1, 8, 64), (A, A, A, 1, 8, 40)])
    assert gg(probs, 2, None) == q4.Q4_ERR_INVALID_ARG        # second problem bad: nothing launched
    assert gg(probs, -1, None) == q4.Q4_ERR_INVALID_ARG
    assert gg(probs, q4.Q4_0_MAX_GROUP + 1, None) == q4.Q4_ERR_INVALID_ARG
    assert gg(None, 3, None) == q4.Q4_ERR_INVALID_ARG
    assert gg(None, 0, None) == q4.Q4_OK
    empty = q4.make_problems([(None, None, None, 0, 8, 64)])
    assert gg(empty, 1, None) == q4.Q4_OK


def test_workspace_size_and_checks(q4):
    assert q4.q4_0_gemm_workspace_size(4096, 3072, 5120) == 4096 * 5120 * 2
    assert q4.q4_0_gemm_workspace_size(33, 8, 32) == 2304   # 33*32*2 = 2112 -> 2304
    assert q4.q4_0_gemm_workspace_size(32, 8, 64) == 0
    assert q4.q4_0_gemm_workspace_size(4, 8, 33) == -1
    ws = q4.lib.q4_0_gemm_ws
    assert ws(A, A, A, 64, 8, 64, None, 16, None) == q4.Q4_ERR_INVALID_ARG    # bytes but no pointer
    assert ws(A, A, A, 64, 8, 64, A + 4, 4096, None) == q4.Q4_ERR_MISALIGNED
    assert ws(A, A, A, 64, 8, 64, A, -1, None) == q4.Q4_ERR_INVALID_ARG
    assert ws(None, None, None, 0, 8, 64, None, 0, None) == q4.Q4_OK


def test_gather_quantize_argument_checks(q4):
    g, qz = q4.lib.q4_0_gather, q4.lib.q4_0_quantize
    assert g(A, A, A, 4, 10, 48, None) == q4.Q4_ERR_INVALID_ARG      # D % 32
    assert g(A, A, A, -1, 10, 64, None) == q4.Q4_ERR_INVALID_ARG     # T < 0
    assert g(A, A, A, 4, 0, 64, None) == q4.Q4_ERR_INVALID_ARG       # no rows to gather from
    assert g(None, A, A, 4, 10, 64, None) == q4.Q4_ERR_INVALID_ARG
    assert g(A, None, A, 4, 10, 64, None) == q4.Q4_ERR_INVALID_ARG
    assert g(A + 2, A, A, 4, 10, 64, None) == q4.Q4_ERR_MISALIGNED
    assert g(A, A + 2, A, 4, 10, 64, None) == q4.Q4_ERR_MISALIGNED
    assert g(A, A, A + 4, 4, 10, 64, None) == q4.Q4_ERR_MISALIGNED
    assert g(None, None, None, 0, 10, 64, None) == q4.Q4_OK         # nothing to do
    assert qz(A, A, 4, 40, None) == q4.Q4_ERR_INVALID_ARG
    assert qz(None, A, 4, 64, None) == q4.Q4_ERR_INVALID_ARG
    assert qz(A + 4, A, 4, 64, None) == q4.Q4_ERR_MISALIGNED
    assert qz(None, None, 0, 64, None) == q4.Q4_OK


def test_grouped_ex_argument_checks(q4):
    def ex(M, N, K, R=A, epi=q4.Q4_0_EPI_RESIDUAL):
        arr = (q4.q4_0_problem_ex * 1)()
        arr[0] = q4.q4_0_problem_ex(A, A, A, M, N, K, R, epi)
        return q4.lib.q4_0_gemm_grouped_ex(arr, 1, None)
    assert ex(0, 128, 256) == q4.Q4_ERR_INVALID_ARG                       # M >= 1
    for M in (4, 300):                                                    # decode and tensor-core paths
        assert ex(M, 128, 288) == q4.Q4_ERR_INVALID_ARG                   # K % 256
        assert ex(M, 128, 256, R=None) == q4.Q4_ERR_INVALID_ARG           # residual needs R
        assert ex(M, 128, 256, R=A + 4) == q4.Q4_ERR_MISALIGNED
        assert ex(M, 192, 256, epi=q4.Q4_0_EPI_SWIGLU) == q4.Q4_ERR_INVALID_ARG   # 2F with F % 64
        assert ex(M, 128, 256, epi=7) == q4.Q4_ERR_INVALID_ARG
    assert ex(4, 128, 288) == q4.Q4_ERR_INVALID_ARG                       # K % 256
    assert ex(4, 128, 256, R=None) == q4.Q4_ERR_INVALID_ARG               # residual needs R
    assert ex(4, 128, 256, R=A + 4) == q4.Q4_ERR_MISALIGNED
    assert ex(4, 192, 256, epi=q4.Q4_0_EPI_SWIGLU) == q4.Q4_ERR_INVALID_ARG   # 2F with F % 64
    assert ex(4, 128, 256, epi=7) == q4.Q4_ERR_INVALID_ARG
    il = q4.lib.q4_0_interleave_gate_up
    assert il(A, A, A, 96, 256, None) == q4.Q4_ERR_INVALID_ARG            # F % 64
    assert il(A, A, A, 64, 288, None) == q4.Q4_ERR_INVALID_ARG            # K % 256
    assert il(A + 8, A, A, 64, 256, None) == q4.Q4_ERR_MISALIGNED
    assert il(None, None, None, 0, 256, None) == q4.Q4_OK


def test_selftest_argument_checks(q4):
    assert q4.lib.q4_0_selftest_wait_timeout(0, None) == q4.Q4_ERR_INVALID_ARG
    assert q4.lib.q4_0_selftest_wait_timeout(1000001, None) == q4.Q4_ERR_INVALID_ARG


def test_stream_read_argument_checks(q4):
    f = q4.lib.q4_0_stream_read
    assert f(A, 0, 256, A, None) == q4.Q4_OK               # nothing to read
    assert f(None, 4, 256, A, None) == q4.Q4_ERR_INVALID_ARG
    assert f(A, 4, 256, None, None) == q4.Q4_ERR_INVALID_ARG
    assert f(A, 4, 96, A, None) == q4.Q4_ERR_INVALID_ARG   # K % 256 != 0
    assert f(A, 4, 250, A, None) == q4.Q4_ERR_INVALID_ARG  # K % 32 != 0
    assert f(A + 8, 4, 256, A, None) == q4.Q4_ERR_MISALIGNED
    assert f(A, 4, 256, A + 2, None) == q4.Q4_ERR_MISALIGNED


def test_header_is_plain_c_and_matches_the_binding(q4, tmp_path):
    """include/q4_0.h compiles as C99 with no CUDA header, and the problem
    structs the binding builds with ctypes have the C layout: same size, same
    field offsets."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("needs gcc")
    fields = {"q4_0_problem": ["W", "X", "Y", "M", "N", "K"],
              "q4_0_problem_ex": ["W", "X", "Y", "M", "N", "K", "R", "epilogue"]}
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "q4_0.h"', "int main(void) {"]
    for st, fs in fields.items():
        lines.append(f'    printf("{st} size %zu\\n", sizeof({st}));')
        for f in fs:
            lines.append(f'    printf("{st} {f} %zu\\n", offsetof({st}, {f}));')
    lines += ["    return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = str(tmp_path / "layout")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", f"-I{os.path.join(ROOT, 'include')}",
                    str(src), "-o", exe], check=True)
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {tuple(l.split()[:2]): int(l.split()[2]) for l in out if l.strip()}
    for st, fs in fields.items():
        cls = getattr(q4, st)
        assert got[(st, "size")] == ctypes.sizeof(cls), st
        for f in fs:
            assert got[(st, f)] == getattr(cls, f).offset, (st, f)


def test_prepared_path_argument_checks(q4):
    pb = q4.lib.q4_0_prepared_x_bytes
    assert pb(4096, 5120) == 4096 * 5120 * 2
    assert pb(3, 256) == 1536 and pb(1, 256) == 512
    assert pb(5, 512) == 5120 and pb(3, 768) == 4608
    assert pb(4, 288) == -1 and pb(-1, 256) == -1
    px = q4.lib.q4_0_prepare_x
    assert px(A, 4, 256, A, 2047, None) == q4.Q4_ERR_INVALID_ARG          # buffer too small
    assert px(A, 4, 288, A, 4096, None) == q4.Q4_ERR_INVALID_ARG          # K % 256
    assert px(A + 8, 4, 256, A, 2048, None) == q4.Q4_ERR_MISALIGNED
    assert px(A, 4, 256, A + 8, 2048, None) == q4.Q4_ERR_MISALIGNED
    assert px(None, 0, 256, None, 0, None) == q4.Q4_OK                    # nothing to convert
    gp = q4.lib.q4_0_gemm_prepared
    assert gp(A, A, A, 64, 128, 288, None) == q4.Q4_ERR_INVALID_ARG       # K % 256
    assert gp(A, A, A, 64, 128, 224, None) == q4.Q4_ERR_INVALID_ARG
    assert gp(A, A + 8, A, 64, 128, 256, None) == q4.Q4_ERR_MISALIGNED
    assert gp(None, None, None, 0, 128, 256, None) == q4.Q4_OK
