"""Host-side checks of the C ABI (no GPU needed).

The library must load, export every function include/sq.h declares, and turn
every malformed argument into SQ_ERR_INVALID_ARG / SQ_ERR_UNSUPPORTED on the
host before anything is enqueued: none of these calls reaches the CUDA
runtime, so they run on a machine without a GPU.
"""
import ctypes
import os
import re
import subprocess

import pytest

import w8a8_int8_gemm_channel_b200 as sq
from w8a8_int8_gemm_channel_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sq.h")

A = 0x7F0000001000  # a 16-byte aligned fake device address (never dereferenced)
B = 0x7F0000002000
C = 0x7F0000003000
D = 0x7F0000004000
E = 0x7F0000005000
MIS = 0x7F0000001004  # misaligned
INV, UNS = sq.SQ_ERR_INVALID_ARG, sq.SQ_ERR_UNSUPPORTED


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return sq.lib()


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^SQ_API\s+[\w\s\*]*?\b(sq_\w+)\s*\(", text, re.M)))


def test_header_declares_the_binding_symbols():
    assert header_functions() == sorted(sq.ABI_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", sq.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = sorted({l.split()[-1] for l in out.splitlines() if l.split()[-1].startswith("sq_")})
    assert exported == header_functions()


def test_status_strings(lib):
    names = [sq.status_string(i) for i in range(5)]
    assert names == ["SQ_OK", "SQ_ERR_INVALID_ARG", "SQ_ERR_UNSUPPORTED", "SQ_ERR_CUDA",
                     "SQ_ERR_TIMEOUT"]
    assert sq.status_string(99) == "SQ_ERR_UNKNOWN"
    assert lib.sq_version() >= 100


def test_calib_absmax_rejects(lib):
    f = lib.sq_calib_absmax
    assert f(None, 1, 8, 64, 64, B, None) == INV           # null x
    assert f(A, 1, 8, 64, 64, None, None) == INV           # null ax
    assert f(A, 7, 8, 64, 64, B, None) == INV              # bad dtype
    assert f(A, 1, 0, 64, 64, B, None) == INV              # T = 0
    assert f(A, 1, 8, 40, 40, B, None) == INV              # K % 16
    assert f(A, 1, 8, 64, 60, B, None) == INV              # ldx < K
    assert f(A, 1, 8, 64, 68, B, None) == INV              # ldx * 2 bytes not a multiple of 16
    assert f(MIS, 1, 8, 64, 64, B, None) == INV            # misaligned x
    assert f(A, 0, 8, 64, 64, MIS, None) == INV            # misaligned ax


def test_smooth_factors_rejects(lib):
    f = lib.sq_smooth_factors
    assert f(A, B, 1, 32, 64, 1.5, C, None, None) == INV   # alpha > 1
    assert f(A, B, 1, 32, 64, -0.1, C, None, None) == INV  # alpha < 0
    assert f(A, B, 1, 32, 64, float("nan"), C, None, None) == INV
    assert f(A, B, 1, 32, 64, 0.5, A, None, None) == INV   # s aliases ax
    assert f(A, B, 1, 32, 64, 0.5, C, C, None) == INV      # aw aliases s
    assert f(A, B, 1, 32, 64, 0.5, C, MIS, None) == INV    # misaligned aw
    assert f(A, B, 1, 0, 64, 0.5, C, None, None) == INV    # N = 0
    assert f(A, B, 1, 32, 8, 0.5, C, None, None) == INV    # K < 16
    assert f(None, B, 1, 32, 64, 0.5, C, None, None) == INV


def test_quantisers_reject(lib):
    for f in (lib.sq_smooth_quant_weight, lib.sq_quant_act):
        assert f(None, 1, 4, 64, B, C, D, None) == INV
        assert f(A, 1, 0, 64, B, C, D, None) == INV       # zero rows
        assert f(A, 1, 4, 50, B, C, D, None) == INV       # K % 16
        assert f(A, 1, 4, 64, B, MIS, D, None) == INV     # misaligned codes
        assert f(A, 3, 4, 64, B, C, D, None) == INV       # bad dtype
        assert f(A, 1, 4, 65536 + 16, B, C, D, None) == UNS   # bf16 row longer than supported
        assert f(A, 0, 4, 32768 + 16, B, C, D, None) == UNS   # fp32 row longer than supported


def test_quantisers_do_not_run_without_valid_args(lib):
    # same calls but with one bad pointer so nothing is launched
    assert lib.sq_quant_act(A, 1, 4, 64, None, C, D, None) == INV
    assert lib.sq_smooth_quant_weight(A, 1, 4, 64, B, C, None, None) == INV


def test_gemm_rejects(lib):
    f = lib.sq_w8a8_gemm
    assert f(A, B, C, D, 0, 64, 64, E, 1, None) == INV     # M = 0
    assert f(A, B, C, D, 4, 40, 64, E, 1, None) == INV     # N % 16
    assert f(A, B, C, D, 4, 64, 72, E, 1, None) == INV     # K % 16
    assert f(A, B, C, D, 4, 64, 133152, E, 1, None) == UNS  # K * 127^2 would overflow int32
    assert f(A, B, C, D, 4, 64, 64, MIS, 1, None) == INV   # misaligned y
    assert f(A, None, C, D, 4, 64, 64, E, 1, None) == INV  # null sx
    assert f(A, B, C, D, 4, 64, 64, E, 2, None) == INV     # bad out dtype
    g = lib.sq_w8a8_gemm_s32
    assert g(A, B, 4, 64, 64, None, None) == INV
    assert g(A, B, -1, 64, 64, C, None) == INV
    assert g(MIS, B, 4, 64, 64, C, None) == INV


def test_linear_rejects_and_workspace_size(lib):
    M, N, K = 100, 64, 256
    need = sq.sq_linear_workspace_size(M, N, K)
    assert need >= M * K + 4 * M and need % 16 == 0
    f = lib.sq_linear
    assert need > 0 and f(A, 1, B, C, D, M, N, K, E, 1, None, 0, None) == INV
    a256 = lambda v: (v + 255) // 256 * 256
    minimum = a256(M * K) + a256(4 * M)  # the codes and scales; the rest only speeds the GEMM
    assert f(A, 1, B, C, D, M, N, K, E, 1, A + 0x100000, minimum - 1, None) == INV
    assert f(A, 1, B, C, D, M, N, K, E, 1, MIS, need, None) == INV
    assert f(A, 1, B, C, D, 0, N, K, E, 1, A, need, None) == INV
    assert f(A, 1, B, C, D, M, 24, K, E, 1, A, need, None) == INV
    assert f(A, 5, B, C, D, M, N, K, E, 1, A, need, None) == INV
    assert sq.sq_linear_workspace_size(0, 64, 64) == 0


def test_binding_fails_loudly_without_device_tensors():
    torch = pytest.importorskip("torch")
    x = torch.zeros(4, 16)
    with pytest.raises(ValueError):
        sq.sq_calib_absmax(x, torch.zeros(16))


def test_rmsnorm_entry_points_reject_bad_arguments(lib):
    f = lib.sq_fold_gamma
    assert f(None, B, 64, C, None) == INV
    assert f(A, B, 24, C, None) == INV        # K not a multiple of 16
    assert f(A, MIS, 64, C, None) == INV      # misaligned s
    g = lib.sq_rmsnorm_quant
    assert g(None, 1, 4, 64, B, 1e-5, C, D, None, None) == INV
    assert g(A, 1, 0, 64, B, 1e-5, C, D, None, None) == INV      # M < 1
    assert g(A, 1, 4, 40, B, 1e-5, C, D, None, None) == INV      # K not a multiple of 16
    assert g(A, 1, 4, 64, B, -1.0, C, D, None, None) == INV      # eps < 0
    assert g(A, 1, 4, 64, B, float("nan"), C, D, None, None) == INV
    assert g(A, 1, 4, 64, B, 1e-5, C, D, MIS, None) == INV       # misaligned rinv
    assert g(A, 7, 4, 64, B, 1e-5, C, D, None, None) == INV      # bad dtype
    assert g(A, 1, 4, 65536, B, 1e-5, C, D, None, None) == UNS   # row too long for one pass


def test_silu_mul_quant_rejects_bad_arguments(lib):
    f = lib.sq_silu_mul_quant
    assert f(None, 1, 4, 64, B, C, D, None, None) == INV
    assert f(A, 1, 0, 64, B, C, D, None, None) == INV           # M < 1
    assert f(A, 1, 4, 40, B, C, D, None, None) == INV           # I not a multiple of 16
    assert f(A, 1, 4, 64, MIS, C, D, None, None) == INV         # misaligned s
    assert f(A, 1, 4, 64, B, C, D, MIS, None) == INV            # misaligned h
    assert f(A, 7, 4, 64, B, C, D, None, None) == INV           # bad dtype
    assert f(A, 1, 4, 65536, B, C, D, None, None) == UNS        # row longer than one pass takes
    assert f(A, 0, 4, 32768, B, C, D, None, None) == UNS        # fp32 rows: at most 16384


def test_gemm_ws_rejects_bad_arguments(lib):
    f = lib.sq_w8a8_gemm_ws
    M, N, K = 300, 512, 1024
    need = lib.sq_w8a8_gemm_workspace_size(M, N, K)
    # 4 x 80 tile counters (1280 bytes), then 2 x 80 CTAs x 2 slots x 128 x 256 int32 partial sums
    assert need == 1280 + 160 * 2 * 128 * 256 * 4
    # few tokens: ceil(N / 128) counters (rounded up to 256 bytes), then
    # min(units, 160) CTAs x 2 slots x 32 tokens x 128 int32
    units = (6144 // 128) * (4096 // 128)
    assert lib.sq_w8a8_gemm_workspace_size(16, 6144, 4096) == 256 + min(units, 160) * 2 * 32 * 128 * 4
    assert lib.sq_w8a8_gemm_workspace_size(0, 6144, 4096) == 0
    assert f(A, B, C, D, M, N, K, E, 1, None, need, None) == INV      # no workspace
    assert f(A, B, C, D, M, N, K, E, 1, A, need - 1, None) == INV     # too small
    assert f(A, B, C, D, M, N, K, E, 1, MIS, need, None) == INV       # misaligned
    assert f(A, B, C, D, M, 24, K, E, 1, A, need, None) == INV        # N not a multiple of 16
    assert f(A, B, C, D, M, N, K, E, 5, A, need, None) == INV         # bad dtype
    assert f(None, B, C, D, M, N, K, E, 1, A, need, None) == INV


def test_gptq_entry_points_reject_bad_arguments(lib):
    assert lib.sq_gptq_workspace_size(4096) == 2 * 4096 * 4096 * 8
    assert lib.sq_gptq_workspace_size(40) == 0                     # not a multiple of 16
    assert lib.sq_gptq_workspace_size(32768) == 0                  # beyond the limit
    h = lib.sq_gptq_hessian
    assert h(None, 1, 8, 64, B, C, None) == INV
    assert h(A, 1, 0, 64, B, C, None) == INV                       # no tokens
    assert h(A, 1, 8, 40, B, C, None) == INV                       # K not a multiple of 16
    assert h(A, 7, 8, 64, B, C, None) == INV                       # bad dtype
    assert h(A, 1, 8, 32768, B, C, None) == UNS
    f = lib.sq_gptq_factor
    assert f(A, 64, 0.01, B, None, 1 << 20, None) == INV           # no workspace
    assert f(A, 64, 0.01, B, C, 2 * 64 * 64 * 8 - 1, None) == INV  # workspace too small
    assert f(A, 64, -0.5, B, C, 1 << 20, None) == INV              # negative damping
    assert f(A, 64, float("nan"), B, C, 1 << 20, None) == INV
    assert f(A, 64, 0.01, A, C, 1 << 20, None) == INV              # U aliases H
    assert f(A, 64, 0.01, MIS, C, 1 << 20, None) == INV
    q = lib.sq_gptq_quant_weight
    assert q(None, 1, 4, 64, B, C, D, E, None) == INV
    assert q(A, 1, 0, 64, B, C, D, E, None) == INV
    assert q(A, 1, 4, 24, B, C, D, E, None) == INV
    assert q(A, 1, 4, 64, B, C, D, MIS, None) == INV


def test_selftest_rejects_limits_out_of_range(lib):
    f = lib.sq_selftest_wait_timeout
    assert f(0, None) == INV
    assert f(2000001, None) == INV


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "sq.h"
int main(void)
{
    if (sq_version() < 100) return 1;
    if (strcmp(sq_status_string(SQ_ERR_INVALID_ARG), "SQ_ERR_INVALID_ARG") != 0) return 2;
    if (sq_gptq_workspace_size(64) != (size_t)2 * 64 * 64 * 8) return 3;
    /* rejected on the host before anything reaches CUDA */
    if (sq_quant_act(NULL, SQ_BF16, 4, 64, NULL, NULL, NULL, NULL) != SQ_ERR_INVALID_ARG) return 4;
    if (sq_silu_mul_quant(NULL, SQ_BF16, 4, 64, NULL, NULL, NULL, NULL, NULL) != SQ_ERR_INVALID_ARG) return 5;
    puts("c-client-ok");
    return 0;
}
"""


def test_plain_c_client_compiles_links_and_runs(tmp_path, lib):
    """include/sq.h is plain C (C11, -pedantic) and a C program links against
    libsq.so and calls it; only host-side entry points are exercised."""
    src = tmp_path / "client.c"
    exe = tmp_path / "client"
    src.write_text(C_CLIENT)
    libdir = os.path.dirname(sq.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), f"-L{libdir}", "-l:libsq.so", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and "c-client-ok" in out.stdout, (out.returncode, out.stderr)
