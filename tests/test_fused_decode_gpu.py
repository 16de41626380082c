"""The fused decode kernel (per-token quantisation inside the split-K GEMM
kernel's prologue), selected with SQ_LINEAR_FUSED=1.  The selection is read
once per process, so the check runs in a child process; it compares
sq_linear against the CPU oracle for 1 to 32 tokens, bit-exact codes and
outputs within 1 bf16 ulp.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import numpy as np, torch
import w8a8_int8_gemm_channel_b200 as sq
from oracle import oracle
from tests.gpu_util import to_np, to_dev, assert_output_close, exact_fraction
assert sq.sq_linear_workspace_size(16, 6144, 4096) == 0, "fused path not selected"
for (M, N, K) in [(1, 272, 4112), (16, 6144, 4096), (32, 512, 2048), (7, 4096, 14336)]:
    g = torch.Generator().manual_seed(M * 7 + N + K)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    x[:, 5] *= 60.0
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    xcal = torch.randn(256, K, generator=g).to(torch.bfloat16)
    xcal[:, 5] *= 60.0
    _, _, s_o, wq_o, sw_o = oracle.prepare(to_np(xcal), to_np(w), 0.5)
    y = sq.linear(x.cuda(), to_dev(s_o), to_dev(wq_o), to_dev(sw_o), out_dtype=torch.bfloat16)
    y_o, _, _, _ = oracle.linear(to_np(x), s_o, wq_o, sw_o, "bf16")
    assert_output_close(to_np(y), y_o, f"fused {M}x{N}x{K}")
    assert exact_fraction(to_np(y), y_o) == 1.0
st, code = sq.sq_device_status()
assert st == sq.SQ_OK, hex(code)
print("fused-ok")
'''


def test_fused_decode_linear_child_process():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, SQ_LINEAR_FUSED="1", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "fused-ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
