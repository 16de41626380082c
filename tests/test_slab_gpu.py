"""Parity of the slab GEMM (at most 32 tokens) against the CPU oracle.

For M <= 32 the GEMM behind sq_linear, sq_w8a8_gemm, sq_w8a8_gemm_ws and
sq_w8a8_gemm_s32 gives every CTA a slab of whole output channels (16-channel
groups, two slab widths when the groups do not divide evenly) over the full
K, with the tokens as the MMA's 128-row side (8, 16 or 32 rows loaded).  The
int32 accumulators must equal the oracle's brute-force dot products exactly,
and the dequantised outputs the oracle's within 1 bf16 ulp / 1e-6 relative
(in practice bit-exact) -- "quant_llm_int8", "The architecture: every piece
explained"; "Understanding W8A8 INT8 LLM Quantization", "Why Activation
Quantization Is Hard, and How SmoothQuant Fixes It".

The kernel is used where the narrower slab is at least 128 channels and the
wider one fits one MMA (N of about 19K to 38K on 148 SMs).  Shapes cover
every token-tile width and the token counts around them, one and two slab
widths, the widest slab (256 channels), K that is not a multiple of the
128-byte k block, and both output types.
The weight-streaming kernel is checked on the same shapes in a child process
with SQ_DECODE_SLAB=0.
"""
import numpy as np
import pytest
import torch

import w8a8_int8_gemm_channel_b200 as sq
from w8a8_int8_gemm_channel_b200 import workloads as wls
from tests.gpu_util import assert_output_close, exact_fraction, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w8a8_int8_gemm_channel_b200 import _build

    _build.build()
    yield
    st, code = sq.sq_device_status()
    assert st == sq.SQ_OK, f"device error word {code:#x}"


def _case(M, N, K, dtype, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, rng.choice(K, max(1, K // 1000), replace=False)] *= 60.0
    if M > 3:
        x[2] = 0.0  # a zero token
    xt = torch.from_numpy(x).to(dtype)
    s = rng.uniform(0.3, 8.0, K).astype(np.float32)
    wq = wls.random_int8((N, K), seed=seed + 1).numpy()
    sw = (rng.uniform(0.5, 2.0, N) * 1e-3).astype(np.float32)
    return xt, s, wq, sw


# (M, N, K) with slab widths for 148 SMs; the slab kernel takes shapes whose
# narrower slab is at least 128 channels (N of about 19K to 38K at M <= 32)
SHAPES = [
    (1, 28672, 4096),    # 138 CTAs of 192 or 208 channels, 8-row token tile
    (8, 28672, 1024),
    (9, 28672, 1024),    # 16-row tile
    (17, 20480, 4112),   # 143 CTAs of 128 or 144, K not a multiple of 128, 32-row tile
    (32, 37888, 256),    # the widest slab: 256 channels
    (32, 19968, 2064),   # 139 CTAs of 128 or 144
    (16, 18944, 16),     # 148 CTAs of 128, one partial k block
]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_slab_linear_bf16(oracle, M, N, K):
    xt, s, wq, sw = _case(M, N, K, torch.bfloat16, seed=M * 5 + N + K)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    need = sq.sq_linear_workspace_size(M, N, K)
    ws = torch.full((max(need, 16),), 0xA5, dtype=torch.uint8, device="cuda")
    sq.sq_linear(xt.cuda(), to_dev(s), to_dev(wq), to_dev(sw), y, ws if need else None)
    torch.cuda.synchronize()
    y_o, _, _, _ = oracle.linear(to_np(xt), s, wq, sw, "bf16")
    assert_output_close(to_np(y), y_o, f"y {M}x{N}x{K}")
    assert exact_fraction(to_np(y), y_o) == 1.0


@pytest.mark.parametrize("M,N,K", [(3, 28672, 2048), (32, 20480, 1040), (12, 37888, 512)])
def test_slab_linear_f32(oracle, M, N, K):
    xt, s, wq, sw = _case(M, N, K, torch.float32, seed=M + N * 3 + K)
    y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    need = sq.sq_linear_workspace_size(M, N, K)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    sq.sq_linear(xt.cuda(), to_dev(s), to_dev(wq), to_dev(sw), y, ws if need else None)
    torch.cuda.synchronize()
    y_o, _, _, _ = oracle.linear(to_np(xt), s, wq, sw, "f32")
    assert_output_close(to_np(y), y_o, f"y {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(1, 28672, 4096), (16, 20480, 1040), (32, 37888, 256), (7, 19968, 208)])
def test_slab_gemm_entry_points(oracle, M, N, K):
    """sq_w8a8_gemm_s32 (the int32 accumulators, exact), sq_w8a8_gemm and
    sq_w8a8_gemm_ws (dequantised, equal to each other bit for bit)."""
    xq = wls.random_int8((M, K), M + K).cuda()
    wq = wls.random_int8((N, K), N + 7).cuda()
    g = torch.Generator().manual_seed(M * N)
    sx = (torch.rand(M, generator=g) * 0.05 + 1e-3).cuda()
    sw = (torch.rand(N, generator=g) * 1e-3 + 1e-5).cuda()
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    sq.sq_w8a8_gemm_s32(xq, wq, acc)
    y0 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    y1 = torch.empty_like(y0)
    sq.sq_w8a8_gemm(xq, sx, wq, sw, y0)
    ws = torch.full((max(sq.sq_w8a8_gemm_workspace_size(M, N, K), 16),), 0xFF, dtype=torch.uint8, device="cuda")
    sq.sq_w8a8_gemm_ws(xq, sx, wq, sw, y1, ws)
    torch.cuda.synchronize()
    acc_o = oracle.gemm_i32(to_np(xq), to_np(wq))
    assert np.array_equal(to_np(acc), acc_o)
    y_o = oracle.dequant(acc_o, to_np(sx), to_np(sw), "bf16")
    assert_output_close(to_np(y0), y_o, "sq_w8a8_gemm")
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))


CHILD_STREAM = r'''
import numpy as np
import torch
import w8a8_int8_gemm_channel_b200 as sq
from oracle import oracle
from w8a8_int8_gemm_channel_b200 import workloads as wls
oracle.build()
bits = lambda t: t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
for (M, N, K) in [(1, 28672, 4096), (9, 28672, 1024), (17, 20480, 4112), (32, 19968, 2064), (32, 37888, 256)]:
    rng = np.random.default_rng(M + N + K)
    x = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
    s = rng.uniform(0.3, 8.0, K).astype(np.float32)
    wq = wls.random_int8((N, K), seed=N).numpy()
    sw = (rng.uniform(0.5, 2.0, N) * 1e-3).astype(np.float32)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.full((max(sq.sq_linear_workspace_size(M, N, K), 16),), 0xFF, dtype=torch.uint8, device="cuda")
    sq.sq_linear(x.cuda(), torch.from_numpy(s).cuda(), torch.from_numpy(wq).cuda(), torch.from_numpy(sw).cuda(), y, ws)
    torch.cuda.synchronize()
    y_o, _, _, _ = oracle.linear(bits(x), s, wq, sw, "bf16")
    assert np.array_equal(bits(y), y_o), (M, N, K)
st, code = sq.sq_device_status()
assert st == sq.SQ_OK, hex(code)
print("stream-ok")
'''


def test_weight_streaming_kernel_child_process():
    """With SQ_DECODE_SLAB=0 (read once per process, so in a child) the same
    few-token shapes take the weight-streaming kernel, whose tiles are summed
    across CTAs through the workspace; its outputs equal the oracle's."""
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SQ_DECODE_SLAB="0", PYTHONPATH=root)
    r = subprocess.run([sys.executable, "-c", CHILD_STREAM], cwd=root, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "stream-ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
