"""Parity of sq_linear's few-token path (M <= 128) against the CPU oracle.

For up to 128 tokens sq_linear runs the activation quantiser and then a GEMM
that streams the weight over every SM: the T x KB weight units (128 output
channels x 128 bytes of K each) are cut into one contiguous range per CTA, a
tile shared by several CTAs is summed through int32 partials in the
workspace, and the quantiser clears the tiles' counters.  The plan weighs
the streamed units per CTA against the reduction, whose cost grows with the
tokens: from 64 tokens, or with more tiles than SMs, ranges of whole tiles
(nothing summed) are chosen too.  (For at most 32
tokens on layers of about 19K-38K output channels the slab kernel runs
instead: tests/test_slab_gpu.py.)  With SQ_DECODE_STREAM=0 the split-K
cluster kernel runs instead (K split across the CTAs of a cluster, partials
summed through distributed shared memory); it is checked on the same shapes
in a child process.  Every output is
compared with the oracle's per-token quantisation, int32 GEMM and
dequantisation ("quant_llm_int8", "The architecture: every piece
explained"; "Understanding W8A8 INT8 LLM Quantization", "Why Activation
Quantization Is Hard, and How SmoothQuant Fixes It"), within 1 bf16 ulp /
1e-6 relative (in practice bit-exact).  Shapes cover one and several tiles a
CTA, tiles split over two and more CTAs, ragged N and K, fewer units than
SMs, and every token-tile width (32, 64, 128).
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


def _run(xt, s, wq, sw, out_dtype, ws=None):
    M, K = xt.shape
    N = wq.shape[0]
    y = torch.empty(M, N, dtype=out_dtype, device="cuda")
    need = sq.sq_linear_workspace_size(M, N, K)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    sq.sq_linear(xt.cuda(), to_dev(s), to_dev(wq), to_dev(sw), y, ws if need else None)
    torch.cuda.synchronize()
    return to_np(y)


@pytest.mark.parametrize("M,N,K", [
    (1, 6144, 4096),      # 1536 units over 148 CTAs: tiles split over two CTAs
    (8, 4096, 4096),
    (16, 28672, 4096),    # the slab kernel's shape (several whole tiles a CTA with SQ_DECODE_SLAB=0)
    (32, 4096, 14336),    # a tile spread over several CTAs
    (32, 4096, 4096),     # two CTAs a tile
    (40, 20480, 2048),    # more tiles than SMs: two whole tiles a CTA, nothing summed
    (64, 28672, 1024),
    (128, 6144, 1024),    # one CTA a tile, nothing summed
    (100, 2048, 8192),    # 128-token tiles shared by three CTAs
    (48, 1024, 8192),     # 64-token tiles shared by three CTAs
    (33, 4112, 4112),     # ragged N and K, 64-token tile
    (64, 1040, 3088),
    (100, 6144, 4096),    # 128-token tile
    (128, 4096, 4096),
    (5, 256, 256),        # fewer units than SMs
    (1, 16, 16),          # one unit
    (7, 144, 208),
])
def test_linear_few_tokens_bf16(oracle, M, N, K):
    xt, s, wq, sw = _case(M, N, K, torch.bfloat16, seed=M * 7 + N + K)
    y = _run(xt, s, wq, sw, torch.bfloat16)
    y_o, _, _, _ = oracle.linear(to_np(xt), s, wq, sw, "bf16")
    assert_output_close(y, y_o, f"y {M}x{N}x{K}")
    assert exact_fraction(y, y_o) == 1.0


@pytest.mark.parametrize("M,N,K", [(16, 256, 256), (3, 1024, 2048), (128, 512, 1024)])
def test_linear_few_tokens_f32(oracle, M, N, K):
    xt, s, wq, sw = _case(M, N, K, torch.float32, seed=M + N * 3 + K)
    y = _run(xt, s, wq, sw, torch.float32)
    y_o, _, _, _ = oracle.linear(to_np(xt), s, wq, sw, "f32")
    assert_output_close(y, y_o, f"y {M}x{N}x{K}")


def test_linear_few_tokens_dirty_workspace_and_repeats(oracle):
    """The workspace may hold anything before the call (the quantiser clears
    the tile counters; every partial slot is written before it is read), and
    consecutive calls on one workspace, with other shapes in between, agree."""
    M, N, K = 16, 6144, 4096
    xt, s, wq, sw = _case(M, N, K, torch.bfloat16, seed=99)
    need = max(sq.sq_linear_workspace_size(M, N, K), sq.sq_linear_workspace_size(32, 1040, 4096))
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")
    y1 = _run(xt, s, wq, sw, torch.bfloat16, ws)
    x2, s2, wq2, sw2 = _case(32, 1040, 4096, torch.bfloat16, seed=100)
    _run(x2, s2, wq2, sw2, torch.bfloat16, ws)
    y2 = _run(xt, s, wq, sw, torch.bfloat16, ws)
    y_o, _, _, _ = oracle.linear(to_np(xt), s, wq, sw, "bf16")
    assert np.array_equal(y1, y_o) and np.array_equal(y2, y_o)


CHILD_SPLITK = r'''
import numpy as np
import torch
import w8a8_int8_gemm_channel_b200 as sq
from oracle import oracle
from w8a8_int8_gemm_channel_b200 import workloads as wls
oracle.build()
bits = lambda t: t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
for (M, N, K) in [(1, 6144, 4096), (8, 4096, 4096), (32, 4096, 14336), (33, 4112, 4112), (100, 6144, 4096), (7, 144, 208)]:
    rng = np.random.default_rng(M * 3 + N + K)
    x = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
    s = rng.uniform(0.3, 8.0, K).astype(np.float32)
    wq = wls.random_int8((N, K), seed=N + 1).numpy()
    sw = (rng.uniform(0.5, 2.0, N) * 1e-3).astype(np.float32)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.full((max(sq.sq_linear_workspace_size(M, N, K), 16),), 0xFF, dtype=torch.uint8, device="cuda")
    sq.sq_linear(x.cuda(), torch.from_numpy(s).cuda(), torch.from_numpy(wq).cuda(), torch.from_numpy(sw).cuda(), y, ws)
    torch.cuda.synchronize()
    y_o, _, _, _ = oracle.linear(bits(x), s, wq, sw, "bf16")
    assert np.array_equal(bits(y), y_o), (M, N, K)
st, code = sq.sq_device_status()
assert st == sq.SQ_OK, hex(code)
print("splitk-ok")
'''


def test_split_k_kernel_child_process():
    """With SQ_DECODE_STREAM=0 (read once per process, so in a child) the
    few-token shapes take the split-K cluster kernel; its outputs equal the
    oracle's bit for bit."""
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SQ_DECODE_STREAM="0", PYTHONPATH=root)
    r = subprocess.run([sys.executable, "-c", CHILD_SPLITK], cwd=root, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "splitk-ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
