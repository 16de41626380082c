"""Parity of the GEMM with a workspace (sq_w8a8_gemm_ws, and sq_linear with
a full workspace):

* up to 128 tokens: the weight-streaming kernel, which splits the weight
  over every SM and sums tiles shared by several CTAs through int32
  partials;
* more tokens: the pair kernel; with SQ_GEMM_SK=1 (off by default, tested in
  a child process) the output tiles that do not fill whole rounds of the
  CTA pairs are split along K over all pairs (stream-K), and a tile shared
  by several pairs is summed through int32 partials.

Integer partial sums are exact in any order, so the outputs must equal
sq_w8a8_gemm's (data-parallel tiles) bit for bit, and the oracle's
("quant_llm_int8", "The architecture: every piece explained") within the
usual 1 bf16 ulp / 1e-6 (in practice bit-exact).  Shapes cover fewer tiles
than pairs, one full round plus a partial one, several full rounds, ragged
M, N and K, and a dirty workspace.
"""
import numpy as np
import pytest
import torch

import w8a8_int8_gemm_channel_b200 as sq
from w8a8_int8_gemm_channel_b200 import workloads as wls
from tests.gpu_util import assert_output_close, to_dev, to_np

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


def _operands(M, N, K, seed):
    xq = wls.random_int8((M, K), seed).cuda()
    wq = wls.random_int8((N, K), seed + 1).cuda()
    g = torch.Generator().manual_seed(seed)
    sx = (torch.rand(M, generator=g) * 0.05 + 1e-3).cuda()
    sw = (torch.rand(N, generator=g) * 1e-3 + 1e-5).cuda()
    return xq, sx, wq, sw


@pytest.mark.parametrize("M,N,K", [
    (300, 528, 1040),      # 6 tiles, fewer than the pairs: every tile split along K
    (1024, 6144, 4096),    # 96 tiles: one round plus a partial one, all stream-K
    (1000, 6160, 2064),    # ragged M, N and K
    (4096, 4096, 4096),    # 256 tiles: three full rounds, the last two stream-K
    (257, 784, 4112),
    (129, 16, 16),         # one tile, one k block
])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_gemm_ws_equals_gemm(M, N, K, out):
    xq, sx, wq, sw = _operands(M, N, K, seed=M + N + K)
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    y0 = torch.empty(M, N, dtype=dt, device="cuda")
    y1 = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
    sq.sq_w8a8_gemm(xq, sx, wq, sw, y0)
    ws = torch.full((sq.sq_w8a8_gemm_workspace_size(M, N, K),), 0xFF, dtype=torch.uint8, device="cuda")
    sq.sq_w8a8_gemm_ws(xq, sx, wq, sw, y1, ws)
    y2 = torch.empty_like(y1)
    sq.sq_w8a8_gemm_ws(xq, sx, wq, sw, y2, ws)  # the same workspace again
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16) if dt == torch.bfloat16 else y0.view(torch.int32),
                       y1.view(torch.int16) if dt == torch.bfloat16 else y1.view(torch.int32))
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("M,N,K", [(1024, 6144, 4096), (300, 528, 1040), (2048, 1040, 8192)])
def test_gemm_ws_against_oracle_rows_and_columns(oracle, M, N, K):
    xq, sx, wq, sw = _operands(M, N, K, seed=3 * M + N)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    sq.sq_w8a8_gemm_ws(xq, sx, wq, sw, y)
    torch.cuda.synchronize()
    xq_h, wq_h, sx_h, sw_h = to_np(xq), to_np(wq), to_np(sx), to_np(sw)
    rng = np.random.default_rng(M)
    ms = np.union1d(rng.choice(M, 5, replace=False), [0, M - 1])
    ns = np.union1d(rng.choice(N, 5, replace=False), [0, N - 1])
    y_h = to_np(y)
    rows = oracle.dequant(oracle.gemm_i32(xq_h[ms], wq_h), sx_h[ms], sw_h, "bf16")
    cols = oracle.dequant(oracle.gemm_i32(xq_h, wq_h[ns]), sx_h, sw_h[ns], "bf16")
    assert_output_close(y_h[ms], rows, "rows")
    assert_output_close(y_h[:, ns], cols, "columns")


@pytest.mark.parametrize("M,N,K", [(1024, 4096, 4096), (2048, 10240, 1024), (513, 2064, 2048)])
def test_linear_full_workspace_against_oracle(oracle, M, N, K):
    """sq_linear with sq_linear_workspace_size bytes (the quantiser clears the
    GEMM's counters) against the oracle, on whole rows and columns, and equal
    to sq_linear with only the codes' and scales' room (data-parallel GEMM)."""
    g = torch.Generator().manual_seed(M + K)
    x = torch.randn(M, K, generator=g)
    x[:, 5] *= 60.0
    xt = x.to(torch.bfloat16)
    s = (torch.rand(K, generator=g) * 4 + 0.3).numpy().astype(np.float32)
    wq = wls.random_int8((N, K), seed=N).numpy()
    sw = (torch.rand(N, generator=g).numpy() * 1e-3 + 1e-5).astype(np.float32)
    full = sq.sq_linear_workspace_size(M, N, K)
    minimum = (M * K + 255) // 256 * 256 + (4 * M + 255) // 256 * 256
    ys = []
    for nbytes in (full, minimum):
        ws = torch.full((nbytes,), 0x5A, dtype=torch.uint8, device="cuda")
        y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        sq.sq_linear(xt.cuda(), to_dev(s), to_dev(wq), to_dev(sw), y, ws)
        ys.append(y)
    torch.cuda.synchronize()
    assert torch.equal(ys[0].view(torch.int16), ys[1].view(torch.int16))
    xq_o, sx_o = oracle.quant_act(to_np(xt), s)
    rng = np.random.default_rng(N)
    ms = np.union1d(rng.choice(M, 5, replace=False), [0, M - 1])
    ns = np.union1d(rng.choice(N, 5, replace=False), [0, N - 1])
    y_h = to_np(ys[0])
    rows = oracle.dequant(oracle.gemm_i32(xq_o[ms], wq), sx_o[ms], sw, "bf16")
    cols = oracle.dequant(oracle.gemm_i32(xq_o, wq[ns]), sx_o, sw[ns], "bf16")
    assert_output_close(y_h[ms], rows, "rows")
    assert_output_close(y_h[:, ns], cols, "columns")


CHILD_SK = r'''
import torch
import w8a8_int8_gemm_channel_b200 as sq
from w8a8_int8_gemm_channel_b200 import workloads as wls
for (M, N, K) in [(300, 528, 1040), (1024, 6144, 4096), (1000, 6160, 2064), (4096, 4096, 4096), (129, 16, 16)]:
    xq = wls.random_int8((M, K), M).cuda()
    wq = wls.random_int8((N, K), N).cuda()
    sx = torch.rand(M).cuda() * 0.05 + 1e-3
    sw = torch.rand(N).cuda() * 1e-3 + 1e-5
    y0 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    y1 = torch.empty_like(y0)
    sq.sq_w8a8_gemm(xq, sx, wq, sw, y0)
    ws = torch.full((sq.sq_w8a8_gemm_workspace_size(M, N, K),), 0xFF, dtype=torch.uint8, device="cuda")
    sq.sq_w8a8_gemm_ws(xq, sx, wq, sw, y1, ws)
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16)), (M, N, K)
st, code = sq.sq_device_status()
assert st == sq.SQ_OK, hex(code)
print("stream-k-ok")
'''


def test_stream_k_tail_child_process():
    """The stream-K tail of the pair GEMM (off by default, SQ_GEMM_SK=1 turns
    it on; read once per process, so in a child): equal to the data-parallel
    GEMM bit for bit."""
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SQ_GEMM_SK="1", PYTHONPATH=root)
    r = subprocess.run([sys.executable, "-c", CHILD_SK], cwd=root, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "stream-k-ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
