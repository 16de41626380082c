"""sq_linear captured in a CUDA graph: a decode-shaped chain of calls (the
few-row and cluster quantisers, the weight-streaming and slab GEMMs, each
launch with programmatic dependent launch) recorded once and replayed.

Replays must equal the oracle on the inputs the static buffers hold at replay
time ("quant_llm_int8", "The architecture: every piece explained";
"Understanding W8A8 INT8 LLM Quantization", "Inter-Token Latency (ITL)": at
decode the same layer calls repeat every step, which is what a graph
replays), and equal the eager calls bit for bit.
"""
import numpy as np
import pytest
import torch

import w8a8_int8_gemm_channel_b200 as sq
from w8a8_int8_gemm_channel_b200 import workloads as wls
from tests.gpu_util import to_np

pytestmark = pytest.mark.gpu

# (M, N, K): few-row quantiser + weight stream; cluster quantiser + weight
# stream; slab GEMM; a 64-token call whose plan gives each CTA whole tiles
CHAIN = [(1, 6144, 1024), (8, 4096, 14336), (32, 20480, 1024), (64, 1024, 2048)]


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w8a8_int8_gemm_channel_b200 import _build

    _build.build()
    yield
    st, code = sq.sq_device_status()
    assert st == sq.SQ_OK, f"device error word {code:#x}"


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _inputs(M, K, seed):
    x = wls.random_tensor((M, K), seed, dtype=torch.bfloat16)
    x[:, 5] *= 60.0
    return x


def test_decode_chain_in_a_cuda_graph(oracle):
    calls = []
    for i, (M, N, K) in enumerate(CHAIN):
        rng = np.random.default_rng(100 + i)
        s = torch.from_numpy(rng.uniform(0.3, 8.0, K).astype(np.float32)).cuda()
        wq = wls.random_int8((N, K), seed=200 + i).cuda()
        sw = torch.from_numpy((rng.uniform(0.5, 2.0, N) * 1e-3).astype(np.float32)).cuda()
        x = _inputs(M, K, 300 + i).cuda()
        y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(max(sq.sq_linear_workspace_size(M, N, K), 16), dtype=torch.uint8, device="cuda")
        calls.append((x, s, wq, sw, y, ws))

    def run():
        for (x, s, wq, sw, y, ws) in calls:
            sq.sq_linear(x, s, wq, sw, y, ws)

    # eager first (also loads the kernels and sets their attributes before capture)
    run()
    torch.cuda.synchronize()
    eager = [_bits(c[4]) for c in calls]

    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        run()
    for c in calls:
        c[4].fill_(0)
    g.replay()
    torch.cuda.synchronize()
    for i, c in enumerate(calls):
        assert np.array_equal(_bits(c[4]), eager[i]), f"replay differs from the eager call {CHAIN[i]}"

    # new inputs in the same buffers: the next replay follows them
    for i, c in enumerate(calls):
        M, N, K = CHAIN[i]
        c[0].copy_(_inputs(M, K, 400 + i).cuda())
    g.replay()
    g.replay()  # twice: the tile counters are cleared by every replay's quantisers
    torch.cuda.synchronize()
    for i, (x, s, wq, sw, y, ws) in enumerate(calls):
        y_o, _, _, _ = oracle.linear(_bits(x), to_np(s), to_np(wq), to_np(sw), "bf16")
        assert np.array_equal(_bits(y), y_o), f"replay vs oracle {CHAIN[i]}"
    del g
