"""sq_linear_noalloc: the linear layer for callers that cannot allocate device
memory (a plugin whose host framework owns every allocation and passes in only
input and output buffers, or a serving loop where an allocation, which can
synchronise the device, is not allowed).  It runs the same kernels as
sq_linear with the library's fixed scratch array in place of a caller
workspace.

This file is named so that pytest collects it last.
"""
import pytest
import torch

import w8a8_int8_gemm_channel_b200 as sq
from w8a8_int8_gemm_channel_b200 import _build
from w8a8_int8_gemm_channel_b200 import workloads as wls
from tests.gpu_util import assert_output_close, to_np


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Checked on the host before anything is enqueued (no GPU needed)."""
    _build.build()
    lib = sq.lib()
    K = 4096
    M = sq.LINEAR_NOALLOC_SCRATCH_BYTES // K + 64  # workspace need exceeds the array
    assert sq.sq_linear_workspace_size(M, 256, K) > sq.LINEAR_NOALLOC_SCRATCH_BYTES
    a = 0x7F0000001000
    st = lib.sq_linear_noalloc(a, sq.SQ_BF16, a, a, a, M, 256, K, a, sq.SQ_BF16, None)
    assert st == sq.SQ_ERR_UNSUPPORTED
    st = lib.sq_linear_noalloc(None, sq.SQ_BF16, a, a, a, 8, 256, K, a, sq.SQ_BF16, None)
    assert st == sq.SQ_ERR_INVALID_ARG


def _case(M, N, K, seed):
    x = wls.random_tensor((M, K), seed, dtype=torch.bfloat16).cuda()
    x[:, 3] *= 60.0
    w = wls.random_tensor((N, K), seed + 1, dtype=torch.bfloat16, scale=0.02).cuda()
    xcal = wls.random_tensor((256, K), seed + 2, dtype=torch.bfloat16).cuda()
    xcal[:, 3] *= 60.0
    ax = sq.calibrate(xcal)
    s, wq, sw = sq.prepare_weight(ax, w, 0.5)
    return x, s, wq, sw


@pytest.mark.gpu
def test_noalloc_matches_sq_linear_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _build.build()
    # a prefill-sized call, a few-token call (the weight-streaming GEMM, whose
    # tile counters and partial sums also live in the scratch array) and one in between
    shapes = [(300, 512, 2048, 101), (16, 1040, 4096, 303), (77, 272, 4112, 202)]
    cases = [_case(M, N, K, seed) for (M, N, K, seed) in shapes]
    outs = [torch.empty(x.shape[0], wq.shape[0], dtype=torch.bfloat16, device="cuda") for (x, s, wq, sw) in cases]
    # first round: the calls back to back, sharing the library's scratch array
    for (x, s, wq, sw), y in zip(cases, outs):
        sq.sq_linear_noalloc(x, s, wq, sw, y)
    torch.cuda.synchronize()
    # second round: nothing is allocated, on the device or in torch's cache
    outs2 = [torch.empty_like(y) for y in outs]
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for (x, s, wq, sw), y in zip(cases, outs2):
        sq.sq_linear_noalloc(x, s, wq, sw, y)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0, "torch memory changed across allocation-free calls"
    assert free1 == free0, f"device free memory changed across allocation-free calls: {free0} -> {free1}"
    for y, y2 in zip(outs, outs2):
        assert torch.equal(y, y2)
    for (x, s, wq, sw), y in zip(cases, outs):
        ref = sq.linear(x, s, wq, sw, out_dtype=torch.bfloat16)  # caller workspace
        torch.cuda.synchronize()
        assert_output_close(to_np(y), to_np(ref), "sq_linear_noalloc vs sq_linear")
    st, code = sq.sq_device_status()
    assert st == sq.SQ_OK, f"device error word {code:#x}"
