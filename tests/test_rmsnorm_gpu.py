"""Parity of the fused RMSNorm + per-token quantiser (sq_fold_gamma,
sq_rmsnorm_quant) against the CPU oracle on the same seeded bytes.

Source: "Understanding W8A8 INT8 LLM Quantization", section "Where the
outlier actually comes from" (RMSNorm, and SmoothQuant dividing gamma by s).

* the folded gamma g = gamma / s: bit-exact;
* 1/RMS per token: bit-exact, or one fp32 ulp apart where the fp64 value
  lies at an fp32 rounding midpoint (the summation order of the squares is
  not fixed);
* given the device's 1/RMS, the scales and codes: bit-exact.
"""
import numpy as np
import pytest
import torch

import w8a8_int8_gemm_channel_b200 as sq
from tests.gpu_util import assert_bits_equal, to_dev, to_np

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


def _rows(M, K, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    h = torch.randn(M, K, generator=g) * torch.exp(torch.randn(M, 1, generator=g) * 2.0)
    out = torch.randperm(K, generator=g)[: max(1, K // 1000)]
    h[:, out] *= 60.0
    if M > 4:
        h[1] = 0.0                    # zero token
        h[2] = 0.25                   # constant token
        h[3] *= 1e-30                 # tiny token (squares far below fp32 range, fine in fp64)
        h[4] *= 1e25                  # huge token
    return h.to(dtype)


def _check_rinv(r_dev, r_ora, h, eps, oracle):
    same = r_dev.view(np.uint32) == r_ora.view(np.uint32)
    if same.all():
        return
    ref = oracle.rmsnorm_rinv_fp64(to_np(h)[~same], eps)
    lo = np.minimum(r_dev[~same], r_ora[~same]).astype(np.float64)
    hi = np.maximum(r_dev[~same], r_ora[~same]).astype(np.float64)
    assert (np.nextafter(lo.astype(np.float32), np.float32(np.inf)).astype(np.float64) == hi).all()
    mid = (lo + hi) / 2
    assert (np.abs(ref - mid) <= mid * 2.0 ** -40).all(), "1/RMS differs away from a rounding midpoint"


@pytest.mark.parametrize("M,K,dtype,eps", [(1, 16, torch.float32, 1e-5), (6, 256, torch.float32, 0.0),
                                           (5, 4096, torch.bfloat16, 1e-5), (37, 4112, torch.bfloat16, 1e-6),
                                           (130, 14336, torch.bfloat16, 1e-5), (9, 8192, torch.float32, 1e-5),
                                           (3, 32768, torch.bfloat16, 1e-5), (4096, 4096, torch.bfloat16, 1e-5)])
def test_rmsnorm_quant(oracle, M, K, dtype, eps):
    rng = np.random.default_rng(M * 131 + K)
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float32)
    gamma[rng.choice(K, max(1, K // 1000), replace=False)] *= 60.0
    s = rng.uniform(0.3, 30.0, K).astype(np.float32)
    g = torch.empty(K, device="cuda")
    sq.sq_fold_gamma(to_dev(gamma), to_dev(s), g)
    g_o = oracle.fold_gamma(gamma, s)
    assert_bits_equal(to_np(g), g_o, "folded gamma")

    h = _rows(M, K, dtype, seed=M + K)
    xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, device="cuda")
    rinv = torch.empty(M, device="cuda")
    sq.sq_rmsnorm_quant(h.cuda(), g, eps, xq, sx, rinv)
    h_np = to_np(h)
    _, _, r_o = oracle.rmsnorm_quant(h_np, g_o, eps)
    _check_rinv(to_np(rinv), r_o, h, eps, oracle)
    q_o, sx_o, _ = oracle.rmsnorm_quant(h_np, g_o, eps, rinv_in=to_np(rinv))
    assert_bits_equal(to_np(sx), sx_o, "sx")
    assert_bits_equal(to_np(xq), q_o, "xq")


def test_rmsnorm_quant_without_rinv_output(oracle):
    M, K = 33, 2048
    h = _rows(M, K, torch.bfloat16, seed=7)
    g_o = np.random.default_rng(8).uniform(0.2, 2.0, K).astype(np.float32)
    xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, device="cuda")
    sq.sq_rmsnorm_quant(h.cuda(), to_dev(g_o), 1e-5, xq, sx)
    rinv = torch.empty(M, device="cuda")
    xq2 = torch.empty_like(xq)
    sx2 = torch.empty_like(sx)
    sq.sq_rmsnorm_quant(h.cuda(), to_dev(g_o), 1e-5, xq2, sx2, rinv)
    assert torch.equal(xq, xq2) and torch.equal(sx, sx2)
    q_o, sx_o, _ = oracle.rmsnorm_quant(to_np(h), g_o, 1e-5, rinv_in=to_np(rinv))
    assert_bits_equal(to_np(xq), q_o, "xq")
