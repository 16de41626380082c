"""Parity of the fused RMSNorm + per-token quantiser (sq_fold_gamma,
sq_rmsnorm_quant) against the CPU oracle on the same seeded bytes.

Source: "Understanding W8A8 INT8 LLM Quantization", section "Where the
outlier actually comes from" (RMSNorm, and SmoothQuant dividing gamma by s).

* the folded gamma g = gamma / s: bit-exact;
* per token, 1/RMS, the scale and the codes: bit-exact against the oracle's
  result.  The summation order of the squares is not fixed, so for a token
  whose fp64 1/RMS lies within the order-independence bound of an fp32
  rounding midpoint the oracle also computes the whole result for the other
  rounding, and the device may match either.  Every expected value comes from
  the oracle on the input bytes alone.
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


def _match_candidates(cand, xq, sx, rinv=None):
    """Every token of the device result equals the oracle's result, or, for a
    flagged token, the oracle's alternate result.  Returns the number of
    tokens that matched the alternate."""
    M = sx.shape[0]
    alt_rows = 0
    for m in range(M):
        prim = np.array_equal(xq[m], cand["xq"][m]) and sx[m].view(np.uint32) == cand["sx"][m].view(np.uint32)
        if rinv is not None:
            prim = prim and rinv[m].view(np.uint32) == cand["rinv"][m].view(np.uint32)
        if prim:
            continue
        assert cand["near"][m], f"token {m}: differs from the oracle and 1/RMS is not near a rounding midpoint"
        alt = np.array_equal(xq[m], cand["xq_alt"][m]) and \
            sx[m].view(np.uint32) == cand["sx_alt"][m].view(np.uint32)
        if rinv is not None:
            alt = alt and rinv[m].view(np.uint32) == cand["rinv_alt"][m].view(np.uint32)
        assert alt, f"token {m}: matches neither rounding of 1/RMS"
        alt_rows += 1
    return alt_rows


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
    cand = oracle.rmsnorm_quant_candidates(to_np(h), g_o, eps)
    assert cand["near"].mean() < 0.05  # flagged tokens are rare: about (K + 16) 2^-27 each
    _match_candidates(cand, to_np(xq), to_np(sx), to_np(rinv))


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
    _match_candidates(oracle.rmsnorm_quant_candidates(to_np(h), g_o, 1e-5), to_np(xq), to_np(sx), to_np(rinv))


def test_rmsnorm_quant_at_a_rounding_midpoint(oracle):
    """A token whose 1/RMS sits 2^-48 above the fp32 midpoint 1 + 2^-24: the
    row [4 - 2^-22, 0, ..., 0] of 16 values has mean square (1 - 2^-24)^2
    exactly, so 1/RMS = 1 + 2^-24 + 2^-48 + ... (flagged by the oracle, which
    also supplies the result for rinv = 1).  The device must give one of the
    two oracle results; the rows around it are ordinary."""
    K = 16
    h = np.zeros((3, K), np.float32)
    h[0] = np.linspace(-2.0, 3.0, K, dtype=np.float32)
    h[1, 0] = np.float32(4.0 - 2.0 ** -22)
    h[2] = np.linspace(0.5, -7.0, K, dtype=np.float32)
    g_o = np.linspace(0.5, 2.0, K, dtype=np.float32)
    cand = oracle.rmsnorm_quant_candidates(h, g_o, 0.0)
    assert cand["near"].tolist() == [False, True, False]
    xq = torch.empty(3, K, dtype=torch.int8, device="cuda")
    sx = torch.empty(3, device="cuda")
    rinv = torch.empty(3, device="cuda")
    sq.sq_rmsnorm_quant(to_dev(h), to_dev(g_o), 0.0, xq, sx, rinv)
    _match_candidates(cand, to_np(xq), to_np(sx), to_np(rinv))
