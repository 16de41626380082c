"""Parity of the gated feed-forward activation fused into the per-token
quantiser (sq_silu_mul_quant) against the CPU oracle on the same seeded bytes.

Sources: "Understanding W8A8 INT8 LLM Quantization", section "Inter-Token
Latency (ITL)" (the per-token quantisation is memory-bound work), and "How
does SmoothQuant int8 LLM calibration work...", section "Hardware
Acceleration and Inference Optimization Strategies" (fuse the feed-forward
network with its neighbours).

Everything is bit-exact: the activation h = SiLU(gate) * up (stored when
asked for), the per-token scales and the codes.  The kernel's fast path
(hardware exp2 and reciprocal approximations) must give the definition's bf16
h wherever it does not fall back; the exhaustive test runs every finite bf16
gate value through it.
"""
import numpy as np
import pytest
import torch

import w8a8_int8_gemm_channel_b200 as sq
from w8a8_int8_gemm_channel_b200 import workloads as wlmod
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


def _run(gu_np, s_np, dtype, with_h=True):
    gu = to_dev(gu_np, dtype)
    s = to_dev(s_np)
    M, I2 = gu.shape
    I = I2 // 2
    xq = torch.empty(M, I, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    h = torch.empty(M, I, dtype=dtype, device="cuda") if with_h else None
    sq.sq_silu_mul_quant(gu, s, xq, sx, h)
    torch.cuda.synchronize()
    return to_np(xq), to_np(sx), (to_np(h) if with_h else None)


def _check(gu_np, s_np, dtype, oracle, what):
    xq, sx, h = _run(gu_np, s_np, dtype)
    q_o, sx_o, h_o = oracle.silu_mul_quant(gu_np, s_np)
    if dtype == torch.bfloat16:
        h_o = (h_o.view(np.uint32) >> 16).astype(np.uint16)  # exact: h is a bf16 value
    assert_bits_equal(h, h_o, f"{what}: h")
    assert_bits_equal(sx, sx_o, f"{what}: sx")
    assert_bits_equal(xq, q_o, f"{what}: codes")


def _smooth(I, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.rand(I, generator=g) * 1.5 + 0.5).numpy().astype(np.float32)


# (M, I): every configuration the launcher picks -- an exact fit with the bf16
# bound (I = 4096, enough rows), bounds-checked rows (few rows, ragged I),
# the fp32 bound (I = 14336, 16384), 16 chunks a lane (I = 32768)
SHAPES = [
    (1, 4096), (37, 4096), (1536, 4096), (5, 4112), (64, 14336), (320, 16384), (8, 32768), (300, 32768),
]


@pytest.mark.parametrize("M,I", SHAPES)
def test_silu_mul_quant_bf16_parity(M, I, oracle):
    wl = wlmod.WORKLOADS["llama3_8b_mlp"]
    lin = wlmod.Linear("down", 4096, I, act="silu_mul")
    gu = to_np(wlmod.gate_up(wl, lin, M, "x", dtype="bf16"))
    _check(gu, _smooth(I, 7 + I), torch.bfloat16, oracle, f"bf16 {M}x{I}")


@pytest.mark.parametrize("M,I", [(1, 16), (3, 48), (64, 1024), (200, 4096), (600, 4096), (9, 16384)])
def test_silu_mul_quant_f32_parity(M, I, oracle):
    g = torch.Generator().manual_seed(M * 131 + I)
    gu = (torch.randn(M, 2 * I, generator=g) * 3.0).numpy().astype(np.float32)
    _check(gu, _smooth(I, I), torch.float32, oracle, f"f32 {M}x{I}")


def test_every_bf16_gate_value(oracle):
    """All 65536 bf16 patterns as gates (non-finite ones replaced by 0), each
    against three up values: a random one in [-1, 1] (so that h stays finite,
    as the contract requires), 1.0, and 2^-120 (h subnormal or zero)."""
    I = 4096
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = (pats & 0x7F80) != 0x7F80
    gate = np.where(finite, pats, 0).astype(np.uint16).reshape(16, I)
    rng = np.random.default_rng(60)
    ups = [
        (np.asarray(rng.uniform(-1.0, 1.0, (16, I)), np.float32).view(np.uint32) >> 16).astype(np.uint16),
        np.full((16, I), 0x3F80, np.uint16),
        np.full((16, I), 0x0380, np.uint16),  # 2^-120
    ]
    gu = np.concatenate([np.concatenate([gate, u], axis=1) for u in ups], axis=0)
    _check(gu, np.ones(I, np.float32), torch.bfloat16, oracle, "all bf16 gates")


def test_near_bf16_midpoints(oracle):
    """Gate/up pairs whose exact fp32 product lies within 64 bit patterns of a
    bf16 rounding midpoint (the fast path must fall back for them), at
    midpoints, and at the window's edges."""
    rng = np.random.default_rng(61)
    n = 1 << 24
    g = (np.asarray(rng.uniform(-16.0, 16.0, n), np.float32).view(np.uint32) >> 16).astype(np.uint16)
    u = (np.asarray(rng.standard_normal(n), np.float32).view(np.uint32) >> 16).astype(np.uint16)
    silu = oracle.silu_f32((g.astype(np.uint32) << 16).view(np.float32))
    v = silu * (u.astype(np.uint32) << 16).view(np.float32)  # one fp32 multiply, as the definition
    low = v.view(np.uint32) & 0xFFFF
    dist = np.abs(low.astype(np.int64) - 0x8000)
    pick = np.flatnonzero(dist <= 80)
    I = 4096
    rows = max(1, pick.size // I)
    pick = pick[: rows * I]
    assert rows >= 4, pick.size
    gate = g[pick].reshape(rows, I)
    up = u[pick].reshape(rows, I)
    _check(np.concatenate([gate, up], axis=1), np.ones(I, np.float32), torch.bfloat16, oracle, "near midpoints")


def test_edge_rows(oracle):
    """Zero gates, zero ups, gates far below -16 (fallback) and above 88 (SiLU
    is the gate itself), huge products (infinite h is outside the contract, so
    kept finite), a lone outlier channel, and h not stored."""
    I = 4096
    rng = np.random.default_rng(62)
    gu = (rng.standard_normal((8, 2 * I)) * 2.0).astype(np.float32)
    gu[0, :I] = 0.0
    gu[1, I:] = 0.0
    gu[2, :I] = -rng.uniform(16.0, 200.0, I)
    gu[3, :I] = rng.uniform(88.0, 1e4, I)
    gu[4, I:] *= 1e30
    gu[5, :] *= 1e-30
    gu[6, 17] = 50.0
    gu[6, I + 17] = 3000.0
    gu[7, :I] = -16.0
    bf = (gu.view(np.uint32) >> 16).astype(np.uint16)  # truncation: any bf16 pattern will do
    s = _smooth(I, 3)
    _check(bf, s, torch.bfloat16, oracle, "edge rows bf16")
    xq, sx, _ = _run(bf, s, torch.bfloat16, with_h=False)
    q_o, sx_o, _ = oracle.silu_mul_quant(bf, s)
    assert_bits_equal(sx, sx_o, "edge rows without h: sx")
    assert_bits_equal(xq, q_o, "edge rows without h: codes")
    _check(gu, s, torch.float32, oracle, "edge rows f32")


def test_fused_equals_unfused_quantiser(oracle):
    """The fused call's codes equal sq_quant_act run on the h it stores: the
    fusion changes where h lives, not the quantisation."""
    M, I = 256, 14336
    wl = wlmod.WORKLOADS["llama3_8b_mlp"]
    gu = wlmod.gate_up(wl, wl.linears[1], M, "x", device="cuda", dtype="bf16")
    s = to_dev(_smooth(I, 11))
    xq = torch.empty(M, I, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, device="cuda")
    h = torch.empty(M, I, dtype=torch.bfloat16, device="cuda")
    sq.sq_silu_mul_quant(gu, s, xq, sx, h)
    xq2 = torch.empty_like(xq)
    sx2 = torch.empty_like(sx)
    sq.sq_quant_act(h, s, xq2, sx2)
    torch.cuda.synchronize()
    assert torch.equal(xq, xq2) and torch.equal(sx, sx2)


def test_full_size_sampled(oracle):
    """The Llama-3-8B down-projection input at M = 8192 (I = 14336), in the
    launch configuration the benchmark times: sampled rows against the oracle."""
    M, I = 8192, 14336
    wl = wlmod.WORKLOADS["llama3_8b_mlp"]
    gu = wlmod.gate_up(wl, wl.linears[1], M, "x", device="cuda", dtype="bf16")
    s_np = _smooth(I, 12)
    s = to_dev(s_np)
    xq = torch.empty(M, I, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, device="cuda")
    sq.sq_silu_mul_quant(gu, s, xq, sx)
    torch.cuda.synchronize()
    rows = np.random.default_rng(63).choice(M, 96, replace=False)
    rows.sort()
    q_o, sx_o, _ = oracle.silu_mul_quant(to_np(gu[torch.from_numpy(rows).cuda()]), s_np)
    assert_bits_equal(to_np(sx)[rows], sx_o, "full size: sx")
    assert_bits_equal(to_np(xq)[rows], q_o, "full size: codes")
