"""GPU parity: every stage of the CUDA path against the CPU oracle on the same
seeded bytes, through the C ABI (via the thin Python binding).

Sizes span several tiles with ragged tails (M not a multiple of the 128-row
tile, N not a multiple of the 256-column tile, K not a multiple of the 128-byte
stage), the degenerate cases (one token, a zero token row, a zero input
channel, a zero weight row, a large-magnitude row) and the smallest legal K.
"""
import numpy as np
import pytest
import torch

import w8a8_int8_gemm_channel_b200 as sq
from w8a8_int8_gemm_channel_b200 import workloads as wls
from tests.gpu_util import (assert_bits_equal, assert_output_close, assert_smooth_factors,
                            exact_fraction, to_dev, to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w8a8_int8_gemm_channel_b200 import _build

    _build.build()
    sq.lib()
    yield
    st, code = sq.sq_device_status()
    assert st == sq.SQ_OK, f"device error word {code:#x}"


def rand(shape, seed, dtype=torch.bfloat16, scale=1.0):
    return wls.random_tensor(shape, seed, dtype=dtype, scale=scale)


# ---------------------------------------------------------------------------
# the small workload, stage by stage (fp32 in, fp32 out)
# ---------------------------------------------------------------------------

def test_small_workload_all_stages(oracle):
    wl = wls.WORKLOADS["small"]
    lin = wl.linears[0]
    xcal = wls.calibration(wl, lin)
    w = wls.weight(wl, lin)
    x = wls.inputs(wl, lin, wl.Ms[0])
    ax_o, aw_o, s_o, wq_o, sw_o = oracle.prepare(to_np(xcal), to_np(w), wl.alpha)

    ax = sq.calibrate(xcal.cuda())
    assert_bits_equal(to_np(ax), ax_o, "ax")
    s = torch.empty(lin.K, device="cuda")
    aw = torch.empty(lin.K, device="cuda")
    sq.sq_smooth_factors(ax, w.cuda(), wl.alpha, s, aw)
    assert_bits_equal(to_np(aw), aw_o, "aw")
    assert_smooth_factors(to_np(s), s_o, ax_o, aw_o, wl.alpha)
    # downstream stages get the oracle's s on both sides
    s_np = s_o
    s = to_dev(s_o)
    wq = torch.empty(lin.N, lin.K, dtype=torch.int8, device="cuda")
    sw = torch.empty(lin.N, device="cuda")
    sq.sq_smooth_quant_weight(w.cuda(), s, wq, sw)
    assert_bits_equal(to_np(wq), wq_o, "wq")
    assert_bits_equal(to_np(sw), sw_o, "sw")

    M = x.shape[0]
    xq = torch.empty(M, lin.K, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, device="cuda")
    sq.sq_quant_act(x.cuda(), s, xq, sx)
    xq_o, sx_o = oracle.quant_act(to_np(x), s_np)
    assert_bits_equal(to_np(xq), xq_o, "xq")
    assert_bits_equal(to_np(sx), sx_o, "sx")

    acc = torch.empty(M, lin.N, dtype=torch.int32, device="cuda")
    sq.sq_w8a8_gemm_s32(xq, wq, acc)
    acc_o = oracle.gemm_i32(xq_o, wq_o)
    assert_bits_equal(to_np(acc), acc_o, "acc")

    y = torch.empty(M, lin.N, device="cuda")
    sq.sq_w8a8_gemm(xq, sx, wq, sw, y)
    y_o = oracle.dequant(acc_o, sx_o, sw_o, "f32")
    assert_output_close(to_np(y), y_o, "y")
    assert exact_fraction(to_np(y), y_o) == 1.0

    y2 = sq.linear(x.cuda(), s, wq, sw, out_dtype=torch.float32)
    assert_bits_equal(to_np(y2), to_np(y), "sq_linear vs stages")


# ---------------------------------------------------------------------------
# calibration absmax
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,K,dtype", [(1, 16, torch.bfloat16), (7, 48, torch.float32),
                                       (1000, 4112, torch.bfloat16), (333, 272, torch.float32),
                                       (70000, 64, torch.bfloat16)])
def test_calib_absmax(oracle, T, K, dtype):
    x = rand((T, K), seed=T * 7 + K, dtype=dtype, scale=3.0)
    if K > 20:
        x[:, 5] = 0  # a zero channel
    ax = torch.zeros(K, device="cuda")
    sq.sq_calib_absmax(x.cuda(), ax)
    torch.cuda.synchronize()
    assert_bits_equal(to_np(ax), oracle.calib_absmax(to_np(x)), "ax")


def test_calib_absmax_accumulates_over_batches(oracle):
    x = rand((513, 256), seed=11, scale=5.0)
    ax = sq.calibrate([x[:200].cuda(), x[200:].cuda()])
    assert_bits_equal(to_np(ax), oracle.calib_absmax(to_np(x)), "ax over batches")


def test_calib_absmax_row_stride(oracle):
    """ldx > K: a column slice of a wider row-major buffer."""
    T, K, ldx = 300, 128, 192
    full = rand((T, ldx), seed=12, scale=2.0).cuda()
    ax = torch.zeros(K, device="cuda")
    st = sq.lib().sq_calib_absmax(full.data_ptr(), sq.SQ_BF16, T, K, ldx, ax.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
    assert st == sq.SQ_OK
    torch.cuda.synchronize()
    assert_bits_equal(to_np(ax), oracle.calib_absmax(to_np(full[:, :K])), "ax strided")


# ---------------------------------------------------------------------------
# smoothing factors
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("alpha", [0.0, 0.5, 0.8, 0.85, 1.0])
@pytest.mark.parametrize("N,K,dtype", [(16, 16, torch.float32), (300, 4112, torch.bfloat16)])
def test_smooth_factors(oracle, alpha, N, K, dtype):
    rng = np.random.default_rng(N + K)
    ax_np = np.abs(rng.standard_normal(K)).astype(np.float32) * 10
    ax_np[rng.integers(0, K, 3)] *= 60
    ax_np[0] = 0.0  # dead calibration channel
    w = rand((N, K), seed=N * K, dtype=dtype, scale=0.02)
    if K > 3:
        w[:, 2] = 0  # dead weight input channel
    s = torch.empty(K, device="cuda")
    aw = torch.empty(K, device="cuda")
    sq.sq_smooth_factors(to_dev(ax_np), w.cuda(), alpha, s, aw)
    aw_o = oracle.weight_in_absmax(to_np(w))
    s_o = oracle.smooth_factors(ax_np, aw_o, alpha)
    assert_bits_equal(to_np(aw), aw_o, "aw")
    assert_smooth_factors(to_np(s), s_o, ax_np, aw_o, alpha)
    assert float(to_np(s)[0]) == 1.0 and (K <= 3 or float(to_np(s)[2]) == 1.0)


# ---------------------------------------------------------------------------
# weight and activation quantisers
# ---------------------------------------------------------------------------

QUANT_SHAPES = [(1, 16, torch.float32), (3, 48, torch.bfloat16), (37, 4096, torch.bfloat16),
                (130, 4112, torch.bfloat16), (5, 14336, torch.bfloat16), (2, 28672, torch.bfloat16),
                (9, 8192, torch.float32), (4, 65536, torch.bfloat16), (2, 32768, torch.float32),
                (2048, 4096, torch.bfloat16), (320, 14336, torch.bfloat16), (300, 8192, torch.bfloat16),
                (513, 2048, torch.bfloat16), (257, 28672, torch.bfloat16), (260, 16384, torch.bfloat16),
                (6, 8192, torch.bfloat16), (3, 32768, torch.bfloat16), (100, 14336, torch.bfloat16)]


@pytest.mark.parametrize("R,K,dtype", QUANT_SHAPES)
def test_quant_act(oracle, R, K, dtype):
    x = rand((R, K), seed=R * 31 + K, dtype=dtype)
    if R > 2:
        x[1] = 0          # zero token row
        x[2] *= 1000      # large-magnitude row
    s_np = np.random.default_rng(K).uniform(0.25, 8.0, K).astype(np.float32)
    s = to_dev(s_np)
    xq = torch.empty(R, K, dtype=torch.int8, device="cuda")
    sx = torch.empty(R, device="cuda")
    sq.sq_quant_act(x.cuda(), s, xq, sx)
    xq_o, sx_o = oracle.quant_act(to_np(x), s_np)
    assert_bits_equal(to_np(sx), sx_o, "sx")
    assert_bits_equal(to_np(xq), xq_o, "xq")


@pytest.mark.parametrize("R,K,dtype", QUANT_SHAPES)
def test_smooth_quant_weight(oracle, R, K, dtype):
    w = rand((R, K), seed=R * 17 + K, dtype=dtype, scale=0.02)
    if R > 2:
        w[0] = 0
    s_np = np.random.default_rng(K + 1).uniform(0.1, 30.0, K).astype(np.float32)
    s = to_dev(s_np)
    wq = torch.empty(R, K, dtype=torch.int8, device="cuda")
    sw = torch.empty(R, device="cuda")
    sq.sq_smooth_quant_weight(w.cuda(), s, wq, sw)
    wq_o, sw_o = oracle.smooth_quant_weight(to_np(w), s_np)
    assert_bits_equal(to_np(sw), sw_o, "sw")
    assert_bits_equal(to_np(wq), wq_o, "wq")


# Few rows of more than 512 chunks: one thread-block cluster of C CTAs a row
# (C = 8, 4, 2 as rows x C fits the SMs and every slice keeps >= 128 chunks),
# slices of 1 to 8 chunks a thread, and slices cut raggedly (K / V not a
# multiple of C).
CLUSTER_SHAPES = [(1, 16384, torch.bfloat16), (2, 28672, torch.bfloat16), (20, 14336, torch.bfloat16),
                  (30, 16384, torch.bfloat16), (40, 28672, torch.bfloat16), (70, 8192, torch.float32),
                  (9, 8192, torch.float32), (5, 8208, torch.bfloat16), (18, 8192, torch.bfloat16),
                  (17, 4112, torch.float32), (60, 16384, torch.bfloat16)]


@pytest.mark.parametrize("R,K,dtype", CLUSTER_SHAPES)
def test_quant_cluster_rows(oracle, R, K, dtype):
    x = rand((R, K), seed=R * 13 + K, dtype=dtype)
    x[0, K - 5] = 900.0  # the row maximum in the last slice
    if R > 2:
        x[1] = 0
        x[2] *= 1000
    s_np = np.random.default_rng(K + 3).uniform(0.25, 8.0, K).astype(np.float32)
    xq = torch.empty(R, K, dtype=torch.int8, device="cuda")
    sx = torch.empty(R, device="cuda")
    sq.sq_quant_act(x.cuda(), to_dev(s_np), xq, sx)
    xq_o, sx_o = oracle.quant_act(to_np(x), s_np)
    assert_bits_equal(to_np(sx), sx_o, "sx")
    assert_bits_equal(to_np(xq), xq_o, "xq")
    wq = torch.empty(R, K, dtype=torch.int8, device="cuda")
    sw = torch.empty(R, device="cuda")
    sq.sq_smooth_quant_weight(x.cuda(), to_dev(s_np), wq, sw)
    wq_o, sw_o = oracle.smooth_quant_weight(to_np(x), s_np)
    assert_bits_equal(to_np(sw), sw_o, "sw")
    assert_bits_equal(to_np(wq), wq_o, "wq")


@pytest.mark.parametrize("K", [8192, 8208])
@pytest.mark.parametrize("s_kind", ["ones", "random", "extreme"])
def test_quant_cluster_fast_path_edges(oracle, s_kind, K):
    """The edge rows (exact ties and their 1-ulp neighbours, tiny, subnormal
    and huge rows, zero rows and zero chunks) repeated along a row of K = 8192
    or 8208 fp32 values, so that every slice of the cluster holds them; for
    "extreme", divisors outside the fast range in several slices."""
    base = _edge_rows(256, 5)
    x = np.tile(base, (1, (K + 255) // 256))[:, :K].copy()
    rng = np.random.default_rng(16)
    if s_kind == "ones":
        s_np = np.ones(K, np.float32)
    elif s_kind == "random":
        s_np = rng.uniform(0.05, 20.0, K).astype(np.float32)
    else:
        s_np = rng.uniform(0.5, 2.0, K).astype(np.float32)
        for col in (3, K // 2 + 1, K - 7):
            s_np[col] = 1e-25
            x[np.abs(x[:, col]) > 1e10, col] = 1.0  # keep x/s finite
        s_np[9] = 1e25
        s_np[K // 3] = 1e25
    sc = np.float32(0.0123)
    nt = (np.arange(K) % 200 - 100 + 0.5).astype(np.float32) * sc * s_np
    nt[K // 2] = np.float32(127.0) * sc * s_np[K // 2]
    x = np.vstack([x, nt.astype(np.float32)])
    xq = torch.empty(x.shape, dtype=torch.int8, device="cuda")
    sx = torch.empty(x.shape[0], device="cuda")
    sq.sq_quant_act(to_dev(x), to_dev(s_np), xq, sx)
    xq_o, sx_o = oracle.quant_act(x, s_np)
    assert_bits_equal(to_np(sx), sx_o, "sx")
    assert_bits_equal(to_np(xq), xq_o, "xq")


CHILD_FEW8 = r'''
import numpy as np
import torch
import w8a8_int8_gemm_channel_b200 as sq
from oracle import oracle
from w8a8_int8_gemm_channel_b200 import workloads as wls
oracle.build()
bits = lambda t: t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
for (R, K) in [(5, 14336), (2, 28672), (4, 16384), (3, 32768), (7, 8208)]:
    x = wls.random_tensor((R, K), R * 7 + K, dtype=torch.bfloat16)
    x[1] = 0
    if R > 2:
        x[2] *= 1000
    s = np.random.default_rng(K).uniform(0.25, 8.0, K).astype(np.float32)
    xq = torch.empty(R, K, dtype=torch.int8, device="cuda")
    sx = torch.empty(R, device="cuda")
    sq.sq_quant_act(x.cuda(), torch.from_numpy(s).cuda(), xq, sx)
    wq = torch.empty(R, K, dtype=torch.int8, device="cuda")
    sw = torch.empty(R, device="cuda")
    sq.sq_smooth_quant_weight(x.cuda(), torch.from_numpy(s).cuda(), wq, sw)
    torch.cuda.synchronize()
    xq_o, sx_o = oracle.quant_act(bits(x), s)
    assert np.array_equal(xq.cpu().numpy(), xq_o) and np.array_equal(sx.cpu().numpy().view(np.uint32), sx_o.view(np.uint32)), (R, K)
    wq_o, sw_o = oracle.smooth_quant_weight(bits(x), s)
    assert np.array_equal(wq.cpu().numpy(), wq_o) and np.array_equal(sw.cpu().numpy().view(np.uint32), sw_o.view(np.uint32)), (R, K)
st, code = sq.sq_device_status()
assert st == sq.SQ_OK, hex(code)
print("few8-ok")
'''


def test_few_row_quantiser_8_warps_child_process():
    """Few long rows take the cluster form and, past the SM count, the 16-warp
    form by default; with SQ_QUANT_CLUSTER=0 and SQ_QUANT_FEW_THREADS=256
    (read once per process, so in a child) they take the 8-warp form (4, 8
    and 16 chunks a lane, exact fits and ragged rows).  Codes and scales equal
    the oracle's bit for bit."""
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SQ_QUANT_FEW_THREADS="256", SQ_QUANT_CLUSTER="0", PYTHONPATH=root)
    r = subprocess.run([sys.executable, "-c", CHILD_FEW8], cwd=root, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "few8-ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]


CHILD_CLUSTER_SHORT = r'''
import numpy as np
import torch
import w8a8_int8_gemm_channel_b200 as sq
from oracle import oracle
from w8a8_int8_gemm_channel_b200 import workloads as wls
oracle.build()
bits = lambda t: t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
for (R, K, dt) in [(1, 4096, torch.bfloat16), (30, 4096, torch.bfloat16), (9, 4112, torch.bfloat16),
                   (5, 4096, torch.float32), (37, 2048, torch.bfloat16)]:
    x = wls.random_tensor((R, K), R * 11 + K, dtype=dt)
    x[0, K - 3] = 700.0
    if R > 2:
        x[1] = 0
        x[2] *= 1000
    s = np.random.default_rng(K + 5).uniform(0.25, 8.0, K).astype(np.float32)
    xq = torch.empty(R, K, dtype=torch.int8, device="cuda")
    sx = torch.empty(R, device="cuda")
    sq.sq_quant_act(x.cuda(), torch.from_numpy(s).cuda(), xq, sx)
    torch.cuda.synchronize()
    xin = bits(x) if dt == torch.bfloat16 else x.numpy()
    xq_o, sx_o = oracle.quant_act(xin, s)
    assert np.array_equal(xq.cpu().numpy(), xq_o) and np.array_equal(sx.cpu().numpy().view(np.uint32), sx_o.view(np.uint32)), (R, K)
st, code = sq.sq_device_status()
assert st == sq.SQ_OK, hex(code)
print("cluster-short-ok")
'''


def test_cluster_form_on_short_rows_child_process():
    """SQ_QUANT_CLUSTER=2 (read once per process, so in a child) gives rows of
    512 chunks or fewer the cluster form too (clusters of 2, 4 and 8 CTAs with
    slices of 128 to 129 chunks, ragged slices at K = 4112); codes and scales
    equal the oracle's bit for bit."""
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SQ_QUANT_CLUSTER="2", PYTHONPATH=root)
    r = subprocess.run([sys.executable, "-c", CHILD_CLUSTER_SHORT], cwd=root, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "cluster-short-ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]


# ---------------------------------------------------------------------------
# GEMM: int32 accumulators and the dequantised output
# ---------------------------------------------------------------------------

GEMM_SHAPES = [(1, 16, 16), (5, 32, 48), (16, 256, 256), (31, 272, 4112), (33, 128, 128),
               (64, 64, 256), (100, 48, 1024), (128, 512, 4096), (129, 272, 4112),
               (300, 528, 1040), (257, 784, 2064), (512, 1024, 512)]


def _int8(shape, seed):
    return wls.random_int8(shape, seed)


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_s32_exact(oracle, M, N, K):
    xq = _int8((M, K), seed=M * 1000 + K)
    wq = _int8((N, K), seed=N * 1000 + K + 1)
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    sq.sq_w8a8_gemm_s32(xq.cuda(), wq.cuda(), acc)
    assert_bits_equal(to_np(acc), oracle.gemm_i32(to_np(xq), to_np(wq)), f"acc {M}x{N}x{K}")


@pytest.mark.parametrize("out", ["bf16", "f32"])
@pytest.mark.parametrize("M,N,K", [(1, 16, 16), (31, 272, 4112), (129, 272, 4112), (300, 528, 1040)])
def test_gemm_dequant(oracle, M, N, K, out):
    xq = _int8((M, K), seed=M + 5 * K)
    wq = _int8((N, K), seed=N + 7 * K)
    rng = np.random.default_rng(M * N)
    sx_np = rng.uniform(1e-3, 2.0, M).astype(np.float32)
    sw_np = rng.uniform(1e-5, 1e-3, N).astype(np.float32)
    if M > 1:
        sx_np[0] = 0.0  # a zero token row
    y = torch.empty(M, N, dtype=torch.bfloat16 if out == "bf16" else torch.float32, device="cuda")
    sq.sq_w8a8_gemm(xq.cuda(), to_dev(sx_np), wq.cuda(), to_dev(sw_np), y)
    acc_o = oracle.gemm_i32(to_np(xq), to_np(wq))
    y_o = oracle.dequant(acc_o, sx_np, sw_np, out)
    assert_output_close(to_np(y), y_o, f"y {out}")
    assert exact_fraction(to_np(y), y_o) == 1.0


# Shapes whose tile counts select each tile width of the CTA-pair prefill
# kernel on 74 pairs (256, 256, 192 and 128 output columns per 256-row tile),
# with ragged M and K; checked exactly on every row and column at the tile edges
# plus a random sample of (token, channel) pairs.
@pytest.mark.parametrize("M,N,K", [(2000, 4096, 272), (4000, 6144, 528), (1000, 6144, 1040), (300, 1040, 2064)])
def test_gemm_pair_widths_sampled(oracle, M, N, K):
    xq = _int8((M, K), seed=M * 7 + K)
    wq = _int8((N, K), seed=N * 11 + K)
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    sq.sq_w8a8_gemm_s32(xq.cuda(), wq.cuda(), acc)
    rng = np.random.default_rng(M + N + K)
    ms = np.unique(np.concatenate([[0, 127, 128, 255, 256, M - 1], rng.integers(0, M, 24)]))
    ns = np.unique(np.concatenate([[0, 63, 64, 95, 96, 127, 128, 191, 192, 255, 256, N - 1],
                                   rng.integers(0, N, 40)]))
    mm, nn = np.meshgrid(ms, ns, indexing="ij")
    xq_h, wq_h = to_np(xq), to_np(wq)
    im, jn = np.meshgrid(np.arange(ms.size), np.arange(ns.size), indexing="ij")
    acc_o = oracle.gemm_i32_pairs(xq_h[ms], wq_h[ns], im.ravel(), jn.ravel())
    assert_bits_equal(to_np(acc)[mm.ravel(), nn.ravel()], acc_o, f"acc {M}x{N}x{K} sampled")
    # y through the dequantising epilogue on the same sample
    rng2 = np.random.default_rng(K)
    sx_np = rng2.uniform(1e-3, 2.0, M).astype(np.float32)
    sw_np = rng2.uniform(1e-5, 1e-3, N).astype(np.float32)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    sq.sq_w8a8_gemm(xq.cuda(), to_dev(sx_np), wq.cuda(), to_dev(sw_np), y)
    y_o = oracle.dequant_pairs(acc_o, sx_np[mm.ravel()], sw_np[nn.ravel()], "bf16")
    assert_output_close(to_np(y)[mm.ravel(), nn.ravel()], y_o, "y sampled")


def test_gemm_extreme_accumulators(oracle):
    """All +127 against all -127 at K = 28672: |acc| = K * 127^2, the largest magnitude."""
    M, N, K = 3, 32, 28672
    xq = torch.full((M, K), 127, dtype=torch.int8)
    wq = torch.full((N, K), -127, dtype=torch.int8)
    wq[1::2] = 127
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    sq.sq_w8a8_gemm_s32(xq.cuda(), wq.cuda(), acc)
    assert_bits_equal(to_np(acc), oracle.gemm_i32(to_np(xq), to_np(wq)), "acc extremes")
    assert int(to_np(acc)[0, 0]) == -K * 127 * 127


# ---------------------------------------------------------------------------
# the online linear (sq_linear) against the oracle, bf16 in / bf16 out
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (8, 272, 4112), (32, 6144, 1024),
                                   (77, 512, 2048), (256, 768, 4096)])
def test_linear_bf16(oracle, M, N, K):
    x = rand((M, K), seed=M + N + K)
    x[:, 7] *= 60.0
    w = rand((N, K), seed=N + K + 3, scale=0.02)
    xcal = rand((512, K), seed=K + 9)
    xcal[:, 7] *= 60.0
    _, _, s_o, wq_o, sw_o = oracle.prepare(to_np(xcal), to_np(w), 0.5)
    s = to_dev(s_o)
    wq = to_dev(wq_o)
    sw = to_dev(sw_o)
    y = sq.linear(x.cuda(), s, wq, sw, out_dtype=torch.bfloat16)
    y_o, _, _, _ = oracle.linear(to_np(x), s_o, wq_o, sw_o, "bf16")
    assert_output_close(to_np(y), y_o, "linear")
    assert exact_fraction(to_np(y), y_o) == 1.0


# ---------------------------------------------------------------------------
# numerics of the quantisers' fast paths: ties, near-ties, tiny and huge
# magnitudes, divisors outside the fast range, zero chunks
# ---------------------------------------------------------------------------

def _edge_rows(K, seed):
    rng = np.random.default_rng(seed)
    rows = []
    # exact ties and 1-ulp neighbours: amax 127 gives scale 1 when s == 1
    t = np.array([127.0] + [k + 0.5 for k in range(-60, 60)] * 4, np.float32)[:K]
    rows.append(t)
    rows.append(np.nextafter(t, np.float32(np.inf)))
    rows.append(np.nextafter(t, np.float32(-np.inf)))
    # tiny, subnormal-adjacent and huge rows (scale outside the fast range)
    rows.append((rng.standard_normal(K) * 1e-33).astype(np.float32))
    rows.append((rng.standard_normal(K) * 1e-40).astype(np.float32))
    rows.append((rng.standard_normal(K) * 1e30).astype(np.float32))
    # a zero row and a row with zero chunks
    rows.append(np.zeros(K, np.float32))
    z = rng.standard_normal(K).astype(np.float32)
    z[: K // 2] = 0.0
    rows.append(z)
    # near-ties for a generic scale: values placed at (k + 1/2) * scale * s_k
    return np.stack(rows).astype(np.float32)


@pytest.mark.parametrize("s_kind", ["ones", "random", "extreme"])
def test_quant_act_fast_path_edges(oracle, s_kind):
    K = 256
    x = _edge_rows(K, 5)
    rng = np.random.default_rng(6)
    if s_kind == "ones":
        s_np = np.ones(K, np.float32)
    elif s_kind == "random":
        s_np = rng.uniform(0.05, 20.0, K).astype(np.float32)
    else:  # divisors outside [2^-60, 2^61): exercises the IEEE fallback
        s_np = rng.uniform(0.5, 2.0, K).astype(np.float32)
        s_np[3] = 1e-25
        s_np[9] = 1e25
        # keep every smoothed value x/s finite (an overflowing quotient is outside the contract)
        x[np.abs(x[:, 3]) > 1e10, 3] = 1.0
    # a generic-scale near-tie row: amax fixed by one element, others at half-integers
    sc = np.float32(0.0123)
    nt = (np.arange(K) % 200 - 100 + 0.5).astype(np.float32) * sc * s_np
    nt[0] = np.float32(127.0) * sc * s_np[0]
    x = np.vstack([x, nt.astype(np.float32)])
    xq = torch.empty(x.shape, dtype=torch.int8, device="cuda")
    sx = torch.empty(x.shape[0], device="cuda")
    sq.sq_quant_act(to_dev(x), to_dev(s_np), xq, sx)
    xq_o, sx_o = oracle.quant_act(x, s_np)
    assert_bits_equal(to_np(sx), sx_o, "sx")
    assert_bits_equal(to_np(xq), xq_o, "xq")
    # the online linear on the same inputs (quantiser, then GEMM)
    wq = wls.random_int8((64, K), seed=7)
    sw = np.full(64, 1e-3, np.float32)
    y = torch.empty(x.shape[0], 64, dtype=torch.float32, device="cuda")
    need = sq.sq_linear_workspace_size(x.shape[0], 64, K)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    sq.sq_linear(to_dev(x), to_dev(s_np), wq.cuda(), to_dev(sw), y, ws if need else None)
    acc_o = oracle.gemm_i32(xq_o, to_np(wq))
    assert_output_close(to_np(y), oracle.dequant(acc_o, sx_o, sw, "f32"), "linear")


@pytest.mark.parametrize("s_kind", ["ones", "random", "extreme"])
def test_smooth_quant_weight_fast_path_edges(oracle, s_kind):
    K = 256
    w = _edge_rows(K, 8)
    rng = np.random.default_rng(9)
    s_np = {"ones": np.ones(K, np.float32),
            "random": rng.uniform(0.05, 20.0, K).astype(np.float32),
            "extreme": np.where(np.arange(K) % 17 == 0, 1e-20, 1.0).astype(np.float32)}[s_kind]
    wq = torch.empty(w.shape, dtype=torch.int8, device="cuda")
    sw = torch.empty(w.shape[0], device="cuda")
    sq.sq_smooth_quant_weight(to_dev(w), to_dev(s_np), wq, sw)
    wq_o, sw_o = oracle.smooth_quant_weight(w, s_np)
    assert_bits_equal(to_np(sw), sw_o, "sw")
    assert_bits_equal(to_np(wq), wq_o, "wq")


# ---------------------------------------------------------------------------
# bf16 rows: the quantisers bound |v| in bf16 arithmetic (within about 0.8%)
# and recompute exactly every chunk within 2^-5 of the largest bound; these
# rows crowd the top of the range so that the bound alone could not order them
# ---------------------------------------------------------------------------

def _bf16_crowded_rows(K, s_np, mode, seed):
    """bf16 rows (as fp32 values) whose smoothed magnitudes crowd the maximum."""
    rng = np.random.default_rng(seed)
    f = (1.0 / s_np) if mode == "x" else s_np  # v = x * f in exact arithmetic
    rows = []
    # 300 elements within 0.5% of 3.0, the rest far below
    r = rng.standard_normal(K) * 0.3
    idx = rng.choice(K, 300, replace=False)
    r[idx] = 3.0 * (1.0 + rng.uniform(-0.005, 0.005, 300)) * np.sign(rng.standard_normal(300))
    rows.append(r / f)
    # every smoothed magnitude equal up to bf16 rounding of x: all chunks are candidates
    rows.append(np.where(rng.random(K) < 0.5, -1.0, 1.0) / f)
    # Gaussian with a few outlier channels, a tiny row and a zero row
    r = rng.standard_normal(K)
    r[rng.choice(K, 5, replace=False)] *= 60.0
    rows.append(r / f)
    rows.append(rng.standard_normal(K) * 1e-33 / f)
    rows.append(np.zeros(K))
    x = torch.from_numpy(np.stack(rows).astype(np.float32)).to(torch.bfloat16)
    return x


@pytest.mark.parametrize("K", [4096, 14336])
@pytest.mark.parametrize("mode", ["x", "w"])
def test_quant_bf16_crowded_maxima(oracle, K, mode):
    rng = np.random.default_rng(K + (1 if mode == "x" else 2))
    s_np = rng.uniform(0.3, 3.0, K).astype(np.float32)
    x = _bf16_crowded_rows(K, s_np, mode, seed=K)
    q = torch.empty(x.shape, dtype=torch.int8, device="cuda")
    sc = torch.empty(x.shape[0], device="cuda")
    if mode == "x":
        sq.sq_quant_act(x.cuda(), to_dev(s_np), q, sc)
        q_o, sc_o = oracle.quant_act(to_np(x), s_np)
    else:
        sq.sq_smooth_quant_weight(x.cuda(), to_dev(s_np), q, sc)
        q_o, sc_o = oracle.smooth_quant_weight(to_np(x), s_np)
    assert_bits_equal(to_np(sc), sc_o, f"scales ({mode})")
    assert_bits_equal(to_np(q), q_o, f"codes ({mode})")
