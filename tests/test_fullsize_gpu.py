"""Full-size parity: every workload at its real sizes, through the same C-ABI
calls (and so the same launch configurations) that bench.py times, checked
against the CPU oracle on the same bytes.

  * calibration absmax and the weight input-channel absmax: every channel,
    bit-exact (the oracle scans the whole calibration batch and weight);
  * smoothing factors: every channel (bit-exact up to the fp64 midpoint rule);
  * smoothed int8 weights and their scales: every output channel, bit-exact;
  * per-token quantisation (where sq_linear runs it as its own kernel):
    every token, bit-exact;
  * the linear's output: whole rows (every output channel) for sampled
    tokens and whole columns (every token) for sampled output channels,
    within 1 bf16 ulp -- so every M tile and every N tile of the GEMM that
    runs at that size has at least one row and one column checked;
  * the int32 accumulators of the two Llama-3-70B reduction widths
    (K = 8192 and K = 28672) at M = 8192, on the same whole rows and
    columns: bit-exact.
The downstream stages are fed the oracle's smoothing factors on both sides.
"""
import numpy as np
import pytest
import torch

import w8a8_int8_gemm_channel_b200 as sq
from w8a8_int8_gemm_channel_b200 import workloads as wls
from tests.gpu_util import (assert_bits_equal, assert_output_close, assert_smooth_factors, to_dev,
                            to_np)

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


def _sample(n, count, rng):
    """`count` random indices of range(n), plus the first and the last."""
    idx = set([0, n - 1])
    idx.update(rng.choice(n, size=min(n, count), replace=False).tolist())
    return np.array(sorted(idx), dtype=np.int64)


def _rows_cols(oracle, xq_o, sx_o, wq_o, sw_o, ms, ns, out):
    """The oracle's outputs on whole rows ms (every n) and whole columns ns (every m)."""
    rows = oracle.dequant(oracle.gemm_i32(xq_o[ms], wq_o), sx_o[ms], sw_o, out)
    cols = oracle.dequant(oracle.gemm_i32(xq_o, wq_o[ns]), sx_o, sw_o[ns], out)
    return rows, cols


@pytest.mark.parametrize("wl_name", ["llama3_8b_attn", "llama3_8b_mlp", "llama3_8b_decode",
                                     "llama3_70b"])
def test_workload_fullsize(oracle, wl_name):
    wl = wls.WORKLOADS[wl_name]
    dev = torch.device("cuda")
    rng = np.random.default_rng(sum(map(ord, wl_name)))
    for lin in wl.linears:
        K, N = lin.K, lin.N
        xcal = wls.calibration(wl, lin, device=dev)
        w = wls.weight(wl, lin, device=dev)
        ax = sq.calibrate(xcal)
        s_dev = torch.empty(K, device=dev)
        aw_dev = torch.empty(K, device=dev)
        sq.sq_smooth_factors(ax, w, wl.alpha, s_dev, aw_dev)
        torch.cuda.synchronize()
        xcal_h = to_np(xcal)
        del xcal
        ax_o = oracle.calib_absmax(xcal_h)
        del xcal_h
        assert_bits_equal(to_np(ax), ax_o, f"{wl_name}/{lin.name} ax")
        w_h = to_np(w)
        aw_o = oracle.weight_in_absmax(w_h)
        assert_bits_equal(to_np(aw_dev), aw_o, f"{wl_name}/{lin.name} aw")
        s_o = oracle.smooth_factors(ax_o, aw_o, wl.alpha)
        assert_smooth_factors(to_np(s_dev), s_o, ax_o, aw_o, wl.alpha)

        s = to_dev(s_o)
        wq = torch.empty(N, K, dtype=torch.int8, device=dev)
        sw = torch.empty(N, device=dev)
        sq.sq_smooth_quant_weight(w, s, wq, sw)
        wq_o, sw_o = oracle.smooth_quant_weight(w_h, s_o)
        assert_bits_equal(to_np(wq), wq_o, f"{wl_name}/{lin.name} wq")
        assert_bits_equal(to_np(sw), sw_o, f"{wl_name}/{lin.name} sw")
        del w, w_h

        for M in wl.Ms:
            x = wls.inputs(wl, lin, M, device=dev)
            x_h = to_np(x)
            xq_o, sx_o = oracle.quant_act(x_h, s_o)
            if sq.sq_linear_workspace_size(M, N, K) > 0:
                xq = torch.empty(M, K, dtype=torch.int8, device=dev)
                sx = torch.empty(M, device=dev)
                sq.sq_quant_act(x, s, xq, sx)
                assert_bits_equal(to_np(xq), xq_o, f"{wl_name}/{lin.name} M={M} xq")
                assert_bits_equal(to_np(sx), sx_o, f"{wl_name}/{lin.name} M={M} sx")
                del xq, sx
            y = sq.linear(x, s, wq, sw, out_dtype=torch.bfloat16)
            ms = _sample(M, 6, rng)
            ns = _sample(N, 6, rng)
            rows_o, cols_o = _rows_cols(oracle, xq_o, sx_o, wq_o, sw_o, ms, ns, "bf16")
            y_h = to_np(y)
            assert_output_close(y_h[ms], rows_o, f"{wl_name}/{lin.name} M={M} y rows {ms.tolist()}")
            assert_output_close(y_h[:, ns], cols_o, f"{wl_name}/{lin.name} M={M} y columns {ns.tolist()}")
            del x, y, y_h
        del wq, sw
        torch.cuda.empty_cache()


@pytest.mark.parametrize("lin_name", ["gate_up", "down"])
def test_llama3_70b_accumulators_fullsize(oracle, lin_name):
    """int32 accumulators of the 70B gate/up (K = 8192, N = 57344) and down
    (K = 28672, N = 8192) projections at M = 8192, whole rows and columns."""
    wl = wls.WORKLOADS["llama3_70b"]
    lin = next(l for l in wl.linears if l.name == lin_name)
    K, N, M = lin.K, lin.N, 8192
    rng = np.random.default_rng(K + N)
    xq_h = wls.random_int8((M, K), seed=K + 1).numpy()
    wq_h = wls.random_int8((N, K), seed=N + 2).numpy()
    # saturated rows and columns reach the accumulator's extremes
    xq_h[5] = 127
    wq_h[7] = 127
    wq_h[9] = -127
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    sq.sq_w8a8_gemm_s32(to_dev(xq_h), to_dev(wq_h), acc)
    torch.cuda.synchronize()
    ms = np.union1d(_sample(M, 6, rng), [5])
    ns = np.union1d(_sample(N, 6, rng), [7, 9])
    acc_h = to_np(acc)
    assert_bits_equal(acc_h[ms], oracle.gemm_i32(xq_h[ms], wq_h), f"{lin_name} acc rows")
    assert_bits_equal(acc_h[:, ns], oracle.gemm_i32(xq_h, wq_h[ns]), f"{lin_name} acc columns")
    assert acc_h[5, 7] == 127 * 127 * K and acc_h[5, 9] == -127 * 127 * K
