"""Full-size parity on sampled outputs: every workload at its real sizes,
through the same C-ABI calls (and so the same launch configurations) that
bench.py times, checked against the CPU oracle on the same bytes.

  * calibration absmax and the weight input-channel absmax: every channel,
    bit-exact (the oracle scans the whole calibration batch and weight);
  * smoothing factors: every channel (bit-exact up to the fp64 midpoint rule);
  * smoothed int8 weights and their scales: sampled output channels, bit-exact;
  * per-token quantisation (M > 32, separate kernel): sampled tokens, bit-exact;
  * the linear's output: sampled (token, channel) pairs, within 1 bf16 ulp.
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
    idx = set([0, n - 1])
    idx.update(rng.choice(n, size=min(n, count), replace=False).tolist())
    return np.array(sorted(idx), dtype=np.int64)


@pytest.mark.parametrize("wl_name", ["llama3_8b_attn", "llama3_8b_mlp", "llama3_8b_decode",
                                     "llama3_70b"])
def test_workload_fullsize_sampled(oracle, wl_name):
    wl = wls.WORKLOADS[wl_name]
    dev = torch.device("cuda")
    rng = np.random.default_rng(abs(hash(wl_name)) % (2 ** 32))
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
        ns = _sample(N, 48, rng)
        wq_o, sw_o = oracle.smooth_quant_weight(w_h[ns], s_o)
        assert_bits_equal(to_np(wq[torch.from_numpy(ns).to(dev)]), wq_o, f"{lin.name} wq rows")
        assert_bits_equal(to_np(sw)[ns], sw_o, f"{lin.name} sw rows")
        del w, w_h

        for M in wl.Ms:
            x = wls.inputs(wl, lin, M, device=dev)
            ms = _sample(M, 12, rng)
            x_h = to_np(x)
            xq_o, sx_o = oracle.quant_act(x_h, s_o, rows=ms)
            if sq.sq_linear_workspace_size(M, N, K) > 0:
                xq = torch.empty(M, K, dtype=torch.int8, device=dev)
                sx = torch.empty(M, device=dev)
                sq.sq_quant_act(x, s, xq, sx)
                assert_bits_equal(to_np(xq)[ms], xq_o, f"{lin.name} M={M} xq rows")
                assert_bits_equal(to_np(sx)[ms], sx_o, f"{lin.name} M={M} sx rows")
            y = sq.linear(x, s, wq, sw, out_dtype=torch.bfloat16)
            mm, nn = np.meshgrid(np.arange(ms.size), np.arange(ns.size), indexing="ij")
            acc_o = oracle.gemm_i32_pairs(xq_o, wq_o, mm.ravel(), nn.ravel())
            y_o = oracle.dequant_pairs(acc_o, sx_o[mm.ravel()], sw_o[nn.ravel()], "bf16")
            y_g = to_np(y)[np.ix_(ms, ns)].ravel()
            assert_output_close(y_g, y_o, f"{wl_name}/{lin.name} M={M} y")
            del x, y
        torch.cuda.empty_cache()
