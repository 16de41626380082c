"""The seeded input generators shared by the CUDA path and the oracle: they
are deterministic, have the shapes and distributions the workloads state, and
hold none of the method's arithmetic (CPU only)."""
import ast
import os

import torch

from w8a8_int8_gemm_channel_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_generators_are_deterministic_and_seed_separated():
    w = wl.WORKLOADS["llama3_8b_attn"]
    lin = w.linears[0]
    a = wl.activations(w, lin, 8, "x")
    b = wl.activations(w, lin, 8, "x")
    c = wl.activations(w, lin, 8, "calib")
    assert torch.equal(a, b) and not torch.equal(a, c)
    assert wl.seed_for("a", "b") == wl.seed_for("a", "b") != wl.seed_for("a", "c")


def test_outlier_channels_follow_the_stated_count():
    w = wl.WORKLOADS["llama3_8b_attn"]
    for K, n in ((4096, 4), (8192, 8), (14336, 14), (28672, 29)):
        ch = wl.outlier_channels(w, K)
        assert len(ch) == n and len(set(ch)) == n and all(0 <= c < K for c in ch)
    assert wl.outlier_channels(wl.WORKLOADS["small"], 256) == [3, 77, 150, 201]


def test_gate_up_layout_and_outliers():
    w = wl.WORKLOADS["llama3_8b_mlp"]
    lin = w.linears[1]  # the down projection, K = 14336
    gu = wl.gate_up(w, lin, 64, "x", dtype="f32")
    K = lin.K
    assert gu.shape == (64, 2 * K) and gu.dtype == torch.float32
    assert torch.equal(gu, wl.gate_up(w, lin, 64, "x", dtype="f32"))
    idx = wl.outlier_channels(w, K)
    rest = [j for j in range(K) if j not in set(idx)][:2000]
    up_out = gu[:, K + torch.tensor(idx)].abs().mean()
    up_rest = gu[:, K + torch.tensor(rest)].abs().mean()
    gate_out = gu[:, torch.tensor(idx)].abs().mean()
    # the up half carries the outlier scaling, the gate half does not
    assert up_out > 20 * up_rest
    assert 0.5 < float(gate_out) < 1.5
    assert wl.gate_up(w, lin, 4, "x").dtype == torch.bfloat16


def test_generator_module_holds_none_of_the_method():
    """No absmax, smoothing, rounding or GEMM in the shared module: it may only
    draw, scale and cast."""
    tree = ast.parse(open(os.path.join(ROOT, "w8a8_int8_gemm_channel_b200", "workloads.py")).read())
    called = {n.func.attr for n in ast.walk(tree) if isinstance(n, ast.Call) and isinstance(n.func, ast.Attribute)}
    forbidden = {"amax", "max", "round", "clamp", "matmul", "mm", "pow", "div", "abs", "rint"}
    assert not (called & forbidden), called & forbidden
