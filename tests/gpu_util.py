"""Helpers shared by the GPU parity tests: tensor <-> NumPy conversion that
keeps bf16 as raw bit patterns, and the comparison rules.

Comparison rules (what the layer promises):
  * integer and byte results (absmax bits, codes, int32 accumulators, scales):
    bit-exact;
  * smoothing factors: bit-exact, except where the fp64 quotient lies within a
    few fp64 ulps of an fp32 rounding midpoint (libm and CUDA pow may then round
    to different neighbours; both are correct roundings of an fp64 value);
  * dequantised output: within 1e-6 relative (fp32) or 1 bf16 ulp (bf16).
"""
import math

import numpy as np
import torch


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def to_dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    if a.dtype == np.uint16 and dtype in (None, torch.bfloat16):
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def assert_bits_equal(got: np.ndarray, want: np.ndarray, what: str):
    assert got.shape == want.shape, (what, got.shape, want.shape)
    g = got.view(np.uint32) if got.dtype == np.float32 else got
    w = want.view(np.uint32) if want.dtype == np.float32 else want
    bad = np.flatnonzero(g.ravel() != w.ravel())
    assert bad.size == 0, f"{what}: {bad.size} mismatches, first at {bad[:5].tolist()}: " \
                          f"got {got.ravel()[bad[:5]].tolist()} want {want.ravel()[bad[:5]].tolist()}"


def assert_smooth_factors(got: np.ndarray, want: np.ndarray, ax: np.ndarray, aw: np.ndarray, alpha):
    """Bit-exact, except for fp64 values within ~1e-14 relative of an fp32 midpoint."""
    bad = np.flatnonzero(got.view(np.uint32) != want.view(np.uint32))
    a = float(np.float32(alpha))
    for j in bad:
        r = math.pow(float(ax[j]), a) / math.pow(float(aw[j]), 1.0 - a)
        lo, hi = sorted((float(got[j]), float(want[j])))
        assert np.nextafter(np.float32(lo), np.float32(np.inf)) == np.float32(hi), (j, got[j], want[j])
        mid = (lo + hi) / 2
        assert abs(r - mid) <= 1e-14 * abs(r), f"s[{j}]: {got[j]} vs {want[j]} (fp64 {r!r})"


def bf16_ulp_diff(got: np.ndarray, want: np.ndarray) -> np.ndarray:
    """|difference| in units in the last place between bf16 bit patterns."""
    def ordered(u):
        v = u.astype(np.int32)
        return np.where(v & 0x8000, 0x8000 - (v & 0x7FFF), v + 0x8000)

    return np.abs(ordered(got) - ordered(want))


def assert_output_close(got: np.ndarray, want: np.ndarray, what: str):
    """fp32: within 1e-6 relative; bf16 (uint16 bit patterns): within 1 ulp."""
    assert got.shape == want.shape
    if got.dtype == np.uint16:
        d = bf16_ulp_diff(got, want)
        assert d.max(initial=0) <= 1, f"{what}: max bf16 ulp diff {d.max()}"
    else:
        tol = 1e-6 * np.abs(want.astype(np.float64))
        err = np.abs(got.astype(np.float64) - want.astype(np.float64))
        bad = np.flatnonzero(err > tol)
        assert bad.size == 0, f"{what}: {bad.size} elements beyond 1e-6 relative"


def exact_fraction(got: np.ndarray, want: np.ndarray) -> float:
    g = got.view(np.uint32) if got.dtype == np.float32 else got
    w = want.view(np.uint32) if want.dtype == np.float32 else want
    return float(np.mean(g == w)) if g.size else 1.0
