"""Helpers shared by the GPU tests: device copies of seeded inputs and the parity criteria."""
import numpy as np
import torch

from workloads import to_bf16_bits, widen_bf16

# Parity criteria (fixed before any kernel was written):
#   fp32 path:  max|err| <= 1e-4 * max|ref|
#   bf16 path:  max|err| <= 2e-2 * max|ref|  and  mean|err| <= 2e-3 * rms(ref)
F32_MAX_REL = 1e-4
BF16_MAX_REL = 2e-2
BF16_MEAN_REL = 2e-3
# The layer backward's outputs pass through up to six bf16 roundings in a chain (the forward's
# U|V|Q|K and G, the attention's P and dS operands, dAV, dU|dV|dQ|dK, dZ), each a relative error of
# rms at most u/sqrt(3) with u = 2^-8 the bf16 unit roundoff.  Independent, they add to a relative
# rms of at most sqrt(6) u / sqrt(3) = sqrt(2) u, which bounds mean|err| / rms(ref) as long as the
# roundings are independent (an rms estimate: correlated ones, such as P and dS taken from the same
# score, could exceed it; over every case of the layer backward's tests the largest observed value
# is 4.0e-3 (dX - dY), 73% of it).  The attention backward's outputs meet the forward's BF16_MEAN_REL
# and are held to it; so are the layer backward's dln_b and dtime.
BWD_MEAN_REL = float(np.sqrt(2.0) * 2.0 ** -8)


def dev(a, dtype="bf16", device="cuda"):
    """numpy -> device tensor.  Float arrays become bf16 (exact: they hold bf16 values) or fp32."""
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype.kind == "i":
        return torch.from_numpy(a.astype(np.int64)).to(device)
    if dtype == "bf16":
        bits = to_bf16_bits(a.astype(np.float32))
        return torch.from_numpy(bits.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a.astype(np.float32)).to(device)


def host(t: torch.Tensor) -> np.ndarray:
    """device tensor -> float64 numpy (exact)."""
    t = t.detach()
    if t.dtype == torch.bfloat16:
        bits = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        return widen_bf16(bits, np.float64)
    return t.float().cpu().numpy().astype(np.float64)


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Storage rounding of an fp64 array to bf16 values (inputs prepared for a bf16 kernel)."""
    return widen_bf16(to_bf16_bits(np.asarray(a, np.float32)), np.float64)


def errors(got: np.ndarray, ref: np.ndarray):
    err = np.abs(got - ref)
    return float(err.max() / max(np.abs(ref).max(), 1e-300)), \
        float(err.mean() / max(np.sqrt(np.mean(ref ** 2)), 1e-300))


def assert_bf16_close(got, ref, what=""):
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    mx, mn = errors(got, ref)
    assert mx <= BF16_MAX_REL and mn <= BF16_MEAN_REL, \
        f"{what}: max|err|/max|ref| = {mx:.3e}, mean|err|/rms(ref) = {mn:.3e}"
    return mx, mn


def assert_bwd_close(got, ref, what=""):
    """The bf16 criteria with the mean bound of the layer backward's chain of roundings."""
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    mx, mn = errors(got, ref)
    assert mx <= BF16_MAX_REL and mn <= BWD_MEAN_REL, \
        f"{what}: max|err|/max|ref| = {mx:.3e}, mean|err|/rms(ref) = {mn:.3e}"
    return mx, mn


def assert_f32_close(got, ref, what=""):
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    mx, _ = errors(got, ref)
    assert mx <= F32_MAX_REL, f"{what}: max|err|/max|ref| = {mx:.3e}"
    return mx


def assert_layer_part_close(got, ref, X, what=""):
    """Diagnostic on the part of Y the layer adds (Y - X, which the residual X otherwise dominates).
    The output's own bf16 rounding is excluded: mean|got - ref| minus the rounding floor
    mean|bf16(ref) - ref| must stay within 2e-3 * rms(ref - X); max|err| within 2e-2 * max|ref - X|
    plus one output quantum."""
    part = ref - X
    err = np.abs(got - ref)
    floor = np.mean(np.abs(round_bf16(ref) - ref))
    quantum = np.max(np.abs(round_bf16(ref) - ref))
    rms = np.sqrt(np.mean(part ** 2))
    excess = (err.mean() - floor) / rms
    mx = (err.max() - quantum) / np.abs(part).max()
    assert excess <= BF16_MEAN_REL and mx <= BF16_MAX_REL, \
        f"{what}: excess mean err {excess:.3e} of rms(Y-X), max err {mx:.3e} of max|Y-X|"
    return excess, mx
