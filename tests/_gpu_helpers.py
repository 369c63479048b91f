"""Shared helpers of the GPU parity tests: NaN-poisoned allocations and the
acceptance checks against the FP64 oracle.

Acceptance (written here once, used by every parity test):
  * O:   max |O - O_ref| <= 2e-2 * max |v|   (16-bit outputs; derivation: P and
         O are rounded to 16 bits, relative error <= 2^-8 each, far inside 2e-2)
  * LSE: max |LSE - LSE_ref| <= 1e-3 log2 units (fp32 accumulation of a D <= 256
         dot product has a forward error bound gamma_D * sum|q_d k_d| ~ 1.5e-5
         relative, the exp2/log2 approximations ~ 2^-22 relative)
  * no NaN and no Inf anywhere, except LSE = -inf exactly where the reference
    row has no keys.
"""
import numpy as np
import torch

O_TOL = 2e-2
LSE_TOL = 1e-3


def nan_like(t: torch.Tensor) -> torch.Tensor:
    return torch.full_like(t, float("nan"))


def nan_empty(shape, dtype, device="cuda") -> torch.Tensor:
    return torch.full(shape, float("nan"), dtype=dtype, device=device)


def check_o(o_gpu: torch.Tensor, o_ref: np.ndarray, vmax: float, tol: float = O_TOL, what: str = "O"):
    o = o_gpu.detach().double().cpu().numpy()
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite values ({np.sum(~np.isfinite(o))})"
    err = np.abs(o - o_ref).max() if o.size else 0.0
    assert err <= tol * vmax, f"{what}: max abs err {err:.3e} > {tol} * {vmax:.3f}"
    return err


def check_lse(l_gpu: torch.Tensor, l_ref: np.ndarray, tol: float = LSE_TOL, what: str = "LSE"):
    l = l_gpu.detach().double().cpu().numpy()
    assert l.shape == l_ref.shape, (l.shape, l_ref.shape)
    empty = np.isneginf(l_ref)
    assert np.all(np.isneginf(l[empty])), f"{what}: empty rows must be -inf"
    assert np.all(np.isfinite(l[~empty])), f"{what}: non-finite values"
    err = np.abs(l[~empty] - l_ref[~empty]).max() if (~empty).any() else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol}"
    return err


def vmax(v: torch.Tensor) -> float:
    return float(v.float().abs().max()) if v.numel() else 1.0
