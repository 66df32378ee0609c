"""Shared helpers for the GPU parity tests (tolerances, guarded buffers)."""

from __future__ import annotations

import numpy as np
import torch

# Tolerances for bf16 inputs, fp32 accumulation against the fp64 oracle on the
# same bf16-rounded inputs:
#   max |O - O_ref|   <= 1e-2 * max |V|
#   max |lse - lse_ref| <= 1e-3 (absolute)
#   max |dX - dX_ref| <= 2e-2 * max |dX_ref|   for X in Q, K, V
O_TOL = 1e-2
LSE_TOL = 1e-3
GRAD_TOL = 2e-2


def to64(t) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def check_forward(o_gpu, lse_gpu, o_ref, lse_ref, vmax, what=""):
    o_gpu, lse_gpu = np.asarray(o_gpu), np.asarray(lse_gpu)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite O"
    assert np.all(np.isfinite(lse_gpu)), f"{what}: non-finite lse"
    e_o = float(np.max(np.abs(o_gpu - o_ref)))
    e_l = float(np.max(np.abs(lse_gpu - lse_ref)))
    assert e_o <= O_TOL * vmax, f"{what}: max|O err| {e_o:.3e} > {O_TOL * vmax:.3e}"
    assert e_l <= LSE_TOL, f"{what}: max|lse err| {e_l:.3e} > {LSE_TOL}"
    return e_o, e_l


def check_grad(g_gpu, g_ref, name, what="", zero_bound=0.0):
    """max|g - ref| <= 2e-2 * max|ref|. Where the exact gradient is identically
    zero (a degenerate case), the relative bar is empty and the caller passes
    the absolute rounding bound ``zero_bound`` that the result must meet."""
    g_gpu = np.asarray(g_gpu)
    assert np.all(np.isfinite(g_gpu)), f"{what}: non-finite {name}"
    ref_max = float(np.max(np.abs(g_ref)))
    err = float(np.max(np.abs(g_gpu - g_ref)))
    bar = GRAD_TOL * ref_max if ref_max > 0 else zero_bound
    assert err <= bar, f"{what}: max|{name} err| {err:.3e} > {bar:.3e}"
    return err


def single_key_zero_bound(x, scale):
    """Rounding bound for dQ and dK when N = 1.

    With one key the softmax is identically 1, so dS = P (dP - D) = dP - D is
    exactly 0 and so are dQ = scale dS K and dK = scale dS^T Q. The GPU forms dP
    (tensor-core dot product of dO and V) and D (dot product of dO and the bf16
    O = V) separately in fp32. Each bf16 x bf16 product is exact in fp32, so
    each sum of d terms is off by at most d * u * sum|dO_k V_k| (u = 2^-24);
    |dP - D| <= 2 d u max|dO| max|V| d, and the gradient is that times
    scale * max(|K|, |Q|)."""
    d = x["q"].shape[-1]
    u = 2.0 ** -24
    mx = lambda t: float(t.abs().max())  # noqa: E731
    return scale * max(mx(x["k"]), mx(x["q"])) * 2 * d * d * u * mx(x["do"]) * mx(x["v"])


class Guarded:
    """A device buffer with sentinel guard bands before and after the payload.

    The payload starts 256 bytes into the allocation, so it keeps the
    alignment the ABI asks for; the guards must be intact after a call."""

    GUARD = 256

    def __init__(self, shape, dtype, device, fill=float("nan")):
        self.shape = tuple(shape)
        self.dtype = dtype
        esz = torch.empty((), dtype=dtype).element_size()
        n = int(np.prod(self.shape))
        g = self.GUARD // esz
        self.raw = torch.empty(n + 2 * g, dtype=dtype, device=device)
        self.raw.fill_(-12345.0 if dtype.is_floating_point else 0x5A)
        self.g = g
        self.n = n
        self.t = self.raw[g:g + n].view(self.shape)
        self.t.fill_(fill)

    def guards_intact(self) -> bool:
        head = self.raw[: self.g]
        tail = self.raw[self.g + self.n:]
        want = -12345.0 if self.dtype.is_floating_point else 0x5A
        return bool(torch.all(head == want).item() and torch.all(tail == want).item())
