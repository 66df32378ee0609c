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


def check_grad(g_gpu, g_ref, name, what=""):
    g_gpu = np.asarray(g_gpu)
    assert np.all(np.isfinite(g_gpu)), f"{what}: non-finite {name}"
    ref_max = float(np.max(np.abs(g_ref)))
    err = float(np.max(np.abs(g_gpu - g_ref)))
    assert err <= GRAD_TOL * ref_max, f"{what}: max|{name} err| {err:.3e} > {GRAD_TOL * ref_max:.3e}"
    return err


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
