"""FP8 (e4m3) inputs for the attention forward, in fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Low-precision inputs are among the optimisation directions that
"FlashAttention：优化大模型训练的内存与计算效率" (cnnetsun.cn) lists; the page
names FP8 but fixes no format or scaling. The reading taken: Q, K and V are
stored as 8-bit e4m3 codes with one fp32 dequantisation scale per tensor, so
the value of code c of Q is decode(c) * q_scale. What is computed is exact
attention of the dequantised tensors; any rounding inside an FP8 kernel (of
the probabilities, for instance) is the kernel's, bounded by its tests.

The e4m3 format (the "fn" variant: no infinities): bit 7 sign, bits 6-3 a
4-bit exponent with bias 7, bits 2-0 a 3-bit mantissa. Exponent field 0 is
subnormal: (-1)^s * m/8 * 2^-6. Otherwise (-1)^s * (1 + m/8) * 2^(e - 7),
except that exponent 15 with mantissa 7 is NaN. The largest finite value is
448, the smallest subnormal 2^-9.
"""

from __future__ import annotations

import numpy as np

from .attention import attention_forward_gqa


def e4m3_decode(codes) -> np.ndarray:
    """fp64 values of e4m3 codes (any integer array of 0..255)."""
    c = np.asarray(codes).astype(np.int64) & 0xFF
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    val = np.where((e == 15) & ((c & 0x7) == 7), np.nan, val)
    return sign * val


def _codes(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor (uint8 or float8 viewed as uint8)
        import torch

        x = x.detach().to("cpu")
        if x.dtype != torch.uint8:
            x = x.view(torch.uint8)
        x = x.numpy()
    return np.asarray(x)


def attention_forward_fp8(q8, k8, v8, q_scale: float, k_scale: float, v_scale: float, scale: float,
                          causal: bool, window=None):
    """O and lse of exact attention of the dequantised e4m3 tensors.

    q8 [B, H, N, d], k8 and v8 [B, H_kv, N, d] hold e4m3 codes (uint8); the
    scales are the per-tensor dequantisation factors. Returns (O [B, H, N, d],
    lse [B, H, N]) in fp64."""
    q = e4m3_decode(_codes(q8)) * q_scale
    k = e4m3_decode(_codes(k8)) * k_scale
    v = e4m3_decode(_codes(v8)) * v_scale
    return attention_forward_gqa(q, k, v, scale, causal, window)
