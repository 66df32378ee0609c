"""Seeded synthetic inputs for exact attention.

This module only draws random tensors. It holds none of the attention
arithmetic, so both the fp64 oracle (``oracle/``) and the CUDA path
(``exact_attention_118_b200``) can take their inputs from it without sharing
any of the method's code.

The five workloads follow the problem statement of the pages: tensors laid out
as ``[B, H, N, d]`` (batch, heads, sequence, head dim), as in the step-1
pseudocode of "写一个flashattention算子" (blog.csdn.net/qq_43527718, the pasted
answer, step 1) and the ``batch, heads, seq_len, dim = q.shape`` unpacking in
"FlashAttention：优化大模型训练的内存与计算效率" (cnnetsun.cn, section 3.1).

Recipe (every workload): a CPU ``torch.Generator`` seeded with the workload's
seed draws ``torch.randn`` fp32 tensors in the order Q, K, V, dO, each of shape
``[B, H, N, d]``; Q and K are multiplied by ``qk_std`` (3 for the long causal
workload, 1 otherwise); then every tensor is rounded to bf16 (round to nearest
even). Both sides consume exactly these bf16 tensors, so parity does not depend
on the generator; reproducibility does.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    seed: int
    backward: bool
    qk_std: float = 1.0
    o_fp32: bool = False

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def shape(self):
        return (self.B, self.H, self.N, self.d)

    def fwd_flops(self) -> float:
        """4*B*H*N^2*d for the two contractions, halved under a causal mask."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        """2.5x the forward count (five contractions instead of two)."""
        return 2.5 * self.fwd_flops()


# The five workloads, named by what they are.
WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("fwd_b1h2_n256_d64", 1, 2, 256, 64, False, 0, False, o_fp32=True),
        Workload("causal_b2h8_n1024_d64", 2, 8, 1024, 64, True, 1, True),
        Workload("b4h16_n4096_d128", 4, 16, 4096, 128, False, 2, True),
        Workload("b1h16_n16384_d128", 1, 16, 16384, 128, False, 3, True),
        Workload("causal_b1h16_n16384_d128", 1, 16, 16384, 128, True, 3, True),
        Workload("causal_b1h32_n32768_d128_qk3", 1, 32, 32768, 128, True, 4, True, qk_std=3.0),
    ]
}


def make_inputs(B: int, H: int, N: int, d: int, seed: int, qk_std: float = 1.0,
                with_grad_out: bool = True, kv_heads: Optional[int] = None):
    """Draw Q, K, V (and dO) as bf16 CPU tensors of shape [B, H, N, d].

    With ``kv_heads`` set (grouped-query attention), K and V are
    [B, kv_heads, N, d] instead. Returns a dict with keys ``q``, ``k``, ``v``
    and, if requested, ``do``.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    shape = (B, H, N, d)
    kv_shape = shape if kv_heads is None else (B, int(kv_heads), N, d)
    out = {}
    for name in ("q", "k", "v", "do"):
        if name == "do" and not with_grad_out:
            break
        t = torch.randn(kv_shape if name in ("k", "v") else shape, generator=g, dtype=torch.float32)
        if name in ("q", "k") and qk_std != 1.0:
            t.mul_(qk_std)
        out[name] = t.to(torch.bfloat16)
    return out


def make_workload_inputs(w: Workload, with_grad_out: Optional[bool] = None):
    if with_grad_out is None:
        with_grad_out = w.backward
    return make_inputs(w.B, w.H, w.N, w.d, w.seed, w.qk_std, with_grad_out)


def make_varlen_inputs(lengths, H: int, Hkv: int, d: int, seed: int, qk_std: float = 1.0):
    """A packed variable-length batch: sequences of the given lengths stored
    back to back. Returns a dict with ``q`` and ``do`` [T, H, d], ``k`` and ``v``
    [T, Hkv, d] (bf16 CPU tensors, drawn in that order from one seeded
    generator) and ``cu_seqlens`` (int32 [B + 1] prefix sums)."""
    lengths = [int(n) for n in lengths]
    T = sum(lengths)
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    out = {}
    for name in ("q", "k", "v", "do"):
        t = torch.randn((T, Hkv if name in ("k", "v") else H, d), generator=g, dtype=torch.float32)
        if name in ("q", "k") and qk_std != 1.0:
            t.mul_(qk_std)
        out[name] = t.to(torch.bfloat16)
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + n)
    out["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32)
    return out


def make_fp8_inputs(B: int, H: int, N: int, d: int, seed: int, kv_heads: Optional[int] = None):
    """Q, K, V as e4m3 codes with per-tensor dequantisation scales.

    Draws standard-normal fp32 Q, K, V (K, V with ``kv_heads`` heads if set)
    from one seeded generator, picks each tensor's scale as its largest
    magnitude / 448 (the largest finite e4m3 value), and rounds x / scale to
    e4m3 with torch's float8_e4m3fn cast. Returns a dict with uint8 tensors
    ``q8``, ``k8``, ``v8`` and floats ``q_scale``, ``k_scale``, ``v_scale``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    Hkv = H if kv_heads is None else int(kv_heads)
    out = {}
    for name, heads in (("q", H), ("k", Hkv), ("v", Hkv)):
        t = torch.randn((B, heads, N, d), generator=g, dtype=torch.float32)
        s = float(t.abs().max()) / 448.0
        out[name + "8"] = (t / s).to(torch.float8_e4m3fn).view(torch.uint8)
        out[name + "_scale"] = s
    return out
