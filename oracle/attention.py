"""Standard (unfused) attention in fp64, forward and backward.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

Definition followed. "FlashAttention原理：从原始Attention到FlashAttention"
(blog.csdn.net/qq_43527718), section 二.2, lists the standard computation for
Q, K, V of size N x d: S = Q K^T, P = softmax(S), O = P V, with S and P written
out in full. The same page (section 二.1) states that FlashAttention computes
exactly this result ("exact attention"), so the plain definition is the
oracle. The scale factor 1/sqrt(d) appears in the score step of the pasted
pseudocode on that page (step 3); here it is an argument.

The softmax is the "safe" form that subtracts the row maximum before the
exponential, as in the ``safe_softmax`` snippet of "FlashAttention：优化大模型
训练的内存与计算效率" (cnnetsun.cn), section 2.2.

Readings of points the pages leave open:
- causal mask: key j is visible to query i iff j <= i (square problem, N_q =
  N_k). Masked logits are -inf before the row max, so they contribute exactly
  0. With j <= i no row is ever fully masked.
- local window ("Local-Window" among the sparse extensions listed in
  "FlashAttention：优化大模型训练的内存与计算效率", cnnetsun.cn, section 6.1;
  the page gives only the name): ``window = (wl, wr)`` makes key j visible to
  query i iff i - wl <= j <= i + wr, a negative bound meaning no limit on that
  side. It combines with ``causal`` by intersection; (-1, 0) is the causal
  mask. With wl, wr >= 0 the diagonal is always visible, so no row is empty.
- lse is the natural logarithm of sum_j exp(scale * q_i . k_j) over visible j:
  lse_i = m_i + ln(l_i) where m_i is the row max of the scaled logits and l_i
  the row sum of exp(S - m_i). The pages say only that the forward stores the
  softmax normalisation factor (blog.csdn.net/qq_43527718, section 二 "做法")
  and works in log space (cnnetsun.cn, section 2.2).
- backward: the pages say only that the backward recomputes the attention
  matrix from the stored normalisation factor instead of reading it from HBM
  (blog.csdn.net/qq_43527718, sections 二 "做法" and 二.5). The gradient
  formulas are the calculus of the forward:
      dV = P^T dO,  dP = dO V^T,  D_i = sum_j P_ij dP_ij,
      dS = P * (dP - D),  dQ = scale * dS K,  dK = scale * dS^T Q.
  They are pinned by central finite differences.

Inputs may be any array-like (numpy, torch CPU tensors of any float dtype);
they are converted to fp64 first. Work is done per (batch, head) and in
chunks of query rows; every chunk holds full rows of S.
"""

from __future__ import annotations

import numpy as np

_CHUNK = 1024


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu")
        import torch

        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def causal_visible(rows: np.ndarray, n_keys: int) -> np.ndarray:
    """Boolean [len(rows), n_keys] matrix: key j visible to query i iff j <= i."""
    return np.arange(n_keys)[None, :] <= np.asarray(rows)[:, None]


def band_visible(rows: np.ndarray, n_keys: int, wl: int, wr: int) -> np.ndarray:
    """Boolean [len(rows), n_keys] matrix: key j visible to query i iff
    i - wl <= j <= i + wr (a negative wl or wr: no bound on that side)."""
    j = np.arange(n_keys)[None, :]
    i = np.asarray(rows)[:, None]
    vis = np.ones((len(rows), n_keys), dtype=bool)
    if wl >= 0:
        vis &= j >= i - wl
    if wr >= 0:
        vis &= j <= i + wr
    return vis


def _scores(q_rows: np.ndarray, k: np.ndarray, scale: float, rows: np.ndarray,
            causal: bool, window=None) -> np.ndarray:
    """S = scale * Q K^T for the given query rows, masked entries set to -inf."""
    s = (q_rows @ k.T) * scale
    if causal:
        s = np.where(causal_visible(rows, k.shape[0]), s, -np.inf)
    if window is not None:
        s = np.where(band_visible(rows, k.shape[0], window[0], window[1]), s, -np.inf)
    return s


def _softmax_rows(s: np.ndarray):
    """Row softmax with the max subtracted; returns (P, m, l)."""
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    return e / l, m[:, 0], l[:, 0]


def _forward_head(q, k, v, scale, causal, rows, window=None):
    o = np.empty((len(rows), v.shape[1]))
    lse = np.empty(len(rows))
    for c0 in range(0, len(rows), _CHUNK):
        r = rows[c0:c0 + _CHUNK]
        s = _scores(q[r], k, scale, r, causal, window)
        p, m, l = _softmax_rows(s)
        o[c0:c0 + len(r)] = p @ v
        lse[c0:c0 + len(r)] = m + np.log(l)
    return o, lse


def attention_forward(q, k, v, scale: float, causal: bool, window=None):
    """O and lse of exact attention.

    q, k, v: [B, H, N, d]; window: None or (wl, wr), see the module notes.
    Returns (O [B, H, N, d] fp64, lse [B, H, N] fp64).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, _ = q.shape
    o = np.empty(q.shape[:3] + (v.shape[3],))
    lse = np.empty((B, H, N))
    rows = np.arange(N)
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = _forward_head(q[b, h], k[b, h], v[b, h], scale, causal, rows, window)
    return o, lse


def attention_forward_rows(q, k, v, scale: float, causal: bool, heads, rows, window=None):
    """O and lse for selected (b, h) heads and query rows only.

    heads: list of (b, h) pairs; rows: 1-D array of query indices.
    Returns (O [len(heads), len(rows), d], lse [len(heads), len(rows)]).
    """
    rows = np.asarray(rows, dtype=np.int64)
    outs_o, outs_l = [], []
    for (b, h) in heads:
        qh, kh, vh = _f64(q[b, h]), _f64(k[b, h]), _f64(v[b, h])
        o, l = _forward_head(qh, kh, vh, scale, causal, rows, window)
        outs_o.append(o)
        outs_l.append(l)
    return np.stack(outs_o), np.stack(outs_l)


def _backward_head(q, k, v, do, scale, causal, rows=None, window=None):
    """Gradients from the query rows ``rows`` (all rows if None) of one head.

    dQ is returned for those rows only; dK and dV are the contributions of
    those rows (they sum to the full dK, dV over any partition of the rows)."""
    N = q.shape[0]
    rows = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    dq = np.zeros((len(rows), q.shape[1]))
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for c0 in range(0, len(rows), _CHUNK):
        r = rows[c0:c0 + _CHUNK]
        s = _scores(q[r], k, scale, r, causal, window)
        p, _, _ = _softmax_rows(s)          # recomputed from the definition
        dv += p.T @ do[r]                   # dV = P^T dO
        dp = do[r] @ v.T                    # dP = dO V^T
        dd = np.sum(p * dp, axis=1, keepdims=True)   # D_i = sum_j P_ij dP_ij
        ds = p * (dp - dd)                  # softmax Jacobian applied to dP
        dq[c0:c0 + len(r)] = scale * (ds @ k)   # dQ = scale dS K
        dk += scale * (ds.T @ q[r])         # dK = scale dS^T Q
    return dq, dk, dv


def attention_backward_rows(q, k, v, do, scale: float, causal: bool, heads, rows):
    """Work of the query rows ``rows`` of the given (b, h) heads: dQ for those
    rows [len(heads), len(rows), d], and their contributions to dK and dV
    [len(heads), N, d]. Used to time a bounded sample of a large workload."""
    res = [
        _backward_head(_f64(q[b, h]), _f64(k[b, h]), _f64(v[b, h]), _f64(do[b, h]), scale, causal, rows)
        for (b, h) in heads
    ]
    return tuple(np.stack([r[i] for r in res]) for i in range(3))


def attention_backward(q, k, v, do, scale: float, causal: bool, heads=None, window=None):
    """dQ, dK, dV of exact attention for upstream gradient dO.

    All inputs [B, H, N, d]. If ``heads`` (a list of (b, h)) is given, only those
    heads are computed and the results are stacked as [len(heads), N, d].
    window: None or (wl, wr), see the module notes.
    """
    if heads is not None:
        res = [
            _backward_head(_f64(q[b, h]), _f64(k[b, h]), _f64(v[b, h]), _f64(do[b, h]), scale, causal,
                           window=window)
            for (b, h) in heads
        ]
        return tuple(np.stack([r[i] for r in res]) for i in range(3))
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H = q.shape[:2]
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    for b in range(B):
        for h in range(H):
            dq[b, h], dk[b, h], dv[b, h] = _backward_head(q[b, h], k[b, h], v[b, h], do[b, h], scale, causal,
                                                          window=window)
    return dq, dk, dv


# ---------------------------------------------------------------- grouped K/V
# Multi-query / grouped-query attention: several query heads share one K/V
# head ("FlashAttention原理：从原始Attention到FlashAttention", blog.csdn.net,
# related-article notes on MQA/GQA: in MQA the query keeps all its heads while
# key and value keep a single shared head). Query head h of H reads K/V head
# h // (H // H_kv). The definition is standard attention with every K/V head
# repeated for its group; the gradient of a shared K/V head is the sum of the
# gradients its group's query heads send it.

def _repeat_kv(x, group: int) -> np.ndarray:
    return np.repeat(_f64(x), group, axis=1)


def attention_forward_gqa(q, k, v, scale: float, causal: bool, window=None):
    """q [B, H, N, d]; k, v [B, H_kv, N, d] with H % H_kv == 0."""
    H, Hkv = q.shape[1], k.shape[1]
    assert H % Hkv == 0
    g = H // Hkv
    return attention_forward(q, _repeat_kv(k, g), _repeat_kv(v, g), scale, causal, window)


def attention_backward_gqa(q, k, v, do, scale: float, causal: bool, window=None):
    """dQ [B, H, N, d]; dK, dV [B, H_kv, N, d] (summed over each group)."""
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    g = H // Hkv
    dq, dk, dv = attention_backward(q, _repeat_kv(k, g), _repeat_kv(v, g), do, scale, causal, window=window)
    return dq, dk.reshape(B, Hkv, g, N, -1).sum(axis=2), dv.reshape(B, Hkv, g, N, -1).sum(axis=2)


# ------------------------------------------------------ variable-length batches
# Packed variable-length batches (the dynamic-shape support listed among the
# optimisation directions of "FlashAttention：优化大模型训练的内存与计算效率",
# cnnetsun.cn): B sequences of different lengths stored back to back without
# padding, q [T, H, d], k and v [T, H_kv, d], sequence b in rows
# [cu[b], cu[b + 1]). Each sequence is attended on its own, as a batch of one
# (masks apply within the sequence). lse is [H, T].

def _sequence(x, a, e):
    """Rows [a, e) of a packed [T, heads, d] array as a [1, heads, L, d] batch."""
    return np.transpose(x[a:e], (1, 0, 2))[None]


def attention_forward_varlen(q, k, v, cu_seqlens, scale: float, causal: bool, window=None):
    """O [T, H, d] and lse [H, T] of packed variable-length attention. Rows no
    sequence covers are left NaN."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    T, H, d = q.shape
    o = np.full((T, H, v.shape[2]), np.nan)
    lse = np.full((H, T), np.nan)
    for a, e in zip(cu[:-1], cu[1:]):
        if e > a:
            ob, lb = attention_forward_gqa(_sequence(q, a, e), _sequence(k, a, e), _sequence(v, a, e), scale, causal,
                                           window)
            o[a:e] = np.transpose(ob[0], (1, 0, 2))
            lse[:, a:e] = lb[0]
    return o, lse


def attention_backward_varlen(q, k, v, do, cu_seqlens, scale: float, causal: bool, window=None):
    """dQ [T, H, d], dK and dV [T, H_kv, d] of packed variable-length attention."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    dq, dk, dv = np.full(q.shape, np.nan), np.full(k.shape, np.nan), np.full(v.shape, np.nan)
    for a, e in zip(cu[:-1], cu[1:]):
        if e > a:
            g = attention_backward_gqa(_sequence(q, a, e), _sequence(k, a, e), _sequence(v, a, e),
                                       _sequence(do, a, e), scale, causal, window)
            for out, gb in zip((dq, dk, dv), g):
                out[a:e] = np.transpose(gb[0], (1, 0, 2))
    return dq, dk, dv
