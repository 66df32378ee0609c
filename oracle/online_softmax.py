"""Blockwise (online) softmax attention, step by step, in fp64 pure Python/NumPy.

TEST INFRASTRUCTURE ONLY: used to pin the full-row oracle, never by the
product path.

It follows the merge rule the pages describe. "FlashAttention：优化大模型训练
的内存与计算效率" (cnnetsun.cn, section 2.2) keeps a max value and a sum value
per block and corrects the partial results when blocks are combined;
"FlashAttention原理：从原始Attention到FlashAttention" (blog.csdn.net/qq_43527718,
section 二.6) names the kept quantities m(x^1), l(x^1), m(x^2), l(x^2). The
pasted answer on the same page (steps 4 and 5) spells the merge out:
    m_new = max(m_prev, m_blk)
    l_new = e^(m_prev - m_new) l_prev + e^(m_blk - m_new) l_blk
    O_new = (e^(m_prev - m_new) l_prev O_prev + e^(m_blk - m_new) P_blk V_blk) / l_new
with P_blk = e^(S_blk - m_blk). That form renormalises O at every step
(``deferred=False``). Section 二.7 of the blog says FlashAttention-2 removes
non-matmul work; the usual reading is to keep O un-normalised and divide by l
once at the end (``deferred=True``). Both are the same mathematics, so both
must reproduce the full-row softmax.

Keys are visited in blocks of ``block`` columns. A block whose entries are all
masked for a row contributes nothing to that row.
"""

from __future__ import annotations

import numpy as np


def blockwise_online_softmax_attention(q, k, v, scale, causal, block, deferred=True):
    """One head: q [Nq, d], k [Nk, d], v [Nk, dv] (fp64). Returns (O, lse)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    nq, nk = q.shape[0], k.shape[0]
    o_out = np.zeros((nq, v.shape[1]))
    lse_out = np.zeros(nq)
    for i in range(nq):
        m_prev = -np.inf
        l_prev = 0.0
        acc = np.zeros(v.shape[1])
        for j0 in range(0, nk, block):
            cols = [j for j in range(j0, min(nk, j0 + block)) if (not causal or j <= i)]
            if not cols:
                continue
            s_blk = np.array([scale * float(np.dot(q[i], k[j])) for j in cols])
            m_blk = float(np.max(s_blk))
            p_blk = np.exp(s_blk - m_blk)
            l_blk = float(np.sum(p_blk))
            pv_blk = p_blk @ v[cols]
            m_new = max(m_prev, m_blk)
            a_prev = np.exp(m_prev - m_new) if l_prev > 0.0 else 0.0
            a_blk = np.exp(m_blk - m_new)
            l_new = a_prev * l_prev + a_blk * l_blk
            if deferred:
                # un-normalised accumulator; one division at the end
                acc = a_prev * acc + a_blk * pv_blk
            else:
                # renormalise at every step (O holds a proper average)
                acc = (a_prev * l_prev * acc + a_blk * pv_blk) / l_new
            m_prev, l_prev = m_new, l_new
        o_out[i] = acc / l_prev if deferred else acc
        lse_out[i] = m_prev + np.log(l_prev)
    return o_out, lse_out
