"""Pins for the fp64 oracle: facts fixed by the pages and by the mathematics,
none of which re-types the oracle's own formula.

- hand-worked closed-form cases (tests/golden/hand_cases.json);
- the blockwise online-softmax merge of the pages equals the full-row softmax;
- softmax rows sum to one and are invariant to a per-row shift of S;
- constant V gives O equal to that constant;
- closed forms for Q = 0 and N = 1;
- permutation equivariance (Q rows) and invariance (joint K/V rows);
- backward against central finite differences;
- forward and backward against torch's fp64 CPU SDPA with autograd.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention_backward, attention_forward, attention_forward_rows
from oracle import blockwise_online_softmax_attention

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def _rand(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


def _as4(x):
    return np.asarray(x, dtype=np.float64)[None, None]


# ---------------------------------------------------------------- golden cases

def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_golden_forward(case):
    o, lse = attention_forward(_as4(case["q"]), _as4(case["k"]), _as4(case["v"]),
                               case["scale"], case["causal"])
    np.testing.assert_allclose(o[0, 0], np.array(case["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], np.array(case["lse"]), rtol=0, atol=1e-14)


@pytest.mark.parametrize("case", [c for c in _golden_cases() if "dq" in c], ids=lambda c: c["name"])
def test_golden_backward(case):
    dq, dk, dv = attention_backward(_as4(case["q"]), _as4(case["k"]), _as4(case["v"]),
                                    _as4(case["do"]), case["scale"], case["causal"])
    np.testing.assert_allclose(dq[0, 0], np.array(case["dq"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(dk[0, 0], np.array(case["dk"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(dv[0, 0], np.array(case["dv"]), rtol=0, atol=1e-14)


# ------------------------------------------------- blockwise merge == full rows

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("block", [1, 3, 64, 128, 256])
@pytest.mark.parametrize("deferred", [True, False])
def test_blockwise_online_merge_equals_full_rows(causal, block, deferred):
    # Block sizes: 1 and 3 (ragged), 64 (pasted pseudocode, step 1),
    # 128 and 256 (the V100 and A100 suggestions of cnnetsun.cn section 3.1).
    n, d = 37, 8
    q, k, v = _rand((n, d), 1), _rand((n, d), 2), _rand((n, d), 3)
    scale = 1 / math.sqrt(d)
    o_blk, lse_blk = blockwise_online_softmax_attention(q, k, v, scale, causal, block, deferred)
    o, lse = attention_forward(q[None, None], k[None, None], v[None, None], scale, causal)
    np.testing.assert_allclose(o_blk, o[0, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_blk, lse[0, 0], rtol=0, atol=1e-12)


def test_blockwise_merge_large_logits():
    # Logits of magnitude ~ 100 exercise the running-max correction.
    n, d = 20, 4
    q, k, v = _rand((n, d), 4, 10.0), _rand((n, d), 5, 10.0), _rand((n, d), 6)
    o_blk, lse_blk = blockwise_online_softmax_attention(q, k, v, 1.0, True, 3, True)
    o, lse = attention_forward(q[None, None], k[None, None], v[None, None], 1.0, True)
    assert np.all(np.isfinite(o)) and np.max(np.abs(lse)) > 50
    np.testing.assert_allclose(o_blk, o[0, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_blk, lse[0, 0], rtol=1e-14, atol=1e-12)


# ------------------------------------------------------- softmax row properties

@pytest.mark.parametrize("causal", [False, True])
def test_softmax_rows_sum_to_one(causal):
    # With V = identity (N keys, N value dims) O is the probability matrix P.
    n, d = 13, 5
    q, k = _rand((1, 1, n, d), 7), _rand((1, 1, n, d), 8)
    v = np.eye(n)[None, None]
    p, _ = attention_forward(q, k, v, 0.7, causal)
    p = p[0, 0]
    assert np.all(p >= 0)
    np.testing.assert_allclose(p.sum(axis=1), np.ones(n), rtol=0, atol=1e-14)
    if causal:
        assert np.all(p[np.triu_indices(n, 1)] == 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_per_row_shift_invariance(causal):
    # Append a column c_i/scale to Q and a column of ones to K: S' = S + c_i.
    # P (hence O) must not change; lse must shift by exactly c_i.
    n, d, scale = 11, 6, 0.4
    q, k, v = _rand((n, d), 9), _rand((n, d), 10), _rand((n, d), 11)
    c = _rand((n,), 12, 5.0)
    q2 = np.concatenate([q, (c / scale)[:, None]], axis=1)
    k2 = np.concatenate([k, np.ones((n, 1))], axis=1)
    o1, l1 = attention_forward(q[None, None], k[None, None], v[None, None], scale, causal)
    o2, l2 = attention_forward(q2[None, None], k2[None, None], v[None, None], scale, causal)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2[0, 0], l1[0, 0] + c, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v(causal):
    n, d = 17, 4
    q, k = _rand((2, 3, n, d), 13), _rand((2, 3, n, d), 14)
    row = np.array([1.5, -2.0, 0.25, 7.0])
    v = np.broadcast_to(row, (2, 3, n, d)).copy()
    o, _ = attention_forward(q, k, v, 0.5, causal)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-13)


# ----------------------------------------------------------------- closed forms

@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_closed_form(causal):
    # Q = 0 makes every visible logit 0: uniform weights over visible keys.
    n, d = 19, 3
    q = np.zeros((1, 1, n, d))
    k, v = _rand((1, 1, n, d), 15), _rand((1, 1, n, d), 16)
    o, lse = attention_forward(q, k, v, 1.0, causal)
    idx = np.arange(n)
    if causal:
        np.testing.assert_allclose(lse[0, 0], np.log(idx + 1), rtol=0, atol=1e-14)
        prefix_mean = np.cumsum(v[0, 0], axis=0) / (idx + 1)[:, None]
        np.testing.assert_allclose(o[0, 0], prefix_mean, rtol=0, atol=1e-13)
    else:
        np.testing.assert_allclose(lse[0, 0], np.full(n, math.log(n)), rtol=0, atol=1e-14)
        np.testing.assert_allclose(o[0, 0], np.broadcast_to(v[0, 0].mean(0), (n, d)), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_single_token(causal):
    q, k, v = _rand((1, 2, 1, 8), 17), _rand((1, 2, 1, 8), 18), _rand((1, 2, 1, 8), 19)
    o, lse = attention_forward(q, k, v, 0.3, causal)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, 0.3 * np.sum(q * k, axis=-1), rtol=0, atol=1e-14)


# ------------------------------------------------------------------ symmetries

def test_query_permutation_equivariance():
    n, d = 23, 5
    q, k, v = _rand((1, 1, n, d), 20), _rand((1, 1, n, d), 21), _rand((1, 1, n, d), 22)
    perm = np.random.default_rng(23).permutation(n)
    o, lse = attention_forward(q, k, v, 0.5, False)
    o_p, lse_p = attention_forward(q[:, :, perm], k, v, 0.5, False)
    np.testing.assert_allclose(o_p, o[:, :, perm], rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse_p, lse[:, :, perm], rtol=0, atol=1e-13)


def test_joint_key_value_permutation_invariance():
    n, d = 23, 5
    q, k, v = _rand((1, 1, n, d), 24), _rand((1, 1, n, d), 25), _rand((1, 1, n, d), 26)
    perm = np.random.default_rng(27).permutation(n)
    o, lse = attention_forward(q, k, v, 0.5, False)
    o_p, lse_p = attention_forward(q, k[:, :, perm], v[:, :, perm], 0.5, False)
    np.testing.assert_allclose(o_p, o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse_p, lse, rtol=0, atol=1e-13)


def test_rows_subset_matches_full():
    B, H, n, d = 2, 2, 300, 8
    q, k, v = _rand((B, H, n, d), 28), _rand((B, H, n, d), 29), _rand((B, H, n, d), 30)
    rows = np.array([0, 1, 127, 128, 255, 299])
    heads = [(0, 1), (1, 0)]
    for causal in (False, True):
        o, lse = attention_forward(q, k, v, 0.35, causal)
        o_r, lse_r = attention_forward_rows(q, k, v, 0.35, causal, heads, rows)
        for t, (b, h) in enumerate(heads):
            # same arithmetic, BLAS may block a row subset differently
            np.testing.assert_allclose(o_r[t], o[b, h][rows], rtol=0, atol=1e-13)
            np.testing.assert_allclose(lse_r[t], lse[b, h][rows], rtol=0, atol=1e-13)


# --------------------------------------------------------- finite differences

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n", [1, 9, 16])
def test_backward_central_finite_differences(causal, n):
    d, scale, h = 4, 0.6, 1e-6
    q, k, v, do = (_rand((1, 1, n, d), s) for s in (31, 32, 33, 34))

    def loss(q_, k_, v_):
        o, _ = attention_forward(q_, k_, v_, scale, causal)
        return float(np.sum(o * do))

    grads = attention_backward(q, k, v, do, scale, causal)
    for which, g in enumerate(grads):
        num = np.zeros_like(g)
        for idx in np.ndindex(*g.shape):
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.max(np.abs(num - g)) / max(1e-300, np.max(np.abs(g)))
        if n == 1 and which in (0, 1):
            # one token: O = V does not depend on q or k
            assert np.max(np.abs(g)) == 0.0 and np.max(np.abs(num)) < 1e-9
        else:
            assert err <= 1e-6, (which, err)


# ----------------------------------------------- library special case (torch)

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d", [(1, 8), (17, 16), (130, 64), (257, 32)])
def test_against_torch_sdpa_fp64(causal, n, d):
    B, H = 2, 3
    q, k, v, do = (_rand((B, H, n, d), s) for s in (35, 36, 37, 38))
    scale = 1 / math.sqrt(d)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
    to.backward(torch.tensor(do))
    o, lse = attention_forward(q, k, v, scale, causal)
    dq, dk, dv = attention_backward(q, k, v, do, scale, causal)
    # Tolerance: assert_close(atol=1e-5, rtol=1e-3) of cnnetsun.cn section 5.2,
    # tightened because both sides are fp64.
    kw = dict(rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(o, to.detach().numpy(), **kw)
    np.testing.assert_allclose(dq, tq.grad.numpy(), **kw)
    np.testing.assert_allclose(dk, tk.grad.numpy(), **kw)
    np.testing.assert_allclose(dv, tv.grad.numpy(), **kw)
    # lse via torch.logsumexp of the masked logits
    s = torch.einsum("bhid,bhjd->bhij", torch.tensor(q), torch.tensor(k)) * scale
    if causal:
        s = s.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), **kw)


def test_backward_heads_subset_matches_full():
    B, H, n, d = 1, 3, 40, 8
    q, k, v, do = (_rand((B, H, n, d), s) for s in (39, 40, 41, 42))
    full = attention_backward(q, k, v, do, 0.5, True)
    sub = attention_backward(q, k, v, do, 0.5, True, heads=[(0, 2), (0, 0)])
    for f, s in zip(full, sub):
        np.testing.assert_allclose(s[0], f[0, 2], rtol=0, atol=1e-13)
        np.testing.assert_allclose(s[1], f[0, 0], rtol=0, atol=1e-13)


def test_oracle_accepts_bf16_torch_inputs():
    t = torch.randn(1, 1, 5, 4).to(torch.bfloat16)
    o, _ = attention_forward(t, t, t, 0.5, True)
    o2, _ = attention_forward(t.to(torch.float64).numpy(), t.to(torch.float64).numpy(),
                              t.to(torch.float64).numpy(), 0.5, True)
    np.testing.assert_array_equal(o, o2)
    assert oracle.attention_forward is attention_forward


@pytest.mark.parametrize("causal", [False, True])
def test_backward_rows_partition_sums_to_full(causal):
    from oracle import attention_backward_rows

    B, H, n, d = 1, 2, 300, 8
    q, k, v, do = (_rand((B, H, n, d), s) for s in (43, 44, 45, 46))
    full = attention_backward(q, k, v, do, 0.4, causal)
    heads = [(0, 0), (0, 1)]
    parts = [np.arange(0, 100), np.arange(100, 257), np.arange(257, 300)]
    dk = np.zeros((2, n, d))
    dv = np.zeros((2, n, d))
    for r in parts:
        dq_r, dk_r, dv_r = attention_backward_rows(q, k, v, do, 0.4, causal, heads, r)
        for t, (b, h) in enumerate(heads):
            np.testing.assert_allclose(dq_r[t], full[0][b, h][r], rtol=0, atol=1e-13)
        dk += dk_r
        dv += dv_r
    for t, (b, h) in enumerate(heads):
        np.testing.assert_allclose(dk[t], full[1][b, h], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dv[t], full[2][b, h], rtol=0, atol=1e-12)


# ------------------------------------------------------------ grouped K/V heads

@pytest.mark.parametrize("causal", [False, True])
def test_gqa_backward_finite_differences_on_shared_kv(causal):
    from oracle import attention_backward_gqa, attention_forward_gqa

    B, H, Hkv, n, d, h = 1, 4, 2, 7, 3, 1e-6
    q, do = _rand((B, H, n, d), 50), _rand((B, H, n, d), 51)
    k, v = _rand((B, Hkv, n, d), 52), _rand((B, Hkv, n, d), 53)

    def loss(q_, k_, v_):
        o, _ = attention_forward_gqa(q_, k_, v_, 0.7, causal)
        return float(np.sum(o * do))

    grads = attention_backward_gqa(q, k, v, do, 0.7, causal)
    for which, g in enumerate(grads):
        num = np.zeros_like(g)
        for idx in np.ndindex(*g.shape):
            ap, am = [q.copy(), k.copy(), v.copy()], [q.copy(), k.copy(), v.copy()]
            ap[which][idx] += h
            am[which][idx] -= h
            num[idx] = (loss(*ap) - loss(*am)) / (2 * h)
        assert np.max(np.abs(num - g)) <= 1e-6 * max(1.0, np.max(np.abs(g))), which


def test_mqa_zero_query_closed_form():
    # One shared K/V head, Q = 0: every query head averages the shared V
    # over its visible keys (prefix mean under the causal mask).
    from oracle import attention_forward_gqa

    B, H, n, d = 1, 3, 9, 2
    q = np.zeros((B, H, n, d))
    k, v = _rand((B, 1, n, d), 54), _rand((B, 1, n, d), 55)
    o, lse = attention_forward_gqa(q, k, v, 1.0, True)
    prefix_mean = np.cumsum(v[0, 0], axis=0) / (np.arange(n) + 1)[:, None]
    for hh in range(H):
        np.testing.assert_allclose(o[0, hh], prefix_mean, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[0, hh], np.log(np.arange(n) + 1), rtol=0, atol=1e-14)


def test_gqa_group_size_one_is_mha():
    from oracle import attention_backward_gqa, attention_forward_gqa

    q, k, v, do = (_rand((2, 3, 11, 4), s) for s in (56, 57, 58, 59))
    o1, l1 = attention_forward_gqa(q, k, v, 0.5, True)
    o2, l2 = attention_forward(q, k, v, 0.5, True)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    for a, b in zip(attention_backward_gqa(q, k, v, do, 0.5, True), attention_backward(q, k, v, do, 0.5, True)):
        np.testing.assert_array_equal(a, b)


# ------------------------------------------------------- local-window (band) mask

def _per_row_window_attention(q, k, v, scale, wl, wr):
    """Row by row in plain Python: list the visible keys explicitly (the band
    i - wl <= j <= i + wr, clipped to the sequence), take their exponentials
    relative to the largest logit, and average V with those weights."""
    n, d = len(q), len(q[0])
    o, lse = [], []
    for i in range(n):
        lo = 0 if wl < 0 else max(0, i - wl)
        hi = n - 1 if wr < 0 else min(n - 1, i + wr)
        logits = [scale * sum(q[i][c] * k[j][c] for c in range(d)) for j in range(lo, hi + 1)]
        mx = max(logits)
        w = [math.exp(x - mx) for x in logits]
        tot = sum(w)
        o.append([sum(w[t] * v[lo + t][c] for t in range(len(w))) / tot for c in range(v.shape[1])])
        lse.append(mx + math.log(tot))
    return np.array(o), np.array(lse)


@pytest.mark.parametrize("wl,wr", [(0, 0), (1, 0), (2, 3), (3, -1), (-1, 2), (5, 5), (0, -1)])
def test_window_against_per_row_python(wl, wr):
    n, d = 9, 3
    q, k, v = (_rand((n, d), s) for s in (81, 82, 83))
    o, lse = attention_forward(_as4(q), _as4(k), _as4(v), 0.7, False, window=(wl, wr))
    o_ref, lse_ref = _per_row_window_attention(q, k, v, 0.7, wl, wr)
    assert np.allclose(o[0, 0], o_ref, rtol=0, atol=1e-13)
    assert np.allclose(lse[0, 0], lse_ref, rtol=0, atol=1e-13)


def test_window_zero_width_closed_form():
    """wl = wr = 0: each query sees only its own key, so O = V and
    lse_i = scale * q_i . k_i exactly."""
    n, d = 12, 5
    q, k, v = (_rand((1, 2, n, d), s) for s in (84, 85, 86))
    o, lse = attention_forward(q, k, v, 0.3, False, window=(0, 0))
    assert np.array_equal(o, v)
    assert np.allclose(lse, 0.3 * np.sum(q * k, axis=-1), rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_window_unbounded_equals_full_and_causal(causal):
    n, d = 33, 8
    q, k, v = (_rand((1, 1, n, d), s) for s in (87, 88, 89))
    o_ref, lse_ref = attention_forward(q, k, v, 0.5, causal)
    windows = [(-1, -1), (n, n), (n - 1, -1)] + ([(-1, 0), (n, 0)] if causal else [])
    for w in windows:
        wc = (w[0], 0) if causal and w[1] < 0 else w
        o, lse = attention_forward(q, k, v, 0.5, False, window=wc) if causal and wc[1] == 0 else \
            attention_forward(q, k, v, 0.5, causal, window=w)
        assert np.array_equal(o, o_ref) and np.array_equal(lse, lse_ref), w


@pytest.mark.parametrize("wl,wr", [(2, 0), (1, 2), (0, 0)])
def test_window_backward_central_finite_differences(wl, wr):
    n, d, scale, h = 8, 3, 0.6, 1e-6
    q, k, v, do = (_rand((1, 1, n, d), s) for s in (91, 92, 93, 94))

    def loss(q_, k_, v_):
        o, _ = attention_forward(q_, k_, v_, scale, False, window=(wl, wr))
        return float(np.sum(o * do))

    grads = attention_backward(q, k, v, do, scale, False, window=(wl, wr))
    for which, g in enumerate(grads):
        num = np.zeros_like(g)
        for idx in np.ndindex(*g.shape):
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        if wl == 0 and wr == 0 and which in (0, 1):
            assert np.max(np.abs(g)) == 0.0 and np.max(np.abs(num)) < 1e-9
        else:
            err = np.max(np.abs(num - g)) / np.max(np.abs(g))
            assert err <= 1e-6, (which, err)


# ------------------------------------------------------ variable-length batches

def test_varlen_against_per_row_python():
    """Three packed sequences (one empty), causal and full: every row against
    a plain-Python softmax over the keys of its own sequence only."""
    from oracle import attention_forward_varlen

    cu = [0, 4, 4, 11, 13]
    T, H, d = 13, 2, 3
    q, k, v = (_rand((T, H, d), s) for s in (101, 102, 103))
    for causal in (False, True):
        o, lse = attention_forward_varlen(q, k, v, np.array(cu), 0.8, causal)
        for a, e in zip(cu[:-1], cu[1:]):
            for i in range(a, e):
                for h in range(H):
                    keys = range(a, i + 1) if causal else range(a, e)
                    x = [0.8 * sum(q[i, h, c] * k[j, h, c] for c in range(d)) for j in keys]
                    mx = max(x)
                    w = [math.exp(t - mx) for t in x]
                    ref = [sum(wt * v[j, h, c] for wt, j in zip(w, keys)) / sum(w) for c in range(d)]
                    assert np.allclose(o[i, h], ref, rtol=0, atol=1e-13)
                    assert abs(lse[h, i] - (mx + math.log(sum(w)))) < 1e-13


def test_varlen_equal_lengths_is_the_fixed_batch():
    from oracle import attention_backward_varlen, attention_forward_varlen

    B, H, N, d = 3, 2, 10, 4
    q, k, v, do = (_rand((B, H, N, d), s) for s in (111, 112, 113, 114))
    packed = lambda x: np.transpose(x, (0, 2, 1, 3)).reshape(B * N, H, d)  # noqa: E731
    cu = np.arange(B + 1) * N
    for causal in (False, True):
        o, lse = attention_forward_varlen(packed(q), packed(k), packed(v), cu, 0.5, causal)
        o_ref, lse_ref = attention_forward(q, k, v, 0.5, causal)
        assert np.array_equal(o, packed(o_ref))
        assert np.array_equal(lse, np.transpose(lse_ref, (1, 0, 2)).reshape(H, B * N))
        g = attention_backward_varlen(packed(q), packed(k), packed(v), packed(do), cu, 0.5, causal)
        g_ref = attention_backward(q, k, v, do, 0.5, causal)
        for a, b in zip(g, g_ref):
            assert np.array_equal(a, packed(b))


def test_varlen_sequences_are_independent():
    from oracle import attention_forward_varlen

    cu = np.array([0, 5, 12, 20])
    q, k, v = (_rand((20, 2, 4), s) for s in (121, 122, 123))
    o, _ = attention_forward_varlen(q, k, v, cu, 0.7, False)
    k2, v2 = k.copy(), v.copy()
    k2[5:12] += 3.0
    v2[5:12] -= 1.0
    o2, _ = attention_forward_varlen(q, k2, v2, cu, 0.7, False)
    assert np.array_equal(o[:5], o2[:5]) and np.array_equal(o[12:], o2[12:])
    assert not np.allclose(o[5:12], o2[5:12])


# ------------------------------------------------------------ FP8 (e4m3) inputs

def test_e4m3_decode_matches_torch_for_every_code():
    from oracle import e4m3_decode

    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = e4m3_decode(codes.numpy())
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.all(both_nan | (ref == got))
    assert np.sum(np.isnan(got)) == 2  # 0x7F and 0xFF


def test_e4m3_decode_hand_values():
    from oracle import e4m3_decode

    table = {0x00: 0.0, 0x80: -0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0,
             0x39: 1.125, 0xB8: -1.0, 0x40: 2.0, 0x7E: 448.0, 0xFE: -448.0, 0x77: 240.0, 0x30: 0.5}
    for c, want in table.items():
        assert e4m3_decode(np.array([c]))[0] == want, hex(c)
    assert np.isnan(e4m3_decode(np.array([0x7F]))[0])


def _fp8_case(seed, n=40, d=16):
    g = np.random.default_rng(seed)
    return [g.integers(0, 256, (1, 2, n, d)) for _ in range(3)]


def _finite(codes):
    return np.where((codes & 0x7F) == 0x7F, 0x38, codes)  # replace NaN codes by 1.0


def test_fp8_scale_trades_with_softmax_scale():
    from oracle import attention_forward_fp8

    q8, k8, v8 = (_finite(c) for c in _fp8_case(131))
    o1, l1 = attention_forward_fp8(q8, k8, v8, 0.01, 0.02, 0.5, 0.125, True)
    o2, l2 = attention_forward_fp8(q8, k8, v8, 0.02, 0.04, 0.5, 0.125 / 4, True)
    assert np.allclose(o1, o2, rtol=1e-13, atol=1e-15) and np.allclose(l1, l2, rtol=1e-13, atol=1e-13)


def test_fp8_v_scale_is_linear_and_leaves_lse():
    from oracle import attention_forward_fp8

    q8, k8, v8 = (_finite(c) for c in _fp8_case(132))
    o1, l1 = attention_forward_fp8(q8, k8, v8, 0.01, 0.02, 0.5, 0.125, False)
    o2, l2 = attention_forward_fp8(q8, k8, v8, 0.01, 0.02, 1.5, 0.125, False)
    assert np.allclose(o2, 3.0 * o1, rtol=1e-13, atol=1e-15) and np.array_equal(l1, l2)
