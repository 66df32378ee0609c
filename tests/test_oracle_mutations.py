"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
catch each one. A pin set that lets a dropped term, a wrong sign, an
off-by-one mask or a transposed operand through would be no pin at all."""

import json
import math
import os

import numpy as np
import pytest

import oracle.attention as att

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _golden_ok():
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        a = lambda x: np.asarray(x, dtype=np.float64)[None, None]  # noqa: E731
        o, lse = att.attention_forward(a(c["q"]), a(c["k"]), a(c["v"]), c["scale"], c["causal"])
        if not (np.allclose(o[0, 0], c["o"], rtol=0, atol=1e-12)
                and np.allclose(lse[0, 0], c["lse"], rtol=0, atol=1e-12)):
            return False
        if "dq" in c:
            g = att.attention_backward(a(c["q"]), a(c["k"]), a(c["v"]), a(c["do"]), c["scale"], c["causal"])
            for name, t in zip(("dq", "dk", "dv"), g):
                if not np.allclose(t[0, 0], c[name], rtol=0, atol=1e-12):
                    return False
    return True


def _fd_ok(causal):
    n, d, scale, h = 7, 3, 0.6, 1e-6
    q, k, v, do = (_rand((1, 1, n, d), s) for s in (1, 2, 3, 4))

    def loss(q_, k_, v_):
        o, _ = att.attention_forward(q_, k_, v_, scale, causal)
        return float(np.sum(o * do))

    grads = att.attention_backward(q, k, v, do, scale, causal)
    for which, g in enumerate(grads):
        for idx in np.ndindex(*g.shape):
            ap = [q.copy(), k.copy(), v.copy()]
            am = [q.copy(), k.copy(), v.copy()]
            ap[which][idx] += h
            am[which][idx] -= h
            num = (loss(*ap) - loss(*am)) / (2 * h)
            if abs(num - g[idx]) > 1e-6 * max(1.0, abs(num)):
                return False
    return True


def _closed_form_ok():
    n = 9
    q = np.zeros((1, 1, n, 2))
    k, v = _rand((1, 1, n, 2), 5), _rand((1, 1, n, 2), 6)
    _, lse = att.attention_forward(q, k, v, 1.0, True)
    return np.allclose(lse[0, 0], np.log(np.arange(n) + 1), rtol=0, atol=1e-13)


def test_unmutated_oracle_passes_all_checks():
    assert _golden_ok() and _fd_ok(False) and _fd_ok(True) and _closed_form_ok()


# The planted mask hides every key from query 0, so that row's softmax is
# NaN (inf - inf); the warning is the mistake showing, not a test problem.
@pytest.mark.filterwarnings("ignore:invalid value encountered:RuntimeWarning")
def test_mask_off_by_one_is_caught(monkeypatch):
    monkeypatch.setattr(att, "causal_visible",
                        lambda rows, n: np.arange(n)[None, :] <= np.asarray(rows)[:, None] - 1
                        | (np.arange(n)[None, :] == 0))
    assert not _closed_form_ok()


def test_transposed_p_in_forward_is_caught(monkeypatch):
    orig = att._forward_head

    def bad(q, k, v, scale, causal, rows, window=None):
        s = att._scores(q[rows], k, scale, rows, causal, window)
        p, m, l = att._softmax_rows(s)
        return p.T @ v, m + np.log(l)

    monkeypatch.setattr(att, "_forward_head", bad)
    assert not _golden_ok()
    monkeypatch.setattr(att, "_forward_head", orig)


def test_lse_missing_max_is_caught(monkeypatch):
    def bad_softmax(s):
        m = np.max(s, axis=1, keepdims=True)
        e = np.exp(s - m)
        l = np.sum(e, axis=1, keepdims=True)
        return e / l, np.zeros(s.shape[0]), l[:, 0]

    monkeypatch.setattr(att, "_softmax_rows", bad_softmax)
    assert not _golden_ok()


def _patch_backward(monkeypatch, variant):
    def bwd(q, k, v, do, scale, causal, rows=None, window=None):
        N = q.shape[0]
        r = np.arange(N)
        s = att._scores(q, k, scale, r, causal, window)
        p, _, _ = att._softmax_rows(s)
        dp = do @ v.T
        dd = np.sum(p * dp, axis=1, keepdims=True)
        ds = p * (dp - dd)
        dq, dk, dv = scale * (ds @ k), scale * (ds.T @ q), p.T @ do
        if variant == "no_scale_dk":
            dk = ds.T @ q
        elif variant == "dropped_D":
            dq = scale * ((p * dp) @ k)
        elif variant == "sign":
            dq = -dq
        elif variant == "dv_untransposed":
            dv = p @ do
        elif variant == "D_rowsum_dp":
            ds2 = p * (dp - np.sum(dp, axis=1, keepdims=True))
            dq = scale * (ds2 @ k)
        return dq, dk, dv

    monkeypatch.setattr(att, "_backward_head", bwd)


@pytest.mark.parametrize("variant", ["no_scale_dk", "dropped_D", "sign", "dv_untransposed", "D_rowsum_dp"])
def test_backward_mistakes_are_caught(monkeypatch, variant):
    _patch_backward(monkeypatch, "none")
    assert _fd_ok(True) and _fd_ok(False)
    _patch_backward(monkeypatch, variant)
    assert not (_fd_ok(True) and _fd_ok(False))


def test_scale_misapplied_is_caught(monkeypatch):
    orig_scores = att._scores
    monkeypatch.setattr(att, "_scores", lambda q, k, scale, rows, causal, window=None:
                        orig_scores(q, k, math.sqrt(scale), rows, causal, window))
    assert not _golden_ok()


def _window_ok():
    """The band mask against an explicit per-row listing of visible keys."""
    n, d, scale = 9, 3, 0.7
    q, k, v = (_rand((n, d), s) for s in (11, 12, 13))
    for wl, wr in ((2, 1), (0, 3), (3, 0)):
        o, lse = att.attention_forward(q[None, None], k[None, None], v[None, None], scale, False, window=(wl, wr))
        for i in range(n):
            js = list(range(max(0, i - wl), min(n, i + wr + 1)))
            x = scale * (k[js] @ q[i])
            w = np.exp(x - x.max())
            if not (np.allclose(o[0, 0, i], w @ v[js] / w.sum(), rtol=0, atol=1e-13)
                    and abs(lse[0, 0, i] - (x.max() + np.log(w.sum()))) < 1e-13):
                return False
    return True


def test_unmutated_window_passes():
    assert _window_ok()


@pytest.mark.parametrize("side", ["left", "right"])
def test_window_off_by_one_is_caught(monkeypatch, side):
    orig = att.band_visible

    def bad(rows, n, wl, wr):
        return orig(rows, n, wl - 1 if side == "left" else wl, wr + 1 if side == "right" else wr)

    monkeypatch.setattr(att, "band_visible", bad)
    assert not _window_ok()


def _e4m3_ok(decode):
    import torch

    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = decode(codes.numpy())
    return bool(np.all((np.isnan(ref) & np.isnan(got)) | (ref == got)))


@pytest.mark.parametrize("mistake", ["bias8", "no_subnormal", "mantissa_over_16"])
def test_e4m3_decoder_mistakes_are_caught(mistake):
    import oracle.fp8 as f8

    assert _e4m3_ok(f8.e4m3_decode)

    def bad(codes):
        c = np.asarray(codes).astype(np.int64) & 0xFF
        s = np.where(c & 0x80, -1.0, 1.0)
        e, m = (c >> 3) & 0xF, (c & 7).astype(np.float64)
        bias, div = (8.0 if mistake == "bias8" else 7.0), (16.0 if mistake == "mantissa_over_16" else 8.0)
        norm = (1.0 + m / div) * np.exp2(e - bias)
        sub = norm if mistake == "no_subnormal" else m / div * 2.0 ** (1 - bias)
        v = np.where(e == 0, sub, norm)
        return s * np.where((e == 15) & ((c & 7) == 7), np.nan, v)

    assert not _e4m3_ok(bad)
