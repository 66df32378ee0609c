"""GPU parity of local-window (band) attention (fa_fwd_window, fa_bwd_window)
against the fp64 oracle, through the C ABI.

Key j is visible to query i iff i - wl <= j <= i + wr (negative: unbounded),
the "Local-Window" extension named in cnnetsun.cn's FlashAttention article,
section 6.1. Windows are chosen to cut tiles in every way: narrower than a
tile, exactly one or two tiles, ragged, one-sided and two-sided."""

import numpy as np
import pytest
import torch

from tests._parity import Guarded, check_forward, check_grad, to64
from workloads import make_inputs

pytestmark = pytest.mark.gpu


def _fa():
    import exact_attention_118_b200 as fa

    return fa


def _fwd(q, k, v, wl, wr, scale):
    fa = _fa()
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    stream = torch.cuda.current_stream().cuda_stream
    o = Guarded((B, H, N, d), torch.bfloat16, q.device)
    lse = Guarded((B, H, N), torch.float32, q.device)
    st = fa.fa_fwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.t.data_ptr(), lse.t.data_ptr(), B, H, Hkv, N,
                          d, scale, wl, wr, fa.FA_BF16, stream)
    assert st == fa.FA_OK, fa.fa_strerror(st)
    assert fa.fa_get_device_error(stream) == fa.FA_OK
    assert o.guards_intact() and lse.guards_intact(), "write outside O or lse"
    return o.t, lse.t


def _bwd(q, k, v, o, lse, do, wl, wr, scale):
    fa = _fa()
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    stream = torch.cuda.current_stream().cuda_stream
    dq = Guarded((B, H, N, d), torch.bfloat16, q.device)
    dk = Guarded((B, Hkv, N, d), torch.bfloat16, q.device)
    dv = Guarded((B, Hkv, N, d), torch.bfloat16, q.device)
    ws_bytes = fa.fa_bwd_gqa_workspace_size(B, H, Hkv, N, d)
    ws = Guarded((ws_bytes,), torch.uint8, q.device, fill=0xFF)
    st = fa.fa_bwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                          dq.t.data_ptr(), dk.t.data_ptr(), dv.t.data_ptr(), ws.t.data_ptr(), ws_bytes,
                          B, H, Hkv, N, d, scale, wl, wr, stream)
    assert st == fa.FA_OK, fa.fa_strerror(st)
    assert fa.fa_get_device_error(stream) == fa.FA_OK
    for g in (dq, dk, dv):
        assert g.guards_intact(), "write outside a gradient buffer"
    assert ws.guards_intact(), "write outside the workspace"
    return dq.t, dk.t, dv.t


def _case(B, H, Hkv, N, d, wl, wr, seed):
    from oracle import attention_backward_gqa, attention_forward_gqa

    x = make_inputs(B, H, N, d, seed, kv_heads=Hkv)
    scale = d ** -0.5
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = _fwd(q, k, v, wl, wr, scale)
    what = f"B{B} H{H} Hkv{Hkv} N{N} d{d} window=({wl},{wr})"
    o_ref, lse_ref = attention_forward_gqa(x["q"], x["k"], x["v"], scale, False, window=(wl, wr))
    check_forward(to64(o), to64(lse), o_ref, lse_ref, float(x["v"].abs().max()), what)
    dq, dk, dv = _bwd(q, k, v, o, lse, do, wl, wr, scale)
    rq, rk, rv = attention_backward_gqa(x["q"], x["k"], x["v"], x["do"], scale, False, window=(wl, wr))
    if (wl == 0 and wr == 0) or N == 1:
        # Each query sees only itself: dQ = dK = 0 exactly in the definition;
        # the GPU forms dP - D from two fp32 dot products of d terms.
        assert np.all(rq == 0) and np.all(rk == 0)
        bound = 4 * d * 2.0 ** -24 * float(x["do"].abs().max()) * float(x["v"].abs().max()) * d * scale \
            * max(float(x["k"].abs().max()), float(x["q"].abs().max())) * (H // Hkv)
        check_grad(to64(dq), rq, "dQ", what, bound)
        check_grad(to64(dk), rk, "dK", what, bound)
    else:
        check_grad(to64(dq), rq, "dQ", what)
        check_grad(to64(dk), rk, "dK", what)
    check_grad(to64(dv), rv, "dV", what)


WINDOWS = [(0, 0), (1, 0), (63, 0), (127, 0), (128, 0), (300, 0), (0, 5), (64, 64), (200, 37), (5, -1), (-1, 130)]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [200, 1000])
@pytest.mark.parametrize("wl,wr", WINDOWS)
def test_window_forward_backward(wl, wr, N, d):
    _case(1, 2, 2, N, d, wl, wr, seed=600 + N + 3 * max(wl, 0) + max(wr, 0))


@pytest.mark.parametrize("wl,wr", [(100, 0), (256, 256)])
def test_window_grouped_kv_heads(wl, wr):
    _case(2, 8, 2, 777, 128, wl, wr, seed=650 + wl)


@pytest.mark.parametrize("N", [1, 2, 129])
def test_window_tiny_sequences(N):
    _case(1, 2, 2, N, 64, 1, 0, seed=660 + N)


def test_unbounded_windows_equal_full_and_causal():
    """(-1,-1) and a window covering the sequence are full attention; (-1,0)
    and (N,0) are causal attention: the same kernels, bit for bit."""
    fa = _fa()
    B, H, N, d = 1, 4, 700, 128
    x = make_inputs(B, H, N, d, seed=670, with_grad_out=False)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    scale = d ** -0.5
    stream = torch.cuda.current_stream().cuda_stream
    for causal, windows in ((0, [(-1, -1), (N, N), (N - 1, 5000)]), (1, [(-1, 0), (N, 0), (10 ** 6, 0)])):
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
        assert fa.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d, scale,
                         causal, fa.FA_BF16, stream) == fa.FA_OK
        for wl, wr in windows:
            o2, lse2 = _fwd(q, k, v, wl, wr, scale)
            torch.cuda.synchronize()
            assert torch.equal(o, o2) and torch.equal(lse, lse2), (causal, wl, wr)


def test_sliding_window_long_sequence():
    """A 4096-key sliding causal window over N = 16384 (several heads): the
    forward on sampled query rows, the backward of one head in full."""
    from oracle import attention_backward, attention_forward_rows

    B, H, N, d, wl = 1, 4, 16384, 128, 4095
    x = make_inputs(B, H, N, d, seed=680)
    scale = d ** -0.5
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = _fwd(q, k, v, wl, 0, scale)
    rows = np.unique(np.concatenate([np.arange(0, 300), np.arange(4000, 4200), np.arange(N - 300, N),
                                     np.random.default_rng(0).integers(0, N, 400)]))
    heads = [(0, h) for h in range(H)]
    o_ref, lse_ref = attention_forward_rows(x["q"], x["k"], x["v"], scale, False, heads, rows, window=(wl, 0))
    check_forward(to64(o[0][:, rows]), to64(lse[0][:, rows]), o_ref, lse_ref, float(x["v"].abs().max()),
                  "sliding window N16384")
    dq, dk, dv = _bwd(q, k, v, o, lse, do, wl, 0, scale)
    rq, rk, rv = attention_backward(x["q"], x["k"], x["v"], x["do"], scale, False, heads=[(0, 1)], window=(wl, 0))
    check_grad(to64(dq[0, 1:2]), rq, "dQ", "sliding window N16384")
    check_grad(to64(dk[0, 1:2]), rk, "dK", "sliding window N16384")
    check_grad(to64(dv[0, 1:2]), rv, "dV", "sliding window N16384")
