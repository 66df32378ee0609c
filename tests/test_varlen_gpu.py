"""GPU parity of packed variable-length attention (fa_fwd_varlen,
fa_bwd_varlen) against the fp64 oracle, through the C ABI.

Sequences of mixed lengths (empty, one token, tile-sized, ragged, long) are
packed back to back as [T, heads, d]; each is attended on its own."""

import numpy as np
import pytest
import torch

from tests._parity import Guarded, check_forward, check_grad, to64
from workloads import make_inputs, make_varlen_inputs

pytestmark = pytest.mark.gpu

MIXES = {
    "mixed": [300, 1, 128, 0, 129, 1000, 64, 513],
    "one_long": [2048],
    "many_short": [17] * 23 + [5, 250],
}


def _fa():
    import exact_attention_118_b200 as fa

    return fa


def _fwd(x, H, Hkv, d, max_len, wl, wr, scale):
    fa = _fa()
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    cu = x["cu_seqlens"].cuda()
    T, B = q.shape[0], cu.numel() - 1
    stream = torch.cuda.current_stream().cuda_stream
    o = Guarded((T, H, d), torch.bfloat16, q.device)
    lse = Guarded((H, T), torch.float32, q.device)
    st = fa.fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.t.data_ptr(), lse.t.data_ptr(), cu.data_ptr(),
                          B, max_len, T, H, Hkv, d, scale, wl, wr, fa.FA_BF16, stream)
    assert st == fa.FA_OK, fa.fa_strerror(st)
    err = fa.fa_get_device_error(stream)
    assert o.guards_intact() and lse.guards_intact(), "write outside O or lse"
    return o.t, lse.t, err


def _bwd(x, o, lse, H, Hkv, d, max_len, wl, wr, scale):
    fa = _fa()
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    cu = x["cu_seqlens"].cuda()
    T, B = q.shape[0], cu.numel() - 1
    stream = torch.cuda.current_stream().cuda_stream
    dq = Guarded((T, H, d), torch.bfloat16, q.device)
    dk = Guarded((T, Hkv, d), torch.bfloat16, q.device)
    dv = Guarded((T, Hkv, d), torch.bfloat16, q.device)
    ws_bytes = fa.fa_bwd_varlen_workspace_size(B, T, H, Hkv, d)
    ws = Guarded((ws_bytes,), torch.uint8, q.device, fill=0xFF)
    st = fa.fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                          dq.t.data_ptr(), dk.t.data_ptr(), dv.t.data_ptr(), cu.data_ptr(), ws.t.data_ptr(), ws_bytes,
                          B, max_len, T, H, Hkv, d, scale, wl, wr, stream)
    assert st == fa.FA_OK, fa.fa_strerror(st)
    err = fa.fa_get_device_error(stream)
    for g in (dq, dk, dv):
        assert g.guards_intact(), "write outside a gradient buffer"
    assert ws.guards_intact(), "write outside the workspace"
    return dq.t, dk.t, dv.t, err


def _case(lengths, H, Hkv, d, wl, wr, seed):
    from oracle import attention_backward_varlen, attention_forward_varlen

    fa = _fa()
    x = make_varlen_inputs(lengths, H, Hkv, d, seed)
    scale = d ** -0.5
    max_len = max(max(lengths), 1)
    o, lse, err = _fwd(x, H, Hkv, d, max_len, wl, wr, scale)
    assert err == fa.FA_OK
    window = (wl, wr)
    o_ref, lse_ref = attention_forward_varlen(x["q"], x["k"], x["v"], x["cu_seqlens"].numpy(), scale, False, window)
    what = f"lengths {lengths[:6]}... H{H} Hkv{Hkv} d{d} window=({wl},{wr})"
    check_forward(to64(o), to64(lse), o_ref, lse_ref, float(x["v"].abs().max()), what)
    dq, dk, dv, err = _bwd(x, o, lse, H, Hkv, d, max_len, wl, wr, scale)
    assert err == fa.FA_OK
    rq, rk, rv = attention_backward_varlen(x["q"], x["k"], x["v"], x["do"], x["cu_seqlens"].numpy(), scale, False,
                                           window)
    # One-token sequences have dQ = dK = 0 exactly; every other row is held
    # to the relative bar, measured against the largest reference gradient.
    check_grad(to64(dq), rq, "dQ", what)
    check_grad(to64(dk), rk, "dK", what)
    check_grad(to64(dv), rv, "dV", what)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("wl,wr", [(-1, -1), (-1, 0), (100, 0), (64, 200)])
@pytest.mark.parametrize("mix", sorted(MIXES))
def test_varlen_forward_backward(mix, wl, wr, d):
    _case(MIXES[mix], 4, 2, d, wl, wr, seed=700 + len(MIXES[mix]) + d + max(wl, 0))


@pytest.mark.parametrize("Hkv", [1, 8])
def test_varlen_head_groupings(Hkv):
    _case(MIXES["mixed"], 8, Hkv, 128, -1, 0, seed=750 + Hkv)


@pytest.mark.parametrize("causal", [0, 1])
def test_equal_lengths_match_the_fixed_layout(causal):
    """A packed batch of equal lengths runs the same arithmetic as the
    fixed-length [B, H, N, d] call: O and lse agree bit for bit."""
    fa = _fa()
    B, H, N, d = 3, 4, 700, 128
    x = make_inputs(B, H, N, d, seed=760, with_grad_out=False)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    scale = d ** -0.5
    stream = torch.cuda.current_stream().cuda_stream
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    assert fa.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d, scale,
                     causal, fa.FA_BF16, stream) == fa.FA_OK
    pack = lambda t: t.transpose(1, 2).reshape(B * N, H, d).contiguous()  # noqa: E731
    xp = {"q": pack(q).cpu(), "k": pack(k).cpu(), "v": pack(v).cpu(),
          "cu_seqlens": torch.arange(B + 1, dtype=torch.int32) * N}
    o2, lse2, err = _fwd(xp, H, H, d, N, -1, 0 if causal else -1, scale)
    assert err == fa.FA_OK
    assert torch.equal(pack(o), o2)
    assert torch.equal(lse.transpose(0, 1).reshape(H, B * N), lse2)


def test_rows_outside_every_sequence_are_untouched():
    fa = _fa()
    H, Hkv, d = 2, 2, 64
    x = make_varlen_inputs([20, 50, 200, 10, 20], H, Hkv, d, seed=770)  # T = 300 finite rows
    x["cu_seqlens"] = torch.tensor([20, 70, 270, 280], dtype=torch.int32)  # rows 0-19, 280-299: no sequence
    o, lse, err = _fwd(x, H, Hkv, d, 200, -1, -1, d ** -0.5)
    assert err == fa.FA_OK
    assert o.shape[0] == 300
    assert torch.isnan(o[:20].float()).all() and torch.isnan(o[280:].float()).all()
    assert torch.isnan(lse[:, :20]).all() and torch.isnan(lse[:, 280:]).all()
    assert torch.isfinite(o[20:280].float()).all()


@pytest.mark.parametrize("bad", [[0, 50, 40, 280], [0, 100, 400], [-5, 100, 280], [0, 250, 280]])
def test_malformed_cu_seqlens_are_clamped_and_reported(bad):
    """Backwards, past-the-end, negative and longer-than-max_seqlen entries:
    the kernels clamp them (every access stays inside the buffers, which the
    guard bands check) and report FA_ERR_INVALID_ARG afterwards."""
    fa = _fa()
    H, Hkv, d = 2, 2, 64
    x = make_varlen_inputs([100, 180], H, Hkv, d, seed=780)
    x["cu_seqlens"] = torch.tensor(bad, dtype=torch.int32)
    o, lse, err = _fwd(x, H, Hkv, d, 200, -1, 0, d ** -0.5)
    assert err == fa.FA_ERR_INVALID_ARG
    x["do"] = x["q"].clone()
    _, _, _, err = _bwd(x, o.nan_to_num(0.0), lse.nan_to_num(0.0), H, Hkv, d, 200, -1, 0, d ** -0.5)
    assert err == fa.FA_ERR_INVALID_ARG
    assert fa.fa_get_device_error(torch.cuda.current_stream().cuda_stream) == fa.FA_OK


def test_varlen_long_and_short_sampled():
    """One 8192-token sequence beside short ones, causal: the short sequences
    in full, the long one on sampled rows (forward) and through dK/dV of its
    first head (backward)."""
    from oracle import attention_backward, attention_forward_rows, attention_forward_varlen

    lengths = [37, 8192, 300, 5]
    H, d = 2, 128
    x = make_varlen_inputs(lengths, H, H, d, seed=790)
    scale = d ** -0.5
    o, lse, _ = _fwd(x, H, H, d, 8192, -1, 0, scale)
    short = {"cu_seqlens": np.array([0, 37]), **{n: x[n][:37] for n in ("q", "k", "v")}}
    o_ref, lse_ref = attention_forward_varlen(short["q"], short["k"], short["v"], short["cu_seqlens"], scale, True)
    check_forward(to64(o[:37]), to64(lse[:, :37]), o_ref, lse_ref, float(x["v"].abs().max()), "short")
    a, e = 37, 37 + 8192
    seq = {n: x[n][a:e].transpose(0, 1)[None] for n in ("q", "k", "v", "do")}
    rows = np.unique(np.concatenate([np.arange(0, 200), np.arange(8000, 8192),
                                     np.random.default_rng(1).integers(0, 8192, 300)]))
    heads = [(0, h) for h in range(H)]
    o_ref, lse_ref = attention_forward_rows(seq["q"], seq["k"], seq["v"], scale, True, heads, rows)
    check_forward(to64(o[a:e][rows].transpose(0, 1)), to64(lse[:, a:e][:, rows]), o_ref, lse_ref,
                  float(x["v"].abs().max()), "long")
    dq, dk, dv, err = _bwd(x, o, lse, H, H, d, 8192, -1, 0, scale)
    assert err == _fa().FA_OK
    rq, rk, rv = attention_backward(seq["q"], seq["k"], seq["v"], seq["do"], scale, True, heads=[(0, 0)])
    check_grad(to64(dk[a:e, 0])[None], rk, "dK", "long")
    check_grad(to64(dv[a:e, 0])[None], rv, "dV", "long")
    check_grad(to64(dq[a:e, 0])[None], rq, "dQ", "long")
