"""GPU parity of grouped-query / multi-query attention (fa_fwd_gqa, fa_bwd_gqa)
against the fp64 oracle, through the C ABI.

Query head h reads K/V head h / (H / Hkv); dK and dV of a shared head are the
sums over its group. The oracle repeats K/V per group and sums the per-head
gradients back (grouped-query attention as the blog's related-article notes on
MQA/GQA describe it)."""

import pytest
import torch

from tests._parity import Guarded, check_forward, check_grad, to64
from workloads import make_inputs

pytestmark = pytest.mark.gpu


def _fa():
    import exact_attention_118_b200 as fa

    return fa


def _fwd(q, k, v, causal, scale):
    fa = _fa()
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    stream = torch.cuda.current_stream().cuda_stream
    o = Guarded((B, H, N, d), torch.bfloat16, q.device)
    lse = Guarded((B, H, N), torch.float32, q.device)
    st = fa.fa_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.t.data_ptr(), lse.t.data_ptr(), B, H, Hkv, N, d,
                       scale, int(causal), fa.FA_BF16, stream)
    assert st == fa.FA_OK, fa.fa_strerror(st)
    assert fa.fa_get_device_error(stream) == fa.FA_OK
    assert o.guards_intact() and lse.guards_intact(), "write outside O or lse"
    return o.t, lse.t


def _bwd(q, k, v, o, lse, do, causal, scale):
    fa = _fa()
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    stream = torch.cuda.current_stream().cuda_stream
    dq = Guarded((B, H, N, d), torch.bfloat16, q.device)
    dk = Guarded((B, Hkv, N, d), torch.bfloat16, q.device)
    dv = Guarded((B, Hkv, N, d), torch.bfloat16, q.device)
    ws_bytes = fa.fa_bwd_gqa_workspace_size(B, H, Hkv, N, d)
    ws = Guarded((ws_bytes,), torch.uint8, q.device, fill=0xFF)
    st = fa.fa_bwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                       dq.t.data_ptr(), dk.t.data_ptr(), dv.t.data_ptr(), ws.t.data_ptr(), ws_bytes,
                       B, H, Hkv, N, d, scale, int(causal), stream)
    assert st == fa.FA_OK, fa.fa_strerror(st)
    assert fa.fa_get_device_error(stream) == fa.FA_OK
    for g in (dq, dk, dv):
        assert g.guards_intact(), "write outside a gradient buffer"
    assert ws.guards_intact(), "write outside the workspace"
    return dq.t, dk.t, dv.t


CASES = [(2, 8, 2), (1, 4, 1), (1, 6, 3), (1, 3, 3)]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [200, 1000])
@pytest.mark.parametrize("B,H,Hkv", CASES)
def test_gqa_forward_backward(B, H, Hkv, N, causal, d):
    from oracle import attention_backward_gqa, attention_forward_gqa

    x = make_inputs(B, H, N, d, seed=400 + 7 * H + Hkv + N, kv_heads=Hkv)
    scale = d ** -0.5
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = _fwd(q, k, v, causal, scale)
    what = f"B{B} H{H} Hkv{Hkv} N{N} d{d} causal={causal}"
    o_ref, lse_ref = attention_forward_gqa(x["q"], x["k"], x["v"], scale, causal)
    check_forward(to64(o), to64(lse), o_ref, lse_ref, float(x["v"].abs().max()), what)
    dq, dk, dv = _bwd(q, k, v, o, lse, do, causal, scale)
    rq, rk, rv = attention_backward_gqa(x["q"], x["k"], x["v"], x["do"], scale, causal)
    check_grad(to64(dq), rq, "dQ", what)
    check_grad(to64(dk), rk, "dK", what)
    check_grad(to64(dv), rv, "dV", what)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_forward_equals_mha_on_repeated_kv(causal):
    """The forward reads K/V head h / g for query head h: with K/V repeated
    per group, fa_fwd runs the very same arithmetic, so O and lse agree bit
    for bit."""
    fa = _fa()
    B, H, Hkv, N, d = 2, 8, 2, 777, 128
    x = make_inputs(B, H, N, d, seed=77, with_grad_out=False, kv_heads=Hkv)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    scale = d ** -0.5
    o, lse = _fwd(q, k, v, causal, scale)
    kr = k.repeat_interleave(H // Hkv, dim=1).contiguous()
    vr = v.repeat_interleave(H // Hkv, dim=1).contiguous()
    o2 = torch.empty_like(q)
    lse2 = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    stream = torch.cuda.current_stream().cuda_stream
    assert fa.fa_fwd(q.data_ptr(), kr.data_ptr(), vr.data_ptr(), o2.data_ptr(), lse2.data_ptr(), B, H, N, d, scale,
                     int(causal), fa.FA_BF16, stream) == fa.FA_OK
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_mqa_long_sequence_sampled_rows():
    """Multi-query attention (Hkv = 1) at N = 4096, 16 query heads: the forward
    on sampled rows of every head, the backward's dK/dV in full against the
    group-summed oracle."""
    from oracle import attention_backward_gqa, attention_forward_gqa

    B, H, Hkv, N, d = 1, 16, 1, 4096, 128
    x = make_inputs(B, H, N, d, seed=91, kv_heads=Hkv)
    scale = d ** -0.5
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = _fwd(q, k, v, True, scale)
    o_ref, lse_ref = attention_forward_gqa(x["q"], x["k"], x["v"], scale, True)
    check_forward(to64(o), to64(lse), o_ref, lse_ref, float(x["v"].abs().max()), "MQA N4096")
    dq, dk, dv = _bwd(q, k, v, o, lse, do, True, scale)
    rq, rk, rv = attention_backward_gqa(x["q"], x["k"], x["v"], x["do"], scale, True)
    check_grad(to64(dq), rq, "dQ", "MQA N4096")
    check_grad(to64(dk), rk, "dK", "MQA N4096")
    check_grad(to64(dv), rv, "dV", "MQA N4096")


@pytest.mark.parametrize("B,H,Hkv,N", [(4, 32, 8, 4096), (4, 16, 8, 8192)])
def test_gqa_backward_large_grid_sampled_groups(B, H, Hkv, N):
    """Grids large enough that a CTA covers more than one query head of its
    K/V head (no split, or a split into fewer shares than the group size).
    Checked on whole groups: the oracle runs one K/V head and its query heads,
    for the first and the last group of the first and the last batch."""
    from oracle import attention_backward_gqa

    d, causal = 64, True
    x = make_inputs(B, H, N, d, seed=500 + H, kv_heads=Hkv)
    scale = d ** -0.5
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = _fwd(q, k, v, causal, scale)
    dq, dk, dv = _bwd(q, k, v, o, lse, do, causal, scale)
    g = H // Hkv
    for b, kv in ((0, 0), (B - 1, Hkv - 1)):
        hs = slice(kv * g, (kv + 1) * g)
        sub = {n: x[n][b:b + 1, hs if n in ("q", "do") else slice(kv, kv + 1)] for n in ("q", "k", "v", "do")}
        rq, rk, rv = attention_backward_gqa(sub["q"], sub["k"], sub["v"], sub["do"], scale, causal)
        what = f"B{B} H{H} Hkv{Hkv} N{N} batch {b} kv head {kv}"
        check_grad(to64(dq[b:b + 1, hs]), rq, "dQ", what)
        check_grad(to64(dk[b:b + 1, kv:kv + 1]), rk, "dK", what)
        check_grad(to64(dv[b:b + 1, kv:kv + 1]), rv, "dV", what)
