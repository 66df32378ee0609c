"""GPU parity of fa_bwd (dQ, dK, dV) against the fp64 oracle, through the C ABI.

The GPU backward consumes the GPU forward's bf16 O and fp32 lse, as a caller
would; the oracle recomputes everything in fp64 from the same bf16 inputs."""

import numpy as np
import pytest
import torch

from tests._parity import Guarded, check_grad, single_key_zero_bound, to64
from workloads import WORKLOADS, make_inputs, make_workload_inputs

pytestmark = pytest.mark.gpu


def _fa():
    import exact_attention_118_b200 as fa

    return fa


def _run(x, causal, scale=None):
    fa = _fa()
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    B, H, N, d = q.shape
    scale = d ** -0.5 if scale is None else scale
    stream = torch.cuda.current_stream().cuda_stream
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    assert fa.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d, scale,
                     int(causal), fa.FA_BF16, stream) == fa.FA_OK
    grads = [Guarded((B, H, N, d), torch.bfloat16, q.device) for _ in range(3)]
    ws_bytes = fa.fa_bwd_workspace_size(B, H, N, d)
    ws = Guarded((ws_bytes,), torch.uint8, q.device, fill=0xFF)
    st = fa.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                   grads[0].t.data_ptr(), grads[1].t.data_ptr(), grads[2].t.data_ptr(), ws.t.data_ptr(), ws_bytes,
                   B, H, N, d, scale, int(causal), stream)
    assert st == fa.FA_OK, fa.fa_strerror(st)
    assert fa.fa_get_device_error(stream) == fa.FA_OK
    for g in grads:
        assert g.guards_intact(), "write outside a gradient buffer"
    assert ws.guards_intact(), "write outside the workspace"
    return [g.t for g in grads]


def _full_case(B, H, N, d, causal, seed, qk_std=1.0, scale=None):
    from oracle import attention_backward

    x = make_inputs(B, H, N, d, seed, qk_std)
    dq, dk, dv = _run(x, causal, scale)
    scale = d ** -0.5 if scale is None else scale
    rq, rk, rv = attention_backward(x["q"], x["k"], x["v"], x["do"], scale, causal)
    what = f"B{B} H{H} N{N} d{d} causal={causal}"
    zb = single_key_zero_bound(x, scale) if N == 1 else 0.0
    if N == 1:
        assert np.all(rq == 0) and np.all(rk == 0)
    return (check_grad(to64(dq), rq, "dQ", what, zb), check_grad(to64(dk), rk, "dK", what, zb),
            check_grad(to64(dv), rv, "dV", what))


def test_bwd_workload_causal_b2h8_n1024_d64():
    w = WORKLOADS["causal_b2h8_n1024_d64"]
    _full_case(w.B, w.H, w.N, w.d, w.causal, w.seed)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 64, 65, 127, 128, 129, 200, 255, 256, 257, 383, 1000])
def test_bwd_ragged(N, causal, d):
    _full_case(1, 2, N, d, causal, seed=200 + N)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_multi_batch_head_d128(causal):
    _full_case(2, 3, 700, 128, causal, seed=8)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_large_logits(causal):
    _full_case(1, 2, 1100, 128, causal, seed=13, qk_std=3.0)


def test_bwd_non_default_scale():
    _full_case(1, 2, 300, 64, True, seed=14, scale=0.3)


def _sampled_heads(w, heads):
    from oracle import attention_backward

    x = make_workload_inputs(w)
    dq, dk, dv = _run(x, w.causal)
    rq, rk, rv = attention_backward(x["q"], x["k"], x["v"], x["do"], w.scale, w.causal, heads=heads)
    for t, (b, h) in enumerate(heads):
        what = f"{w.name} head ({b},{h})"
        check_grad(to64(dq[b, h]), rq[t], "dQ", what)
        check_grad(to64(dk[b, h]), rk[t], "dK", what)
        check_grad(to64(dv[b, h]), rv[t], "dV", what)
    for g in (dq, dk, dv):
        assert torch.isfinite(g).all().item()


def test_bwd_workload_b4h16_n4096_d128():
    _sampled_heads(WORKLOADS["b4h16_n4096_d128"], [(0, 0), (2, 5), (3, 15)])


# First, middle and last head: the causal launch order and the grouping of
# heads map heads to CTAs differently, so each end of the order is checked.
def test_bwd_workload_b1h16_n16384_d128():
    _sampled_heads(WORKLOADS["b1h16_n16384_d128"], [(0, 0), (0, 7), (0, 15)])


def test_bwd_workload_causal_b1h16_n16384_d128():
    _sampled_heads(WORKLOADS["causal_b1h16_n16384_d128"], [(0, 0), (0, 8), (0, 15)])


def test_bwd_workload_causal_b1h32_n32768_d128_qk3():
    _sampled_heads(WORKLOADS["causal_b1h32_n32768_d128_qk3"], [(0, 0), (0, 16), (0, 31)])


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_odd_tile_count_n16383(causal):
    # ceil(16383 / 128) = 128 key and query tiles with a ragged last one, at
    # the headline length: full oracle comparison of one head.
    _full_case(1, 1, 16383, 128, causal, seed=16383)


def test_bwd_repeat_is_deterministic_up_to_reduction_order():
    # dQ is accumulated with fp32 adds whose order may vary between runs; dK and
    # dV are accumulated in a fixed order on chip and must match bit for bit.
    x = make_inputs(1, 2, 700, 128, 15)
    a = _run(x, True)
    b = _run(x, True)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert float((a[0].float() - b[0].float()).abs().max()) <= 1e-2 * float(a[0].float().abs().max())


def test_bwd_torch_convenience_wrapper():
    fa = _fa()
    x = make_inputs(1, 2, 300, 128, 16)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=True)
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, causal=True)
    ref = _run(x, True)
    assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])
    assert np.isfinite(to64(dq)).all()
