"""fa_bwd_noalloc: the backward for callers that may not allocate device memory.

Some callers cannot call cudaMalloc: code running inside a host application
that owns every GPU allocation (a plug-in that is handed only its tensors), or
a latency-critical path where an allocation's unpredictable cost is not
allowed. fa_bwd_noalloc serves them by keeping the backward's scratch in one
fixed device array inside the library instead of a caller-owned workspace.

This test calls it through the C ABI twice in a row, on different problems.
It runs the same kernels as fa_bwd (the entry point with a caller-owned
workspace), so dK and dV must equal fa_bwd's bit for bit; dQ is summed with
fp32 adds whose order may differ between runs, so it is checked against the
fp64 oracle within the gradient tolerance the parity tests use. The second
call would show a dQ accumulator left over from the first one. The file is
named so pytest collects it last.
"""

import pytest
import torch

from tests._parity import check_grad, to64
from workloads import make_inputs

pytestmark = pytest.mark.gpu


def _both(B, H, N, d, causal, seed):
    import exact_attention_118_b200 as fa

    x = make_inputs(B, H, N, d, seed)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    scale = d ** -0.5
    stream = torch.cuda.current_stream().cuda_stream
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    assert fa.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d, scale,
                     int(causal), fa.FA_BF16, stream) == fa.FA_OK
    ref = [torch.full_like(q, float("nan")) for _ in range(3)]
    ws_bytes = fa.fa_bwd_workspace_size(B, H, N, d)
    assert ws_bytes <= fa.FA_NOALLOC_SCRATCH_BYTES
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    assert fa.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                     ref[0].data_ptr(), ref[1].data_ptr(), ref[2].data_ptr(), ws.data_ptr(), ws_bytes, B, H, N, d,
                     scale, int(causal), stream) == fa.FA_OK
    got = [torch.full_like(q, float("nan")) for _ in range(3)]
    st = fa.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                           do.data_ptr(), got[0].data_ptr(), got[1].data_ptr(), got[2].data_ptr(), B, H, N, d,
                           scale, int(causal), stream)
    assert st == fa.FA_OK, fa.fa_strerror(st)
    assert fa.fa_get_device_error(stream) == fa.FA_OK
    assert torch.equal(got[1], ref[1]), "dK differs from fa_bwd"
    assert torch.equal(got[2], ref[2]), "dV differs from fa_bwd"
    from oracle import attention_backward

    rq, _, _ = attention_backward(x["q"], x["k"], x["v"], x["do"], scale, causal)
    check_grad(to64(got[0]), rq, "dQ", f"noalloc B{B} H{H} N{N} d{d} causal={causal}")


def test_noalloc_matches_fa_bwd_on_two_calls_in_a_row():
    _both(1, 4, 1000, 128, True, seed=301)
    _both(2, 2, 777, 64, False, seed=302)
