"""Failure detection on the GPU without a GPU fault.

Every device-side wait in the kernels is bounded; when one gives up it records
a timeout in a device error word and the kernel exits normally. This test makes
such a wait run out on purpose (a barrier that nothing completes, through the
library's own bounded wait), checks that the host reads FA_ERR_TIMEOUT, that the
word is cleared by reading it, and that the context still runs attention
correctly afterwards."""

import pytest
import torch

from tests._parity import check_forward, to64
from workloads import make_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import exact_attention_118_b200 as fa
    from oracle import attention_forward

    stream = torch.cuda.current_stream().cuda_stream
    assert fa.fa_get_device_error(stream) == fa.FA_OK
    assert fa.fa_selftest_wait_timeout(stream) == fa.FA_OK
    assert fa.fa_get_device_error(stream) == fa.FA_ERR_TIMEOUT
    assert fa.fa_get_device_error(stream) == fa.FA_OK  # reading clears it

    x = make_inputs(1, 2, 300, 128, seed=77, with_grad_out=False)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa.attention_forward(q, k, v, causal=True)
    fa.check_device_error()
    o_ref, lse_ref = attention_forward(x["q"], x["k"], x["v"], 128 ** -0.5, True)
    check_forward(to64(o), to64(lse), o_ref, lse_ref, float(x["v"].abs().max()), "after timeout")
