"""GPU parity of fa_fwd against the fp64 oracle, through the C ABI."""

import math

import numpy as np
import pytest
import torch

from tests._parity import Guarded, check_forward, to64
from workloads import WORKLOADS, make_inputs, make_workload_inputs

pytestmark = pytest.mark.gpu


def _fa():
    import exact_attention_118_b200 as fa

    return fa


def _run_fwd(q, k, v, causal, out_fp32=False, scale=None):
    fa = _fa()
    B, H, N, d = q.shape
    scale = d ** -0.5 if scale is None else scale
    o = Guarded((B, H, N, d), torch.float32 if out_fp32 else torch.bfloat16, q.device)
    lse = Guarded((B, H, N), torch.float32, q.device)
    st = fa.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.t.data_ptr(), lse.t.data_ptr(), B, H, N, d,
                   scale, int(causal), fa.FA_F32 if out_fp32 else fa.FA_BF16,
                   torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_OK, fa.fa_strerror(st)
    assert fa.fa_get_device_error(torch.cuda.current_stream().cuda_stream) == fa.FA_OK
    assert o.guards_intact() and lse.guards_intact(), "write outside the output buffers"
    return o.t, lse.t


def _full_case(B, H, N, d, causal, seed, out_fp32=False, qk_std=1.0):
    from oracle import attention_forward

    x = make_inputs(B, H, N, d, seed, qk_std, with_grad_out=False)
    qc, kc, vc = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = _run_fwd(qc, kc, vc, causal, out_fp32)
    o_ref, lse_ref = attention_forward(x["q"], x["k"], x["v"], d ** -0.5, causal)
    vmax = float(x["v"].abs().max())
    return check_forward(to64(o), to64(lse), o_ref, lse_ref, vmax, f"B{B} H{H} N{N} d{d} causal={causal}")


def test_fwd_workload_fwd_b1h2_n256_d64_fp32_out():
    w = WORKLOADS["fwd_b1h2_n256_d64"]
    _full_case(w.B, w.H, w.N, w.d, w.causal, w.seed, out_fp32=True)


def test_fwd_workload_causal_b2h8_n1024_d64():
    w = WORKLOADS["causal_b2h8_n1024_d64"]
    _full_case(w.B, w.H, w.N, w.d, w.causal, w.seed)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 127, 128, 129, 200, 255, 256, 257, 383, 1000])
def test_fwd_ragged(N, causal, d):
    _full_case(1, 2, N, d, causal, seed=100 + N)


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_multi_batch_head_d128(causal):
    _full_case(3, 5, 700, 128, causal, seed=7)


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_large_logits_rescale_path(causal):
    # std-3 Q and K: logits with a wide range force running-max updates.
    _full_case(1, 2, 1500, 128, causal, seed=11, qk_std=3.0)


def test_fwd_fp32_output_d128():
    _full_case(2, 2, 300, 128, True, seed=12, out_fp32=True)


def _sampled_case(w, heads, n_rows=48, seed=0):
    """Full-size launch; oracle on sampled (head, row) outputs."""
    from oracle import attention_forward_rows

    x = make_workload_inputs(w, with_grad_out=False)
    qc, kc, vc = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = _run_fwd(qc, kc, vc, w.causal)
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 255, 256, w.N - 129, w.N - 1],
                                     rng.integers(0, w.N, n_rows)]))
    o_ref, lse_ref = attention_forward_rows(x["q"], x["k"], x["v"], w.scale, w.causal, heads, rows)
    vmax = float(x["v"].abs().max())
    for t, (b, h) in enumerate(heads):
        check_forward(to64(o[b, h][rows]), to64(lse[b, h][rows]), o_ref[t], lse_ref[t], vmax,
                      f"{w.name} head ({b},{h})")
    # every output everywhere finite and lse bounded below by the diagonal logit
    assert torch.isfinite(o).all().item() and torch.isfinite(lse).all().item()


def test_fwd_workload_b4h16_n4096_d128():
    w = WORKLOADS["b4h16_n4096_d128"]
    _sampled_case(w, heads=[(0, 0), (1, 7), (3, 15)], n_rows=128)


def test_fwd_workload_b1h16_n16384_d128():
    w = WORKLOADS["b1h16_n16384_d128"]
    _sampled_case(w, heads=[(0, 0), (0, 9), (0, 15)])


def test_fwd_workload_causal_b1h16_n16384_d128():
    w = WORKLOADS["causal_b1h16_n16384_d128"]
    _sampled_case(w, heads=[(0, 0), (0, 9), (0, 15)])


def test_fwd_workload_causal_b1h32_n32768_d128_qk3():
    w = WORKLOADS["causal_b1h32_n32768_d128_qk3"]
    _sampled_case(w, heads=[(0, 0), (0, 31)], n_rows=32)


def test_fwd_repeat_is_deterministic():
    x = make_inputs(1, 4, 1000, 128, 5, with_grad_out=False)
    qc, kc, vc = (x[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = _run_fwd(qc, kc, vc, True)
    o2, l2 = _run_fwd(qc, kc, vc, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fwd_non_default_scale():
    from oracle import attention_forward

    x = make_inputs(1, 2, 300, 64, 21, with_grad_out=False)
    qc, kc, vc = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = _run_fwd(qc, kc, vc, True, scale=0.37)
    o_ref, lse_ref = attention_forward(x["q"], x["k"], x["v"], 0.37, True)
    check_forward(to64(o), to64(lse), o_ref, lse_ref, float(x["v"].abs().max()), "scale 0.37")


def test_fwd_torch_convenience_wrapper():
    fa = _fa()
    x = make_inputs(1, 2, 130, 64, 22, with_grad_out=False)
    qc, kc, vc = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa.attention_forward(qc, kc, vc, causal=True)
    o2, lse2 = _run_fwd(qc, kc, vc, True)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert math.isfinite(float(lse.sum()))
