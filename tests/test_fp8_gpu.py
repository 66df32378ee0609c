"""GPU parity of the FP8 (e4m3) forward, fa_fwd_fp8, against the fp64 oracle
(exact attention of the dequantised inputs), through the C ABI.

Tolerance, derived from the kernel's one rounding that the bf16 path does not
have: P is rounded to e4m3 before it multiplies V. For row i let
q_j = 2^(lambda s_ij - M_i) over the visible keys (M_i the row's true maximum,
so q_j <= 1). The kernel's p_j = c q_j with c = 2^(M_i - m_i) in [1, 2^8]
(m_i its running maximum), and e4m3 rounding gives |p~_j - p_j| <= 2^-4 p_j
(3 mantissa bits) or, below 2^-6, <= 2^-10 (half the subnormal spacing). The
row sum l = sum p_j is kept unrounded, so
  |O_i - O_ref_i| <= (2^-4 sum_j q_j |v_j| + 2^-10 sum_j |v_j|) / sum_j q_j,
per column, plus fp32 accumulation (negligible) and the rounding of O to bf16
(2^-9 relative, taken as 2^-8). lse comes from the unrounded sums: the bf16
path's 1e-3 bound holds."""

import numpy as np
import pytest
import torch

from tests._parity import LSE_TOL, Guarded, to64
from workloads import make_fp8_inputs

pytestmark = pytest.mark.gpu


def _fa():
    import exact_attention_118_b200 as fa

    return fa


def _row_bounds(x, scale, causal, window):
    """Per-row, per-column error bound of the module docstring, [B, H, N, d]."""
    from oracle import band_visible, causal_visible, e4m3_decode

    q = e4m3_decode(x["q8"].numpy()) * x["q_scale"]
    k = e4m3_decode(x["k8"].numpy()) * x["k_scale"]
    v = e4m3_decode(x["v8"].numpy()) * x["v_scale"]
    B, H, N, d = q.shape
    g = H // k.shape[1]
    bound = np.empty((B, H, N, d))
    rows = np.arange(N)
    vis = np.ones((N, N), dtype=bool)
    if causal:
        vis &= causal_visible(rows, N)
    if window is not None:
        vis &= band_visible(rows, N, *window)
    for b in range(B):
        for h in range(H):
            s = scale * (q[b, h] @ k[b, h // g].T)
            s = np.where(vis, s, -np.inf)
            qq = np.exp2((s - s.max(axis=1, keepdims=True)) / np.log(2.0))
            av = np.abs(v[b, h // g])
            bound[b, h] = (2.0 ** -4 * (qq @ av) + 2.0 ** -10 * (vis @ av)) / qq.sum(axis=1, keepdims=True)
    return bound


def _run(x, B, H, Hkv, N, causal, window, o_fp32):
    fa = _fa()
    d = 128
    scale = d ** -0.5
    q8, k8, v8 = (x[n].cuda() for n in ("q8", "k8", "v8"))
    stream = torch.cuda.current_stream().cuda_stream
    o = Guarded((B, H, N, d), torch.float32 if o_fp32 else torch.bfloat16, q8.device)
    lse = Guarded((B, H, N), torch.float32, q8.device)
    wl, wr = window if window is not None else (-1, 0 if causal else -1)
    if causal and window is not None:
        wr = 0
    st = fa.fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), o.t.data_ptr(), lse.t.data_ptr(), B, H, Hkv, N,
                       d, scale, x["q_scale"], x["k_scale"], x["v_scale"], wl, wr,
                       fa.FA_F32 if o_fp32 else fa.FA_BF16, stream)
    assert st == fa.FA_OK, fa.fa_strerror(st)
    assert fa.fa_get_device_error(stream) == fa.FA_OK
    assert o.guards_intact() and lse.guards_intact(), "write outside O or lse"
    return o.t, lse.t


def _case(B, H, Hkv, N, causal, window, seed, o_fp32=False):
    from oracle import attention_forward_fp8

    x = make_fp8_inputs(B, H, N, 128, seed, kv_heads=Hkv)
    scale = 128 ** -0.5
    o, lse = _run(x, B, H, Hkv, N, causal, window, o_fp32)
    o_ref, lse_ref = attention_forward_fp8(x["q8"], x["k8"], x["v8"], x["q_scale"], x["k_scale"], x["v_scale"],
                                           scale, causal, window)
    bound = _row_bounds(x, scale, causal, window)
    og, lg = to64(o), to64(lse)
    what = f"B{B} H{H} Hkv{Hkv} N{N} causal={causal} window={window}"
    assert np.all(np.isfinite(og)) and np.all(np.isfinite(lg)), what
    err = np.abs(og - o_ref)
    slack = 2.0 ** -8 * np.abs(o_ref) + 1e-5 * float(np.max(np.abs(o_ref)))
    worst = float(np.max(err / (1.01 * bound + slack)))
    assert worst <= 1.0, f"{what}: |O err| exceeds the e4m3 bound by {worst:.3f}x"
    assert float(np.max(np.abs(lg - lse_ref))) <= LSE_TOL, what
    return float(np.max(err)), float(np.max(bound))


@pytest.mark.parametrize("N", [200, 1000])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_forward(N, causal):
    _case(1, 2, 2, N, causal, None, seed=800 + N + causal)


def test_fp8_forward_grouped_heads_fp32_out():
    _case(2, 4, 2, 777, True, None, seed=810, o_fp32=True)


@pytest.mark.parametrize("window", [(100, 0), (64, 64)])
def test_fp8_forward_window(window):
    _case(1, 2, 2, 700, False, window, seed=820 + window[1])


@pytest.mark.parametrize("N", [1, 17, 129])
def test_fp8_forward_tiny(N):
    _case(1, 2, 1, N, True, None, seed=830 + N)


def test_fp8_error_is_well_inside_its_bound():
    """The bound is a worst case; the measured error should sit well under it
    (a kernel that used the wrong scale or dropped a tile would not)."""
    err, bound = _case(1, 4, 4, 2048, False, None, seed=840)
    assert err < 0.5 * bound
