"""The seeded input generators shared by the oracle and the GPU tests: fixed
shapes, dtypes and determinism, and the recipes they promise (bf16 rounding,
packed prefix sums, e4m3 codes whose largest magnitude maps to the tensor's
largest value)."""

import numpy as np
import torch

from workloads import WORKLOADS, make_fp8_inputs, make_inputs, make_varlen_inputs, make_workload_inputs


def test_make_inputs_is_deterministic_and_bf16():
    a = make_inputs(2, 3, 17, 64, seed=5)
    b = make_inputs(2, 3, 17, 64, seed=5)
    c = make_inputs(2, 3, 17, 64, seed=6)
    for n in ("q", "k", "v", "do"):
        assert a[n].dtype == torch.bfloat16 and tuple(a[n].shape) == (2, 3, 17, 64)
        assert torch.equal(a[n], b[n])
        assert not torch.equal(a[n], c[n])


def test_kv_heads_shapes_and_unchanged_default_stream():
    x = make_inputs(1, 8, 33, 128, seed=9, kv_heads=2)
    assert tuple(x["q"].shape) == (1, 8, 33, 128) and tuple(x["do"].shape) == (1, 8, 33, 128)
    assert tuple(x["k"].shape) == (1, 2, 33, 128) and tuple(x["v"].shape) == (1, 2, 33, 128)
    # kv_heads = H draws exactly what the default does.
    y, z = make_inputs(1, 4, 20, 64, seed=3, kv_heads=4), make_inputs(1, 4, 20, 64, seed=3)
    for n in ("q", "k", "v", "do"):
        assert torch.equal(y[n], z[n])


def test_qk_std_scales_only_q_and_k():
    a = make_inputs(1, 2, 64, 64, seed=4)
    b = make_inputs(1, 2, 64, 64, seed=4, qk_std=3.0)
    for n in ("q", "k"):
        assert torch.allclose(b[n].float(), (a[n].float() * 3.0).to(torch.bfloat16).float(), rtol=1e-2, atol=0)
    assert torch.equal(a["v"], b["v"]) and torch.equal(a["do"], b["do"])


def test_workload_table_matches_its_names():
    for name, w in WORKLOADS.items():
        assert f"n{w.N}" in name and f"d{w.d}" in name and f"h{w.H}" in name
        assert ("causal" in name) == bool(w.causal)
    x = make_workload_inputs(WORKLOADS["fwd_b1h2_n256_d64"])
    assert "do" not in x and tuple(x["q"].shape) == (1, 2, 256, 64)


def test_varlen_inputs_prefix_sums_and_shapes():
    lengths = [5, 0, 17, 1]
    x = make_varlen_inputs(lengths, 4, 2, 64, seed=1)
    assert x["cu_seqlens"].dtype == torch.int32
    assert x["cu_seqlens"].tolist() == [0, 5, 5, 22, 23]
    T = sum(lengths)
    assert tuple(x["q"].shape) == (T, 4, 64) and tuple(x["k"].shape) == (T, 2, 64)
    assert all(x[n].dtype == torch.bfloat16 for n in ("q", "k", "v", "do"))


def test_fp8_inputs_codes_and_scales():
    from oracle import e4m3_decode

    x = make_fp8_inputs(1, 2, 50, 128, seed=2, kv_heads=1)
    assert x["q8"].dtype == torch.uint8 and tuple(x["k8"].shape) == (1, 1, 50, 128)
    for n in ("q", "k", "v"):
        vals = e4m3_decode(x[n + "8"].numpy())
        assert np.all(np.isfinite(vals))
        # the largest magnitude maps to the largest finite code, 448
        assert np.max(np.abs(vals)) == 448.0
        assert x[n + "_scale"] > 0
