"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/fa.h declares, and rejects bad arguments before it
touches the device."""

import ctypes

import pytest

import exact_attention_118_b200 as fa

FAKE = 1 << 20  # an aligned, non-null address that is never dereferenced


def test_library_loads_and_exports_every_header_symbol():
    names = fa.header_symbols()
    assert set(names) == {"fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_bwd_noalloc", "fa_get_device_error",
                          "fa_decode_device_error",
                          "fa_fwd_gqa", "fa_bwd_gqa", "fa_bwd_gqa_workspace_size",
                          "fa_fwd_window", "fa_bwd_window", "fa_fwd_varlen", "fa_bwd_varlen",
                          "fa_bwd_varlen_workspace_size", "fa_fwd_fp8",
                          "fa_set_bwd_main_events", "fa_last_cuda_error", "fa_selftest_wait_timeout",
                          "fa_selftest_exp2_fma",
                          "fa_strerror", "fa_version"}
    lib = ctypes.CDLL(fa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_strerror_and_version():
    assert fa.fa_strerror(fa.FA_OK) == "success"
    for s in range(1, 5):
        assert fa.fa_strerror(s) and fa.fa_strerror(s) != "success"
    assert fa.fa_strerror(99) == "unknown status"
    assert fa.fa_version() >= 100


@pytest.mark.parametrize("word", range(16))
def test_device_error_word_decoding(word):
    # Every combination of the three defined bits and one undefined bit (8):
    # a timeout wins; then a misaligned shared-memory window or an unknown
    # bit (a broken launch environment, nothing computed) is a CUDA error;
    # malformed cu_seqlens alone is the caller's argument error.
    got = fa.fa_decode_device_error(word)
    if word == 0:
        want = fa.FA_OK
    elif word & fa.FA_DEVERR_TIMEOUT:
        want = fa.FA_ERR_TIMEOUT
    elif word & (fa.FA_DEVERR_SMEM_ALIGN | 8):
        want = fa.FA_ERR_CUDA
    else:
        assert word == fa.FA_DEVERR_SEQLENS
        want = fa.FA_ERR_INVALID_ARG
    assert got == want, (word, got, want)
    assert fa.fa_decode_device_error(0x80000000 | fa.FA_DEVERR_SEQLENS) == fa.FA_ERR_CUDA


def test_device_error_bits_match_header():
    import re

    with open(fa.HEADER_PATH) as f:
        text = f.read()
    bits = {m.group(1): int(m.group(2)) for m in re.finditer(r"#define (FA_DEVERR_\w+) (\d+)u", text)}
    assert bits == {"FA_DEVERR_TIMEOUT": fa.FA_DEVERR_TIMEOUT, "FA_DEVERR_SMEM_ALIGN": fa.FA_DEVERR_SMEM_ALIGN,
                    "FA_DEVERR_SEQLENS": fa.FA_DEVERR_SEQLENS}


def test_workspace_size():
    B, H, N, d = 2, 3, 1000, 128
    rows = B * H * N
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    np_ = (N + 3) // 4 * 4
    assert fa.fa_bwd_workspace_size(B, H, N, d) == up(rows * d * 4) + 2 * up(B * H * np_ * 4)
    assert fa.fa_bwd_workspace_size(1, 1, 17, 64) == up(17 * 64 * 4) + 2 * up(20 * 4)
    assert fa.fa_bwd_workspace_size(0, 1, 1, 64) == 0
    assert fa.fa_bwd_workspace_size(1, 1, 1, 96) == 0


def _fwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, H=1, N=16, d=64, scale=0.125, causal=0,
             o_dtype=fa.FA_BF16, stream=None)
    a.update(kw)
    return fa.fa_fwd(*a.values())


@pytest.mark.parametrize("kw,want", [
    (dict(q=None), fa.FA_ERR_INVALID_ARG),
    (dict(k=FAKE + 8), fa.FA_ERR_INVALID_ARG),
    (dict(lse=FAKE + 4), fa.FA_ERR_INVALID_ARG),
    (dict(N=0), fa.FA_ERR_INVALID_ARG),
    (dict(B=-1), fa.FA_ERR_INVALID_ARG),
    (dict(H=0), fa.FA_ERR_INVALID_ARG),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(d=256), fa.FA_ERR_UNSUPPORTED),
    (dict(d=0), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(scale=-1.0), fa.FA_ERR_INVALID_ARG),
    (dict(causal=2), fa.FA_ERR_INVALID_ARG),
    (dict(o_dtype=7), fa.FA_ERR_INVALID_ARG),
    (dict(B=1 << 16, H=1 << 10, N=1 << 10), fa.FA_ERR_INVALID_ARG),
])
def test_fwd_rejects_bad_arguments_without_launching(kw, want):
    assert _fwd(**kw) == want


def _bwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, dO=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, ws=FAKE,
             ws_bytes=1 << 30, B=1, H=1, N=16, d=64, scale=0.125, causal=1, stream=None)
    a.update(kw)
    return fa.fa_bwd(*a.values())


@pytest.mark.parametrize("kw,want", [
    (dict(dO=None), fa.FA_ERR_INVALID_ARG),
    (dict(dq=FAKE + 2), fa.FA_ERR_INVALID_ARG),
    (dict(ws=None), fa.FA_ERR_INVALID_ARG),
    (dict(ws=FAKE + 16), fa.FA_ERR_INVALID_ARG),
    (dict(ws_bytes=100), fa.FA_ERR_INVALID_ARG),
    (dict(N=-5), fa.FA_ERR_INVALID_ARG),
    (dict(d=32), fa.FA_ERR_UNSUPPORTED),
    (dict(scale=float("inf")), fa.FA_ERR_INVALID_ARG),
    (dict(causal=-1), fa.FA_ERR_INVALID_ARG),
])
def test_bwd_rejects_bad_arguments_without_launching(kw, want):
    assert _bwd(**kw) == want


def test_product_path_does_not_import_oracle():
    import os
    import re

    pkg = os.path.dirname(fa.__file__)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(root, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", text, re.M), f


def test_set_bwd_main_events_is_host_only():
    assert fa.fa_set_bwd_main_events(None, None) == fa.FA_OK


def test_last_cuda_error_starts_clear():
    assert fa.fa_last_cuda_error() == 0


def test_noalloc_rejects_problems_beyond_its_fixed_scratch():
    # 32 heads x 16384 rows x d=128 needs ~269 MB of scratch: more than the array holds.
    assert fa.fa_bwd_workspace_size(1, 32, 16384, 128) > fa.FA_NOALLOC_SCRATCH_BYTES
    st = fa.fa_bwd_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 32, 16384, 128, 0.088, 1, None)
    assert st == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_bwd_noalloc(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 64, 64, 0.1, 0,
                             None) == fa.FA_ERR_INVALID_ARG


def test_noalloc_scratch_size_matches_header():
    import re

    with open(fa.HEADER_PATH) as f:
        m = re.search(r"#define FA_NOALLOC_SCRATCH_BYTES \((\d+)u \* 1024u \* 1024u\)", f.read())
    assert m and int(m.group(1)) * 1024 * 1024 == fa.FA_NOALLOC_SCRATCH_BYTES


@pytest.mark.parametrize("H,Hkv", [(8, 3), (4, 0), (4, -2), (2, 4)])
def test_gqa_rejects_bad_head_counts(H, Hkv):
    assert fa.fa_fwd_gqa(FAKE, FAKE, FAKE, FAKE, FAKE, 1, H, Hkv, 16, 64, 0.1, 0, fa.FA_BF16,
                         None) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_bwd_gqa(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, 1, H, Hkv, 16, 64,
                         0.1, 0, None) == fa.FA_ERR_INVALID_ARG


def test_gqa_workspace_size_formula():
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    for B, H, Hkv, N, d in ((1, 16, 16, 1000, 128), (2, 8, 2, 777, 64), (1, 16, 1, 16384, 128)):
        base = fa.fa_bwd_workspace_size(B, H, N, d)
        extra = 0 if Hkv == H else 2 * up(B * Hkv * N * d * 4)
        assert fa.fa_bwd_gqa_workspace_size(B, H, Hkv, N, d) == base + extra
    assert fa.fa_bwd_gqa_workspace_size(1, 8, 3, 64, 64) == 0
    assert fa.fa_bwd_gqa_workspace_size(1, 8, 0, 64, 64) == 0


def test_gqa_bwd_rejects_small_workspace():
    need = fa.fa_bwd_gqa_workspace_size(1, 8, 2, 256, 64)
    assert need > fa.fa_bwd_workspace_size(1, 8, 256, 64)
    assert fa.fa_bwd_gqa(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need - 1, 1, 8, 2, 256, 64,
                         0.1, 0, None) == fa.FA_ERR_INVALID_ARG


def test_window_calls_reject_bad_arguments():
    # bad head grouping, bad head dim, null pointer, small workspace
    assert fa.fa_fwd_window(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 3, 64, 64, 0.1, 4, 0, fa.FA_BF16,
                            None) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_fwd_window(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 2, 64, 96, 0.1, 4, 0, fa.FA_BF16,
                            None) == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_fwd_window(None, FAKE, FAKE, FAKE, FAKE, 1, 8, 2, 64, 64, 0.1, 4, 0, fa.FA_BF16,
                            None) == fa.FA_ERR_INVALID_ARG
    need = fa.fa_bwd_gqa_workspace_size(1, 8, 2, 256, 64)
    assert fa.fa_bwd_window(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need - 1, 1, 8, 2, 256, 64,
                            0.1, 16, 16, None) == fa.FA_ERR_INVALID_ARG


def test_varlen_workspace_size_formula():
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    for B, T, H, Hkv, d in ((3, 1000, 8, 8, 64), (7, 4097, 16, 4, 128)):
        S = (T + 4 * B + 4 + 3) // 4 * 4
        want = up(T * H * d * 4) + 2 * up(H * S * 4) + (2 * up(T * Hkv * d * 4) if Hkv < H else 0)
        assert fa.fa_bwd_varlen_workspace_size(B, T, H, Hkv, d) == want
    assert fa.fa_bwd_varlen_workspace_size(2, 100, 8, 3, 64) == 0
    assert fa.fa_bwd_varlen_workspace_size(0, 100, 8, 8, 64) == 0


def test_varlen_calls_reject_bad_arguments():
    ok = dict(B=2, max_seqlen=64, T=100, H=4, Hkv=2, d=64)

    def fwd(cu=FAKE, **kw):
        a = {**ok, **kw}
        return fa.fa_fwd_varlen(FAKE, FAKE, FAKE, FAKE, FAKE, cu, a["B"], a["max_seqlen"], a["T"], a["H"], a["Hkv"],
                                a["d"], 0.1, -1, 0, fa.FA_BF16, None)

    assert fwd(cu=None) == fa.FA_ERR_INVALID_ARG
    assert fwd(cu=FAKE + 2) == fa.FA_ERR_INVALID_ARG  # cu_seqlens not 4-byte aligned
    assert fwd(B=0) == fa.FA_ERR_INVALID_ARG
    assert fwd(max_seqlen=0) == fa.FA_ERR_INVALID_ARG
    assert fwd(T=0) == fa.FA_ERR_INVALID_ARG
    assert fwd(Hkv=3) == fa.FA_ERR_INVALID_ARG
    assert fwd(d=80) == fa.FA_ERR_UNSUPPORTED
    need = fa.fa_bwd_varlen_workspace_size(2, 100, 4, 2, 64)
    assert fa.fa_bwd_varlen(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need - 1, 2, 64, 100,
                            4, 2, 64, 0.1, -1, 0, None) == fa.FA_ERR_INVALID_ARG


def test_fp8_forward_rejects_bad_arguments():
    def call(d=128, qs=1.0, ks=1.0, vs=1.0, Hkv=2):
        return fa.fa_fwd_fp8(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, Hkv, 256, d, 0.1, qs, ks, vs, -1, 0, fa.FA_BF16, None)

    assert call(d=64) == fa.FA_ERR_UNSUPPORTED
    assert call(qs=0.0) == fa.FA_ERR_INVALID_ARG
    assert call(ks=-1.0) == fa.FA_ERR_INVALID_ARG
    assert call(vs=float("inf")) == fa.FA_ERR_INVALID_ARG
    assert call(vs=float("nan")) == fa.FA_ERR_INVALID_ARG
    assert call(Hkv=3) == fa.FA_ERR_INVALID_ARG


def test_sequence_length_limit():
    # N up to 2^29 keeps the kernels' 32-bit tile and band arithmetic exact.
    assert fa.fa_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, (1 << 29) + 1, 64, 0.1, 0, fa.FA_BF16,
                     None) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_bwd_workspace_size(1, 1, (1 << 29) + 1, 64) == 0
