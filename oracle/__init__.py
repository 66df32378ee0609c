"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it. It shares
no code with the CUDA library and does not import it.

Functions and what pins them (the pins live in ``tests/test_oracle_*.py``):

- ``attention_forward``      standard three-step attention, full rows of S.
  Pinned by: torch fp64 SDPA (library special case), closed forms (Q = 0,
  N = 1, constant V), permutation equivariance/invariance, hand-worked golden
  cases, and the blockwise online merge below.
- ``attention_forward_rows`` the same for a chosen subset of query rows.
  Pinned by: equality with the rows of ``attention_forward``.
- ``attention_backward``     analytic gradients of the forward.
  Pinned by: central finite differences on N <= 16, torch fp64 autograd.
- ``attention_backward_rows`` the work of a subset of query rows (dQ rows,
  partial dK/dV). Pinned by: its pieces over a partition of the rows add up
  to ``attention_backward``.
- ``attention_forward_gqa`` / ``attention_backward_gqa`` grouped K/V heads
  (MQA/GQA): the definition with K/V heads repeated per group; dK, dV summed
  over the group. Pinned by: central finite differences with respect to the
  shared K/V tensors, the MQA closed form for Q = 0, and group size 1 = MHA.
- ``window=(wl, wr)`` on the forward and backward functions: the local-window
  (band) mask i - wl <= j <= i + wr. Pinned by: a pure-Python per-row
  computation over the explicitly listed visible keys, the closed form for
  wl = wr = 0 (O = V, lse = scale q.k), unbounded windows equal to the full and
  causal masks, and central finite differences of the backward.
- ``attention_forward_varlen`` / ``attention_backward_varlen`` packed
  variable-length batches: each sequence attended on its own. Pinned by: a
  pure-Python per-row computation over each row's own sequence, equal
  lengths = the fixed-length batch, and independence from the other
  sequences' contents.
- ``e4m3_decode`` the 8-bit e4m3 code to value map, written from the format
  definition. Pinned by: torch's float8_e4m3fn for all 256 codes and
  hand-worked codes (448, 2^-6, 2^-9, NaN).
- ``attention_forward_fp8`` exact attention of per-tensor-scaled e4m3 Q, K,
  V. Pinned by: the decoder's pins, the trade between a tensor's scale and the
  softmax scale, linearity of O in the V scale, and lse's independence of it.
- ``blockwise_online_softmax_attention`` the tiled merge with running max and
  running sum. Pinned by: equality with the full-row softmax on tiny inputs,
  for several block sizes.

No function here is "parity unpinned".
"""

from .attention import (  # noqa: F401
    attention_forward,
    attention_forward_rows,
    attention_backward,
    attention_backward_rows,
    attention_backward_gqa,
    attention_forward_gqa,
    attention_backward_varlen,
    attention_forward_varlen,
    band_visible,
    causal_visible,
)
from .fp8 import attention_forward_fp8, e4m3_decode  # noqa: F401
from .online_softmax import blockwise_online_softmax_attention  # noqa: F401
