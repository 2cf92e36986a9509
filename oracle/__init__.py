"""CPU oracle for the fused exact-attention forward — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import anything from here. The
product path (the C-ABI library and its Python binding) never does, and shares
no code with it: this package widens bf16 bit patterns itself, does its
arithmetic in numpy fp64 (fp32 only where the 8-bit method fixes fp32 as the
precision that decides an integer code), and materialises S and P.

Modules
  attention  exact definition softmax(scale * Q K^T [+ causal mask]) V and LSE
  quant8     the SageAttention-style 8-bit prepass steps (K mean smoothing,
             INT8 block quantisation, FP8 e4m3 encoding) and a one-shot
             quantised attention built from them
  backward   gradients dQ, dK, dV of the definition, in fp64
  partial    attention over a range of keys (global causal mask) and the
             exact merge of partial results by their LSE

Pins (tests/test_oracle.py, CPU-only) tie every function to something other
than itself: brute force on tiny inputs, closed forms, invariants the pages
state (rows of P sum to 1, online softmax equals one-shot softmax, shift
invariance under K mean smoothing, permutation equivariance), and library
special cases (torch SDPA in float64, torch float8_e4m3fn casts). The
backward is pinned by tests/test_oracle_backward.py (float64 autograd and
central finite differences), the key-range partials and their merge by
tests/test_oracle_partial.py (brute force, merged splits equal the full
attention, closed forms).
"""
from .attention import (attention_fp64, attention_f64, attention_varlen_fp64,  # noqa: F401
                        score_matrix_fp64, widen_bf16)
from . import quant8  # noqa: F401
from .backward import attention_bwd_fp64  # noqa: F401
from .partial import attention_partial_fp64, merge_partials_fp64  # noqa: F401
