"""FP64 CPU oracle for non-causal scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the C-ABI library and
its Python binding) may import, call or link anything here; only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference arm
use it.  It shares no code with the CUDA path.

Modules:

* ``attention`` -- monolithic softmax(scale*Q*K^T)*V per head plus the per-row
  natural-log log-sum-exp, written as the plain definition (full logits row,
  max-subtracted exponentials, sum, divide).
* ``chunked``   -- the KV-chunked form: one partial (output, LSE) per chunk of
  keys, then the exact log-sum-exp merge; and the ring step that folds one
  chunk into a running (output, LSE).
* ``stack``     -- the stacked self-attention block: fused QKV projection,
  attention, output projection and residual add, rounded to fp16 at the
  tensor boundaries the C-ABI stores.

Every function is pinned by ``tests/test_oracle_pins.py`` against closed forms,
invariants, brute-force loops and library routines; none is "parity unpinned".
"""
from . import attention, chunked, stack  # noqa: F401
