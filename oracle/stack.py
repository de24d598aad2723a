"""Stacked self-attention blocks in FP64 (test infrastructure only).

The sample model is a self-attention block on ``(S, B, 4096)`` fp16 with 32
heads of 128, built from Q/K/V projections, scaled dot-product attention and
an output projection ("Multi-Device Attention Inference with TensorRT",
Generating the ONNX Models, step 1); the compute-bound benchmark stacks six
such blocks ("TensorRT Multi-Device (multi-GPU) support", Validation,
multi-layer model).  Projections follow "Tensor Parallelism: Sharding Weights
for Parallel Layer Execution", section 3: ``Q = X W_Q`` etc., heads split,
attention per head, ``Z = Concat(heads) W_O``.

Readings where the pages are silent:

* Weights are stored ``[out, in]`` and applied as ``y = x W^T``; no bias.
* The fused QKV output has columns ``[q | k | v]``, each ``H*d`` wide and
  head-major (column ``head*d + e``).
* The block output is ``x + Z`` (a residual add).
* RMSNorm, listed in the sample model without placement or epsilon, is not
  part of ``block``/``stack``.  ``qkv_qknorm`` gives the reading used when it
  is asked for: the sample names the norm after the Q/K/V projections and
  ahead of the attention in its layer list, so the norm acts on the
  projected q and k, per head, before attention (``qkv_qknorm``
  below; epsilon 1e-6 unless given, one weight vector of length d for q and
  one for k, shared by the heads).
* Tensors are rounded to fp16 (round-to-nearest-even) exactly where the
  library stores fp16: after the QKV projection, after attention, after the
  residual add.  Everything between those boundaries is float64.
"""
from __future__ import annotations

import numpy as np

from .attention import attention


def round16(x) -> np.ndarray:
    """Round to the nearest fp16 (ties to even), returned as fp16."""
    return np.asarray(x, dtype=np.float64).astype(np.float16)


def linear(x, w) -> np.ndarray:
    """``x [M, K] @ w[N, K]^T`` in float64."""
    return np.asarray(x).astype(np.float64) @ np.asarray(w).astype(np.float64).T


def rmsnorm(x, g, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: ``x / sqrt(mean(x**2) + eps) * g``, float64."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(g, dtype=np.float64)


def qkv_qknorm(x16, w_qkv16, g_q16, g_k16, H: int, d: int, eps: float):
    """The fused QKV projection with the RMSNorm reading applied: every head
    of q and of k (``d`` features each) is RMS-normalised and scaled by the
    per-feature weights ``g_q`` / ``g_k`` (length ``d``, shared by the heads),
    from the exact projection; v is left as projected.  One fp16 rounding.
    Returns ``qkv16 [S, 3*H*d]``.
    """
    S = x16.shape[0]
    h = H * d
    acc = linear(x16, w_qkv16)                             # [S, 3h] exact
    q = rmsnorm(acc[:, 0:h].reshape(S, H, d), g_q16, eps).reshape(S, h)
    k = rmsnorm(acc[:, h:2 * h].reshape(S, H, d), g_k16, eps).reshape(S, h)
    return round16(np.concatenate([q, k, acc[:, 2 * h:3 * h]], axis=1))


def block(x16, w_qkv16, w_o16, H: int, d: int, scale: float, norm=None):
    """One block on all rows.  Returns ``(y16, qkv16, a16)``, all fp16.

    ``norm = (g_q16, g_k16, eps)`` applies the q/k RMSNorm reading.
    """
    S = x16.shape[0]
    h = H * d
    if norm is None:
        qkv16 = round16(linear(x16, w_qkv16))              # [S, 3h]
    else:
        qkv16 = qkv_qknorm(x16, w_qkv16, norm[0], norm[1], H, d, norm[2])
    q = qkv16[:, 0 * h:1 * h].reshape(S, H, d)
    k = qkv16[:, 1 * h:2 * h].reshape(S, H, d)
    v = qkv16[:, 2 * h:3 * h].reshape(S, H, d)
    a, _ = attention(q, k, v, scale)
    a16 = round16(a.reshape(S, h))
    y16 = round16(np.asarray(x16, dtype=np.float64) + linear(a16, w_o16))
    return y16, qkv16, a16


def block_rows(x16, w_qkv16, w_o16, H: int, d: int, scale: float, rows):
    """One block evaluated on selected query rows only.

    K and V need every row of the input, so they are projected in full; Q,
    attention, output projection and residual are evaluated on ``rows``.
    Returns ``(y16[rows], qkv16[rows], a16[rows])``.
    """
    S = x16.shape[0]
    h = H * d
    rows = np.asarray(rows, dtype=np.int64)
    kv16 = round16(linear(x16, w_qkv16[h:3 * h]))          # [S, 2h]
    q16 = round16(linear(x16[rows], w_qkv16[0:h]))         # [R, h]
    k = kv16[:, 0:h].reshape(S, H, d)
    v = kv16[:, h:2 * h].reshape(S, H, d)
    a, _ = attention(q16.reshape(len(rows), H, d), k, v, scale)
    a16 = round16(a.reshape(len(rows), h))
    y16 = round16(np.asarray(x16[rows], dtype=np.float64) + linear(a16, w_o16))
    qkv_rows = np.concatenate([q16, kv16[rows]], axis=1)
    return y16, qkv_rows, a16


def stack(x16, weights, H: int, d: int, scale: float):
    """Run the blocks in order; ``weights`` is a list of ``(w_qkv16, w_o16)``.

    Returns the list of per-block ``(y16, qkv16, a16)``.
    """
    outs = []
    x = x16
    for w_qkv16, w_o16 in weights:
        y, qkv, a = block(x, w_qkv16, w_o16, H, d, scale)
        outs.append((y, qkv, a))
        x = y
    return outs
