"""Monolithic non-causal attention in FP64 (test infrastructure only).

What it computes, per head ``h`` and query row ``i`` (every query attends to
every key: "Multi-Device Attention Inference with TensorRT", Introduction;
no causal mask: the TensorRT 11.0 multi-device article, section on choosing a
parallel strategy, context parallelism for bidirectional DiT attention;
per-head scaled dot-product attention: "Tensor Parallelism: Sharding Weights
for Parallel Layer Execution", section 3, steps 2-3):

    s_ij  = scale * sum_e q_ie k_je
    m_i   = max_j s_ij
    l_i   = sum_j exp(s_ij - m_i)
    o_i   = (sum_j exp(s_ij - m_i) v_j) / l_i
    lse_i = m_i + ln(l_i)

Readings where the pages are silent:

* ``scale`` multiplies the logits (the sample's graph feeds a pre-scaled Q,
  "What is hint.json?", ``q_scaled``); the oracle applies it in FP64 to the
  exact products rather than rounding ``q*scale`` to fp16.
* The log-sum-exp is the natural log and includes ``scale``.
* No keys (``Skv == 0``) gives ``o = 0`` and ``lse = -inf``: the empty sum.

Inputs of any float dtype are widened exactly to float64.  The logits of a
block of query rows against all keys are materialised with one numpy matmul;
there is no online rescaling, tiling of keys or reordering.
"""
from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x).astype(np.float64)


def attention(q, k, v, scale: float, rows=None, row_block: int = 512):
    """Return ``(out [R, H, d], lse [H, R])`` in float64.

    ``q [Sq, H, d]``, ``k, v [Skv, H, d]``.  ``rows`` (optional) selects the
    query rows to evaluate, either one index array for all heads or a list of
    one array per head; ``R`` is their count (``Sq`` when omitted).  With a
    per-head list every head must select the same number of rows.
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    Sq, H, d = q.shape
    Skv = k.shape[0]
    if rows is None:
        rows_h = [np.arange(Sq)] * H
    elif isinstance(rows, (list, tuple)):
        rows_h = [np.asarray(r, dtype=np.int64) for r in rows]
    else:
        rows_h = [np.asarray(rows, dtype=np.int64)] * H
    R = len(rows_h[0])
    out = np.zeros((R, H, d), dtype=np.float64)
    lse = np.full((H, R), -np.inf, dtype=np.float64)
    if Skv == 0:
        return out, lse
    scale = float(scale)
    for h in range(H):
        kh = _f64(k[:, h, :])                 # [Skv, d]
        vh = _f64(v[:, h, :])                 # [Skv, d]
        rh = rows_h[h]
        for r0 in range(0, R, row_block):
            sel = rh[r0:r0 + row_block]
            qh = _f64(q[sel, h, :])           # [b, d]
            s = scale * (qh @ kh.T)           # [b, Skv] logits
            m = s.max(axis=1, keepdims=True)  # row max
            e = np.exp(s - m)                 # unnormalised probabilities
            l = e.sum(axis=1, keepdims=True)  # row sum
            out[r0:r0 + len(sel), h, :] = (e @ vh) / l
            lse[h, r0:r0 + len(sel)] = m[:, 0] + np.log(l[:, 0])
    return out, lse


def probabilities(q, k, scale: float, head: int):
    """The softmax matrix ``[Sq, Skv]`` of one head, for invariant checks."""
    qh = _f64(np.asarray(q)[:, head, :])
    kh = _f64(np.asarray(k)[:, head, :])
    s = float(scale) * (qh @ kh.T)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=1, keepdims=True)
