"""KV-chunked attention and the exact log-sum-exp merge (test infrastructure).

Ring attention streams K/V chunks past a rank's queries and keeps an online
softmax, so no rank holds all of K/V (TensorRT 11.0 multi-device article,
section on the three context-parallel implementations, Ring Attention).  On
one device this is: split the keys into ``P`` contiguous chunks, compute a
partial result per chunk, merge the partials.  For chunk ``p`` (keys
``[floor(p*S/P), floor((p+1)*S/P))``) the partial is plain attention over
those keys only:

    o_p, lse_p = attention(q, k[chunk p], v[chunk p])

and the merge (the split-reduction the accuracy table of "TensorRT
Multi-Device (multi-GPU) support", Validation, attributes its FP16 error to):

    L   = max_p lse_p
    lse = L + ln(sum_p exp(lse_p - L))
    o   = sum_p exp(lse_p - lse) * o_p

which equals monolithic attention in exact arithmetic.  Folding the chunks
in one at a time with the two-term form of the same merge (``accumulate``)
is what each ring rank does per step.  An empty chunk has
``lse_p = -inf`` and ``o_p = 0`` and contributes nothing.  This module does
not import ``oracle.attention``'s merge logic (there is none there); it calls
``attention`` only to produce each chunk's partial.
"""
from __future__ import annotations

import numpy as np

from .attention import attention


def chunk_bounds(S: int, P: int):
    """Contiguous chunk ``p`` covers keys ``[floor(p*S/P), floor((p+1)*S/P))``."""
    return [((p * S) // P, ((p + 1) * S) // P) for p in range(P)]


def partials(q, k, v, scale: float, P: int, rows=None):
    """Per-chunk partials: ``o_parts [P, R, H, d]``, ``lse_parts [P, H, R]``."""
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    o_list, l_list = [], []
    for lo, hi in chunk_bounds(k.shape[0], P):
        o_p, lse_p = attention(q, k[lo:hi], v[lo:hi], scale, rows=rows)
        o_list.append(o_p)
        l_list.append(lse_p)
    return np.stack(o_list), np.stack(l_list)


def merge(o_parts, lse_parts):
    """Exact merge of partials.

    ``o_parts [P, S, H, d]`` and ``lse_parts [P, H, S]`` (any float dtype,
    widened to float64) -> ``(o [S, H, d], lse [H, S])`` in float64.
    Rows whose every chunk is empty get ``o = 0``, ``lse = -inf``.
    """
    o_parts = np.asarray(o_parts).astype(np.float64)
    lse_parts = np.asarray(lse_parts).astype(np.float64)
    P, S, H, d = o_parts.shape
    L = lse_parts.max(axis=0)                                  # [H, S]
    finite = np.isfinite(L)
    L_safe = np.where(finite, L, 0.0)
    w = np.exp(lse_parts - L_safe[None])                       # [P, H, S]
    w = np.where(np.isneginf(lse_parts), 0.0, w)
    total = w.sum(axis=0)                                      # [H, S]
    lse = np.where(finite, L_safe + np.log(np.where(finite, total, 1.0)), -np.inf)
    lse_safe = np.where(finite, lse, 0.0)
    coef = np.exp(lse_parts - lse_safe[None])                  # exp(lse_p - lse)
    coef = np.where(np.isneginf(lse_parts) | ~finite[None], 0.0, coef)
    # o[s, h, :] = sum_p coef[p, h, s] * o_parts[p, s, h, :]
    o = np.einsum("phs,pshd->shd", coef, o_parts)
    return o, lse


def fp16_partials(o_parts):
    """The FP16 split-reduction: partial outputs stored in fp16.

    The accuracy table of "TensorRT Multi-Device (multi-GPU) support"
    (Validation) attributes the multi-device error to an FP16 split-reduction.
    Reading: each chunk's normalised output ``o_p`` is rounded to fp16
    (round to nearest, ties to even) where it is stored, while ``lse_p`` stays
    fp32; the merge above then runs on the rounded values.  numpy's float64 ->
    float16 cast rounds once, to nearest even.  Returns float16 ``o_parts``.
    """
    return np.asarray(o_parts, dtype=np.float64).astype(np.float16)


def accumulate(o_acc, lse_acc, o_c, lse_c):
    """One ring step: fold chunk ``(o_c, lse_c)`` into the running ``(o_acc, lse_acc)``.

    The online-softmax update a ring-attention rank applies as each K/V
    block arrives (TensorRT 11.0 multi-device article, Ring Attention),
    written as the two-term case of the merge above:

        lse_new = ln(exp(lse_acc) + exp(lse_c))
        o_new   = exp(lse_acc - lse_new) * o_acc + exp(lse_c - lse_new) * o_c

    ``o_* [S, H, d]``, ``lse_* [H, S]`` (widened to float64).  A row with
    ``lse_acc = -inf`` has seen no key: its ``o_acc`` is ignored (it may hold
    anything) and the result is ``(o_c, lse_c)``; an empty chunk
    (``lse_c = -inf``, its ``o_c`` likewise ignored) leaves the row
    unchanged.  Returns float64 arrays.
    """
    o_acc = np.asarray(o_acc).astype(np.float64)
    lse_acc = np.asarray(lse_acc).astype(np.float64)
    o_c = np.asarray(o_c).astype(np.float64)
    lse_c = np.asarray(lse_c).astype(np.float64)
    seen_a = ~np.isneginf(lse_acc)
    seen_c = ~np.isneginf(lse_c)
    L = np.maximum(lse_acc, lse_c)
    L_safe = np.where(np.isneginf(L), 0.0, L)
    ea = np.where(seen_a, np.exp(np.where(seen_a, lse_acc, 0.0) - L_safe), 0.0)
    ec = np.where(seen_c, np.exp(np.where(seen_c, lse_c, 0.0) - L_safe), 0.0)
    total = ea + ec
    any_seen = seen_a | seen_c
    lse_new = np.where(any_seen, L_safe + np.log(np.where(any_seen, total, 1.0)), -np.inf)
    wa = np.where(any_seen, ea / np.where(any_seen, total, 1.0), 0.0)   # [H, S]
    wc = np.where(any_seen, ec / np.where(any_seen, total, 1.0), 0.0)
    o_a = np.where(seen_a.T[:, :, None], o_acc, 0.0)                    # ignore unseen rows' o_acc
    o_b = np.where(seen_c.T[:, :, None], o_c, 0.0)                      # and an empty chunk's o_c
    o_new = wa.T[:, :, None] * o_a + wc.T[:, :, None] * o_b
    return o_new, lse_new


def ring_attention(q, k, v, scale: float, P: int, rows=None):
    """The per-rank ring loop on one device: start empty, fold the ``P``
    chunks' partials in order with ``accumulate``."""
    q = np.asarray(q)
    H, d = q.shape[1], q.shape[2]
    R = q.shape[0] if rows is None else len(rows if not isinstance(rows, (list, tuple)) else rows[0])
    o = np.zeros((R, H, d))
    lse = np.full((H, R), -np.inf)
    for lo, hi in chunk_bounds(np.asarray(k).shape[0], P):
        o_c, lse_c = attention(q, np.asarray(k)[lo:hi], np.asarray(v)[lo:hi], scale, rows=rows)
        o, lse = accumulate(o, lse, o_c, lse_c)
    return o, lse


def chunked_attention(q, k, v, scale: float, P: int, rows=None):
    """Partials over ``P`` chunks followed by the merge."""
    o_parts, lse_parts = partials(q, k, v, scale, P, rows=rows)
    return merge(o_parts, lse_parts)
