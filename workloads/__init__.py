"""Seeded synthetic inputs and the workload table.

This module is the only code shared by the CUDA path's callers (tests, bench)
and the FP64 oracle's callers.  It draws random numbers and names shapes; it
holds none of the attention arithmetic.

Input recipe (the pages print no data; they describe the workloads only):

* Q, K, V are ``[S, H, d]`` fp16, drawn in that order from one
  ``numpy.random.default_rng(seed)`` stream as float32 standard normals,
  multiplied by their standard deviation in float32 and rounded to fp16
  (round-to-nearest-even).  The self-attention block of the TensorRT sample
  ("Multi-Device Attention Inference with TensorRT", Generating the ONNX
  Models) feeds ``(S, B, 4096)`` fp16 activations into 32 heads of 128.
* The 6-block stack ("TensorRT Multi-Device (multi-GPU) support", Validation,
  multi-layer table): x ``[S, 4096]`` N(0,1) from seed ``seed``; block ``i``
  weights ``W_qkv [3h, h]`` from seed ``100 + 2i`` and ``W_o [h, h]`` from
  seed ``101 + 2i``, both N(0, 0.02**2), nn.Linear ``[out, in]`` layout.
* Sampled query rows for sequences too long for a full FP64 pass.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class AttnWorkload:
    """One attention workload: batch 1, ``S`` tokens, ``H`` heads of ``d``."""

    name: str
    S: int
    H: int
    d: int
    q_sigma: float = 1.0
    kv_sigma: float = 1.0
    P: int = 1               # KV chunks for the partial + merge form
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def hidden(self) -> int:
        return self.H * self.d

    @property
    def flops(self) -> float:
        """4*S^2*d*H: two GEMM-shaped contractions of 2*S^2*d each, per head."""
        return 4.0 * self.S * self.S * self.d * self.H


@dataclasses.dataclass(frozen=True)
class StackWorkload:
    """``blocks`` stacked self-attention blocks on ``x [S, H*d]``."""

    name: str
    S: int
    H: int
    d: int
    blocks: int
    w_sigma: float = 0.02
    seed: int = 0

    @property
    def hidden(self) -> int:
        return self.H * self.d

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


# The workloads of the pages (TensorRT Multi-Device support, Validation
# tables: seq 8192..65536 at hidden 4096, seq 8192 at hidden 8192, a 6-block
# stack at seq 32768) plus a tiny case an FP64 pass finishes in milliseconds.
TINY = AttnWorkload("tiny_s256_h2_d64", S=256, H=2, d=64, P=2)
SEQ8K = AttnWorkload("s8192_h32_d128", S=8192, H=32, d=128, P=2)
SEQ32K = AttnWorkload("s32768_h32_d128_qsig4", S=32768, H=32, d=128, q_sigma=4.0, P=8)
SEQ64K = AttnWorkload("s65536_h32_d128", S=65536, H=32, d=128, P=1)
SEQ8K_H64 = AttnWorkload("s8192_h64_d128", S=8192, H=64, d=128, P=1)
# The sample's default run ("Multi-Device Attention Inference with TensorRT",
# Running the Sample: --sequence-length 56320 --batch-size 1).
SEQ56K = AttnWorkload("s56320_h32_d128", S=56320, H=32, d=128, P=1)
STACK6 = StackWorkload("stack6_s32768_h4096", S=32768, H=32, d=128, blocks=6)
# A shorter stack that a full (unsampled) FP64 pass can follow end to end.
STACK6_S2048 = StackWorkload("stack6_s2048_h4096", S=2048, H=32, d=128, blocks=6)

ATTN_WORKLOADS = {w.name: w for w in (TINY, SEQ8K, SEQ32K, SEQ64K, SEQ8K_H64, SEQ56K)}
STACK_WORKLOADS = {w.name: w for w in (STACK6, STACK6_S2048)}


def _normal16(rng: np.random.Generator, shape, sigma: float) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    return x.astype(np.float16)


def qkv(S: int, H: int, d: int, seed: int = 0, q_sigma: float = 1.0,
        kv_sigma: float = 1.0, Skv: int | None = None):
    """Q ``[S,H,d]``, K and V ``[Skv,H,d]`` fp16, drawn in the order Q, K, V."""
    Skv = S if Skv is None else Skv
    rng = np.random.default_rng(seed)
    q = _normal16(rng, (S, H, d), q_sigma)
    k = _normal16(rng, (Skv, H, d), kv_sigma)
    v = _normal16(rng, (Skv, H, d), kv_sigma)
    return q, k, v


def workload_qkv(w: AttnWorkload):
    return qkv(w.S, w.H, w.d, seed=w.seed, q_sigma=w.q_sigma, kv_sigma=w.kv_sigma)


def stack_x(w: StackWorkload) -> np.ndarray:
    rng = np.random.default_rng(w.seed)
    return _normal16(rng, (w.S, w.hidden), 1.0)


def stack_weights(w: StackWorkload, block: int):
    """``(W_qkv [3h, h], W_o [h, h])`` fp16 for block ``block``."""
    h = w.hidden
    w_qkv = _normal16(np.random.default_rng(100 + 2 * block), (3 * h, h), w.w_sigma)
    w_o = _normal16(np.random.default_rng(101 + 2 * block), (h, h), w.w_sigma)
    return w_qkv, w_o


def gemm_operands(M: int, N: int, K: int, seed: int = 0, a_sigma: float = 1.0,
                  w_sigma: float = 0.02):
    """``A [M,K]`` and ``W [N,K]`` fp16 for a standalone projection GEMM."""
    rng = np.random.default_rng(seed)
    a = _normal16(rng, (M, K), a_sigma)
    wt = _normal16(rng, (N, K), w_sigma)
    return a, wt


def merge_operands(P: int, S: int, H: int, d: int, seed: int = 0,
                   lse_sigma: float = 4.0, empty_chunks=()):
    """Random partials in the merge's layouts.

    ``o_parts [P,S,H,d]`` float32 N(0,1) and ``lse_parts [P,H,S]`` float32
    N(0, lse_sigma**2).  Chunks listed in ``empty_chunks`` get ``lse = -inf``
    and ``o = 0``, the values an empty KV chunk produces.
    """
    rng = np.random.default_rng(seed)
    o = rng.standard_normal((P, S, H, d), dtype=np.float32)
    lse = rng.standard_normal((P, H, S), dtype=np.float32) * np.float32(lse_sigma)
    for p in empty_chunks:
        o[p] = 0.0
        lse[p] = -np.inf
    return o, lse


def sample_rows(S: int, P: int, head: int, seed: int = 0, n: int = 256) -> np.ndarray:
    """Query rows to compare for one head when a full FP64 pass is too slow.

    Always the first and last rows and the rows on both sides of every chunk
    boundary floor(p*S/P); the rest are drawn without replacement from
    ``default_rng([seed, head])``; sorted, at most ``n`` rows.
    """
    fixed = {0, S - 1}
    for p in range(1, P):
        b = (p * S) // P
        fixed.update({b - 1, b})
    fixed = sorted(r for r in fixed if 0 <= r < S)
    if S <= n:
        return np.arange(S, dtype=np.int64)
    rng = np.random.default_rng([seed, head])
    pool = np.setdiff1d(np.arange(S, dtype=np.int64), np.array(fixed, dtype=np.int64))
    extra = rng.choice(pool, size=max(0, n - len(fixed)), replace=False)
    return np.sort(np.concatenate([np.array(fixed, dtype=np.int64), extra]))[:n]
