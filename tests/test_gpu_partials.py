"""attn_fwd_partials: every key chunk's partial in one call.

Short chunks run as one launch of the single-CTA kernel over (row block,
chunk, head); long chunks as one CTA-pair launch each; Skv < P (empty
chunks) one call per chunk.  Each chunk's result must be bit for bit that of
an attn_fwd_partial call on the chunk, and match the FP64 oracle.
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import chunked as OC
from parity import assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def b2a():
    import long_context_bidirectional_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def per_chunk(b2a, q, k, v, P, scale, dtype):
    Sq, H, d = q.shape
    o = torch.empty((P, Sq, H, d), dtype=dtype, device="cuda")
    l = torch.empty((P, H, Sq), dtype=torch.float32, device="cuda")
    part = b2a.attn_fwd_partial_f16 if dtype == torch.float16 else b2a.attn_fwd_partial
    for c, (lo, hi) in enumerate(b2a.chunk_bounds(k.shape[0], P)):
        part(q, k[lo:hi], v[lo:hi], o[c], l[c], scale=scale)
    return o, l


# (Sq, Skv, P, H, d): even and uneven chunks, ragged tiles, d = 64, chunks
# long enough for CTA pairs, and more chunks than keys
SHAPES = [
    (300, 1024, 2, 2, 128), (129, 1000, 3, 1, 128), (256, 513, 4, 3, 128), (1000, 4096, 8, 2, 128),
    (77, 129, 7, 2, 64), (500, 1000, 3, 2, 64), (64, 13000, 2, 1, 128), (40, 5, 8, 2, 128),
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16])
@pytest.mark.parametrize("Sq,Skv,P,H,d", SHAPES)
def test_partials_equal_per_chunk_calls_and_oracle(b2a, Sq, Skv, P, H, d, dtype):
    q, k, v = W.qkv(Sq, H, d, seed=Sq + Skv + P, q_sigma=2.0, Skv=Skv)
    scale = 1 / math.sqrt(d)
    qd, kd, vd = dev(q), dev(k), dev(v)
    o, l = b2a.attn_fwd_partials(qd, kd, vd, P, scale=scale, partial_dtype=dtype)
    o_ref, l_ref = per_chunk(b2a, qd, kd, vd, P, scale, dtype)
    b2a.check_status()
    assert torch.equal(o, o_ref)
    assert torch.equal(l, l_ref)
    ref_o, ref_l = OC.partials(q, k, v, scale, P)
    for c in range(P):
        if np.all(np.isneginf(ref_l[c])):           # an empty chunk
            assert torch.all(o[c] == 0) and torch.all(torch.isneginf(l[c]))
            continue
        assert_out_close(o[c].cpu().numpy().astype(np.float64), ref_o[c], f"partial {c}")
        assert_lse_close(l[c].cpu().numpy(), ref_l[c])


def test_partials_with_forced_kernels(b2a):
    # single CTAs forced on chunks the library would give to CTA pairs, and
    # pairs forced on short ones: all agree bit for bit
    Sq, Skv, P, H, d = 200, 12800, 2, 2, 128
    q, k, v = W.qkv(Sq, H, d, seed=91, q_sigma=3.0, Skv=Skv)
    qd, kd, vd = dev(q), dev(k), dev(v)
    outs = []
    for choice in (b2a.ATTN_KERNEL_AUTO, b2a.ATTN_KERNEL_SINGLE, b2a.ATTN_KERNEL_PAIR):
        b2a.set_attn_kernel(choice)
        try:
            outs.append(b2a.attn_fwd_partials(qd, kd, vd, P, scale=0.1))
            b2a.check_status()
        finally:
            b2a.set_attn_kernel(b2a.ATTN_KERNEL_AUTO)
    for o, l in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1])
