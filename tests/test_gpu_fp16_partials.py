"""The FP16 split-reduction: fp16 chunk partials and their merge.

attn_fwd_partial_f16 stores o_part in fp16 (lse in fp32); attn_merge_f16
merges such partials.  Checked against the FP64 oracle (exact monolithic
attention, and the oracle merge of the same fp16 partials), and for
consistency with the fp32 partial form of the same kernels.
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
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


@pytest.mark.parametrize("P,S,H,d,empty", [
    (1, 64, 2, 64, ()), (2, 300, 3, 128, ()), (3, 257, 1, 64, (1,)), (8, 1000, 4, 128, (0, 7)),
    (5, 33, 32, 128, (0, 1, 2, 3)), (64, 40, 2, 64, (10,)),
])
def test_merge_f16_random_partials(b2a, P, S, H, d, empty):
    o, lse = W.merge_operands(P, S, H, d, seed=P * 1000 + S + 1, empty_chunks=empty)
    o16 = o.astype(np.float16)
    ref, ref_lse = OC.merge(o16, lse)
    out, lse_out = b2a.attn_merge_f16(dev(o16), dev(lse))
    b2a.check_status()
    assert_out_close(out.cpu().numpy().astype(np.float64), ref, "merge_f16 out")
    assert_lse_close(lse_out.cpu().numpy(), ref_lse)


def test_merge_f16_all_empty_rows(b2a):
    o, lse = W.merge_operands(3, 20, 2, 64, seed=4, empty_chunks=(0, 1, 2))
    out, lse_out = b2a.attn_merge_f16(dev(o.astype(np.float16)), dev(lse))
    b2a.check_status()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse_out))


def test_merge_f16_full_size_sampled(b2a):
    P, S, H, d = 8, 32768, 32, 128
    o, lse = W.merge_operands(P, S, H, d, seed=22)
    o16 = o.astype(np.float16)
    del o
    out, lse_out = b2a.attn_merge_f16(dev(o16), dev(lse))
    b2a.check_status()
    rows = W.sample_rows(S, P, 0, seed=22)
    ref, ref_lse = OC.merge(o16[:, rows], lse[:, :, rows])
    assert_out_close(out.cpu().numpy()[rows].astype(np.float64), ref, "merge_f16 32k sampled")
    assert_lse_close(lse_out.cpu().numpy()[:, rows], ref_lse)


@pytest.mark.parametrize("kernel", ["single", "pair"])
@pytest.mark.parametrize("Sq,Skv,H,d", [(256, 256, 2, 64), (1000, 333, 2, 128), (129, 1, 1, 128),
                                        (300, 700, 3, 128), (77, 5, 2, 64)])
def test_partial_f16_is_the_rounded_fp32_partial(b2a, kernel, Sq, Skv, H, d):
    # same kernel, same arithmetic: the fp16 partial is the fp32 partial rounded once
    if kernel == "pair" and d != 128:
        pytest.skip("the CTA-pair kernel is head dim 128 only")
    q, k, v = W.qkv(Sq, H, d, seed=Sq + Skv, Skv=Skv)
    b2a.set_attn_kernel(b2a.ATTN_KERNEL_PAIR if kernel == "pair" else b2a.ATTN_KERNEL_SINGLE)
    try:
        qd, kd, vd = dev(q), dev(k), dev(v)
        o32, l32 = b2a.attn_fwd_partial(qd, kd, vd, scale=1 / math.sqrt(d))
        o16, l16 = b2a.attn_fwd_partial_f16(qd, kd, vd, scale=1 / math.sqrt(d))
        b2a.check_status()
    finally:
        b2a.set_attn_kernel(b2a.ATTN_KERNEL_AUTO)
    assert torch.equal(o16, o32.half())
    assert torch.equal(l16, l32)
    ref, ref_lse = OA.attention(q, k, v, 1 / math.sqrt(d))
    assert_out_close(o16.cpu().numpy().astype(np.float64), ref, "fp16 partial")
    assert_lse_close(l16.cpu().numpy(), ref_lse)


def test_partial_f16_empty_chunk(b2a):
    q, _, _ = W.qkv(50, 2, 64, seed=9)
    qd = dev(q)
    o = torch.full((50, 2, 64), 7.0, dtype=torch.float16, device="cuda")
    l = torch.zeros((2, 50), dtype=torch.float32, device="cuda")
    b2a.attn_fwd_partial_f16(qd, qd[:0], qd[:0], o, l, scale=0.125)
    b2a.check_status()
    assert torch.all(o == 0) and torch.all(torch.isneginf(l))


@pytest.mark.parametrize("kernel", ["auto", "pair"])
@pytest.mark.parametrize("S,H,d,P", [(256, 2, 64, 2), (1000, 2, 128, 3), (129, 1, 64, 7),
                                     (5, 2, 128, 8), (700, 2, 128, 1), (1500, 2, 128, 4)])
def test_chunked_fp16_partials_against_oracle(b2a, kernel, S, H, d, P):
    if kernel == "pair" and d != 128:
        pytest.skip("the CTA-pair kernel is head dim 128 only")
    q, k, v = W.qkv(S, H, d, seed=200 + S + P, q_sigma=2.0)
    scale = 1 / math.sqrt(d)
    b2a.set_attn_kernel(b2a.ATTN_KERNEL_PAIR if kernel == "pair" else b2a.ATTN_KERNEL_AUTO)
    try:
        qd, kd, vd = dev(q), dev(k), dev(v)
        out, lse = b2a.attn_chunked(qd, kd, vd, P, scale=scale, partial_dtype=torch.float16)
        out32, lse32 = b2a.attn_chunked(qd, kd, vd, P, scale=scale)
        b2a.check_status()
    finally:
        b2a.set_attn_kernel(b2a.ATTN_KERNEL_AUTO)
    ref, ref_lse = OA.attention(q, k, v, scale)
    got = out.cpu().numpy().astype(np.float64)
    assert_out_close(got, ref, f"fp16 partials S={S} P={P}")
    assert_lse_close(lse.cpu().numpy(), ref_lse)
    # Against the fp32-partial form of the same kernels: the fp16 partials are
    # those partials rounded once (half an ulp each; the merge weights sum to
    # 1), and both results are rounded to fp16 at the end.
    assert torch.equal(lse, lse32)
    o_parts, _ = OC.partials(q, k, v, scale, P)
    ulp_p = np.spacing(np.abs(OC.fp16_partials(o_parts))).astype(np.float64).max(axis=0)
    got32 = out32.cpu().numpy().astype(np.float64)
    ulp_o = np.spacing(np.abs(got32).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(got - got32) <= ulp_p + ulp_o + 1e-6)
