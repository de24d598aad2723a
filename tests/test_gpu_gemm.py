"""CUDA projection GEMMs (qkv_proj, out_proj) against the FP64 oracle.

The GPU accumulates fp16 products in fp32 and rounds once to fp16.  Each
element may differ from the exact product by the final rounding (at most one
fp16 ulp of the exact value, allowing for a result that rounds across a
power of two) plus the fp32 summation error, bounded by the standard
K * 2^-24 * sum_k |a_k w_k| (Higham, Accuracy and Stability of Numerical
Algorithms, section 3.1).  The max_abs / rel-Frobenius bars apply on top.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import stack as OS
from parity import assert_out_close, fp16_ulp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def b2a():
    import long_context_bidirectional_b200 as m
    return m


def check(gpu16, exact, what, abs_sum, K):
    gpu = np.asarray(gpu16, dtype=np.float64)
    err = np.abs(gpu - exact)
    bound = fp16_ulp(exact) + K * 2.0 ** -24 * abs_sum
    worst = float(np.max(err / bound))
    assert worst <= 1.0, f"{what}: worst error {worst:.2f} of the bound"
    assert_out_close(gpu, exact, what)


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (200, 264, 72), (1000, 768, 1024), (77, 8, 8),
                                   (513, 520, 4096)])
def test_qkv_proj_shapes(b2a, M, N, K):
    a, w = W.gemm_operands(M, N, K, seed=M + N + K)
    out = b2a.qkv_proj(torch.from_numpy(a).cuda(), torch.from_numpy(w).cuda())
    b2a.check_status()
    check(out.cpu().numpy(), OS.linear(a, w), f"qkv {M}x{N}x{K}", OS.linear(np.abs(a), np.abs(w)), K)


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 512, 256), (1000, 4096, 4096)])
def test_out_proj_with_residual(b2a, M, N, K):
    a, w = W.gemm_operands(M, N, K, seed=M * 3 + K)
    r = np.random.default_rng(5).standard_normal((M, N), dtype=np.float32).astype(np.float16)
    rd = torch.from_numpy(r).cuda()
    y = b2a.out_proj(torch.from_numpy(a).cuda(), torch.from_numpy(w).cuda(), residual=rd)
    b2a.check_status()
    check(y.cpu().numpy(), r.astype(np.float64) + OS.linear(a, w), f"out {M}x{N}x{K}",
          OS.linear(np.abs(a), np.abs(w)), K)
    # in place: residual aliases the output
    y2 = rd.clone()
    b2a.out_proj(torch.from_numpy(a).cuda(), torch.from_numpy(w).cuda(), residual=y2, out=y2)
    b2a.check_status()
    np.testing.assert_array_equal(y2.cpu().numpy(), y.cpu().numpy())


def test_qkv_proj_full_size_sampled_rows(b2a):
    # the stack's fused projection: [32768, 4096] x [12288, 4096]^T
    w = W.STACK6
    x = W.stack_x(w)
    w_qkv, _ = W.stack_weights(w, 0)
    out = b2a.qkv_proj(torch.from_numpy(x).cuda(), torch.from_numpy(w_qkv).cuda())
    b2a.check_status()
    rows = W.sample_rows(w.S, 1, 0, seed=3)
    check(out.cpu().numpy()[rows], OS.linear(x[rows], w_qkv), "qkv 32768x12288x4096 sampled",
          OS.linear(np.abs(x[rows]), np.abs(w_qkv)), w.hidden)
