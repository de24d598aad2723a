"""CUDA projection GEMMs (qkv_proj, out_proj) against the FP64 oracle.

The GPU rounds fp32 accumulators once to fp16; the oracle's exact product is
rounded by the same rule.  Each element may differ from the exact value by
half an fp16 ulp of rounding plus the fp32 accumulation error, so the
per-element bound is one fp16 ulp of the exact value (or 1e-6 near zero),
on top of the benchmark spec max_abs / rel-Frobenius bars.
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


def check(gpu16, exact, what):
    gpu = np.asarray(gpu16, dtype=np.float64)
    err = np.abs(gpu - exact)
    bound = np.maximum(fp16_ulp(exact), 1e-6)
    worst = float(np.max(err / bound))
    assert worst <= 1.0, f"{what}: worst error {worst:.2f} ulp"
    assert_out_close(gpu, exact, what)


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (200, 264, 72), (1000, 768, 1024), (77, 8, 8),
                                   (513, 520, 4096)])
def test_qkv_proj_shapes(b2a, M, N, K):
    a, w = W.gemm_operands(M, N, K, seed=M + N + K)
    out = b2a.qkv_proj(torch.from_numpy(a).cuda(), torch.from_numpy(w).cuda())
    b2a.check_status()
    check(out.cpu().numpy(), OS.linear(a, w), f"qkv {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 512, 256), (1000, 4096, 4096)])
def test_out_proj_with_residual(b2a, M, N, K):
    a, w = W.gemm_operands(M, N, K, seed=M * 3 + K)
    r = np.random.default_rng(5).standard_normal((M, N), dtype=np.float32).astype(np.float16)
    rd = torch.from_numpy(r).cuda()
    y = b2a.out_proj(torch.from_numpy(a).cuda(), torch.from_numpy(w).cuda(), residual=rd)
    b2a.check_status()
    check(y.cpu().numpy(), r.astype(np.float64) + OS.linear(a, w), f"out {M}x{N}x{K}")
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
    check(out.cpu().numpy()[rows], OS.linear(x[rows], w_qkv), "qkv 32768x12288x4096 sampled")
