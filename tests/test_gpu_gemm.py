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


# ------------------------------------------------ q/k RMSNorm epilogue ----
# Reading: the sample block's RMSNorm acts on every head of q and of k after
# the projection (oracle/stack.py, qkv_qknorm).  Bound per element, first
# order in the fp32 errors: the final fp16 rounding, the element's own
# accumulation error times the normalising factor r*|g|, and the relative
# error every element of a head inherits from its mean square (twice the
# head's largest relative accumulation error) and rsqrt/products (2^-20),
# all doubled for safety.

def qknorm_bound(x, w, g_q, g_k, H, d, eps, K):
    acc = OS.linear(x, w)
    delta = K * 2.0 ** -24 * OS.linear(np.abs(x), np.abs(w))
    exact_f = np.concatenate([
        OS.rmsnorm(acc[:, :H * d].reshape(-1, H, d), g_q, eps).reshape(acc.shape[0], -1),
        OS.rmsnorm(acc[:, H * d:2 * H * d].reshape(-1, H, d), g_k, eps).reshape(acc.shape[0], -1),
        acc[:, 2 * H * d:]], axis=1)
    bound = fp16_ulp(exact_f) + delta
    h = H * d
    for sec, g in ((0, g_q), (1, g_k)):
        a = acc[:, sec * h:(sec + 1) * h].reshape(-1, H, d)
        dl = delta[:, sec * h:(sec + 1) * h].reshape(-1, H, d)
        r = 1.0 / np.sqrt(np.mean(a * a, axis=-1, keepdims=True) + eps)
        rel = 2 * np.max(dl * r, axis=-1, keepdims=True) + 2.0 ** -20
        y = np.abs(exact_f[:, sec * h:(sec + 1) * h].reshape(-1, H, d))
        own = dl * r * np.abs(np.asarray(g, dtype=np.float64))
        bound[:, sec * h:(sec + 1) * h] = (fp16_ulp(y) + 2 * (own + y * rel)).reshape(-1, h)
    return exact_f, bound


def norm_weights(d, seed):
    rng = np.random.default_rng(seed)
    g_q = (1.0 + 0.1 * rng.standard_normal(d)).astype(np.float16)
    g_k = (1.0 + 0.1 * rng.standard_normal(d)).astype(np.float16)
    return g_q, g_k


@pytest.mark.parametrize("M,H,d,K", [(300, 2, 64, 128), (129, 3, 128, 256), (1000, 4, 128, 512), (77, 1, 64, 64)])
def test_qkv_proj_qknorm_shapes(b2a, M, H, d, K):
    x, w = W.gemm_operands(M, 3 * H * d, K, seed=M + H + K)
    g_q, g_k = norm_weights(d, M)
    eps = 1e-6
    out = b2a.qkv_proj_qknorm(torch.from_numpy(x).cuda(), torch.from_numpy(w).cuda(),
                              torch.from_numpy(g_q).cuda(), torch.from_numpy(g_k).cuda(), H, d, eps)
    b2a.check_status()
    exact, bound = qknorm_bound(x, w, g_q, g_k, H, d, eps, K)
    gpu = out.cpu().numpy().astype(np.float64)
    worst = float(np.max(np.abs(gpu - exact) / bound))
    assert worst <= 1.0, f"qknorm {M}x{H}x{d}x{K}: worst error {worst:.2f} of the bound"
    assert_out_close(gpu, OS.qkv_qknorm(x, w, g_q, g_k, H, d, eps), f"qknorm {M}x{H}x{d}x{K}")


def test_qkv_proj_qknorm_unit_mean_square(b2a):
    # g = 1, eps = 0: every q and k head comes out with mean square 1 (up to
    # fp16 rounding); v is the plain projection
    M, H, d, K = 500, 3, 128, 256
    x, w = W.gemm_operands(M, 3 * H * d, K, seed=31)
    ones = torch.ones(d, dtype=torch.float16, device="cuda")
    xd, wd = torch.from_numpy(x).cuda(), torch.from_numpy(w).cuda()
    out = b2a.qkv_proj_qknorm(xd, wd, ones, ones, H, d, 0.0).cpu().numpy().astype(np.float64)
    b2a.check_status()
    qk = out[:, :2 * H * d].reshape(M, 2 * H, d)
    np.testing.assert_allclose(np.mean(qk * qk, axis=-1), 1.0, atol=2e-3)
    plain = b2a.qkv_proj(xd, wd).cpu().numpy()
    np.testing.assert_array_equal(out[:, 2 * H * d:], plain[:, 2 * H * d:].astype(np.float64))


def test_qkv_proj_qknorm_full_size_sampled_rows(b2a):
    w = W.STACK6
    x = W.stack_x(w)
    w_qkv, _ = W.stack_weights(w, 0)
    g_q, g_k = norm_weights(w.d, 7)
    out = b2a.qkv_proj_qknorm(torch.from_numpy(x).cuda(), torch.from_numpy(w_qkv).cuda(),
                              torch.from_numpy(g_q).cuda(), torch.from_numpy(g_k).cuda(), w.H, w.d, 1e-6)
    b2a.check_status()
    rows = W.sample_rows(w.S, 1, 0, seed=4)[:64]
    exact, bound = qknorm_bound(x[rows], w_qkv, g_q, g_k, w.H, w.d, 1e-6, w.hidden)
    gpu = out.cpu().numpy()[rows].astype(np.float64)
    worst = float(np.max(np.abs(gpu - exact) / bound))
    assert worst <= 1.0, f"qknorm full size: worst error {worst:.2f} of the bound"
