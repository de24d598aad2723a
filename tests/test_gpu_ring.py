"""Ring-step accumulation and both head-dim-128 kernels against the FP64 oracle.

``attn_fwd_accumulate`` folds one key chunk into a running (o_acc, lse_acc)
in place, the per-step update of a ring-attention rank (TensorRT 11.0
multi-device article, Ring Attention).  After P steps over the chunks the
result must match monolithic attention (oracle ``attention``) and the
oracle's own ring fold (``chunked.ring_attention``) elementwise.

Head dim 128 has two kernels (single CTAs, and two-SM CTA pairs); the library
picks one by key count.  Here each is forced in turn over small and ragged
shapes so that both meet the same bars everywhere, not only at the sizes the
automatic choice sends them.
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


@pytest.fixture
def kernel(b2a, request):
    b2a.set_attn_kernel(request.param)
    assert b2a.get_attn_kernel() == request.param
    yield request.param
    b2a.set_attn_kernel(b2a.ATTN_KERNEL_AUTO)


SINGLE, PAIR, AUTO = 1, 2, 0


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def host(t):
    return t.detach().cpu().numpy()


# ------------------------------------------------------- forced kernel ----

@pytest.mark.parametrize("kernel", [SINGLE, PAIR], indirect=True)
@pytest.mark.parametrize("S,H", [(1, 1), (64, 1), (127, 2), (129, 2), (257, 3), (1000, 1)])
def test_forced_kernel_monolithic(b2a, kernel, S, H):
    q, k, v = W.qkv(S, H, 128, seed=S + 3 * H)
    scale = 1 / math.sqrt(128)
    out, lse = b2a.attn_fwd(dev(q), dev(k), dev(v), scale=scale)
    b2a.check_status()
    ref, ref_lse = OA.attention(q, k, v, scale)
    assert_out_close(host(out).astype(np.float64), ref, f"kernel {kernel} S={S} H={H}")
    assert_lse_close(host(lse), ref_lse)


@pytest.mark.parametrize("kernel", [SINGLE, PAIR], indirect=True)
@pytest.mark.parametrize("Sq,Skv", [(200, 700), (1000, 64), (300, 1), (130, 515), (5, 2000)])
def test_forced_kernel_partial(b2a, kernel, Sq, Skv):
    q, k, v = W.qkv(Sq, 2, 128, seed=Sq + Skv + 1, Skv=Skv)
    scale = 1 / math.sqrt(128)
    o, l = b2a.attn_fwd_partial(dev(q), dev(k), dev(v), scale=scale)
    b2a.check_status()
    ref, ref_lse = OA.attention(q, k, v, scale)
    assert_out_close(host(o), ref, f"kernel {kernel} partial Sq={Sq} Skv={Skv}")
    assert_lse_close(host(l), ref_lse)


@pytest.mark.parametrize("kernel", [SINGLE, PAIR], indirect=True)
def test_forced_kernel_rising_max(b2a, kernel):
    # keys sorted by their logit with query row 0: that row's running max
    # rises tile after tile and its O is rescaled repeatedly
    q, k, v = W.qkv(1500, 2, 128, seed=5, q_sigma=4.0)
    order = np.argsort(k[:, 0, :].astype(np.float64) @ q[0, 0, :].astype(np.float64))
    ks, vs = np.ascontiguousarray(k[order]), np.ascontiguousarray(v[order])
    scale = 1 / math.sqrt(128)
    out, lse = b2a.attn_fwd(dev(q), dev(ks), dev(vs), scale=scale)
    b2a.check_status()
    ref, ref_lse = OA.attention(q, ks, vs, scale)
    assert_out_close(host(out).astype(np.float64), ref, f"kernel {kernel} rising max")
    assert_lse_close(host(lse), ref_lse)


def test_both_kernels_agree_bitwise(b2a):
    # same arithmetic in the same order per row: identical bits
    q, k, v = W.qkv(2000, 3, 128, seed=21, q_sigma=2.0)
    res = []
    for choice in (SINGLE, PAIR):
        b2a.set_attn_kernel(choice)
        try:
            out, lse = b2a.attn_fwd(dev(q), dev(k), dev(v))
            b2a.check_status()
        finally:
            b2a.set_attn_kernel(AUTO)
        res.append((host(out), host(lse)))
    np.testing.assert_array_equal(res[0][0], res[1][0])
    np.testing.assert_array_equal(res[0][1], res[1][1])


# ---------------------------------------------------------- ring steps ----

def ring_on_gpu(b2a, q, k, v, P, scale, junk=True):
    """P accumulate steps; o_acc starts as NaN junk (must be ignored)."""
    S, H, d = q.shape
    qd, kd, vd = dev(q), dev(k), dev(v)
    o_acc = torch.full((S, H, d), float("nan") if junk else 0.0, dtype=torch.float32, device="cuda")
    lse_acc = torch.full((H, S), float("-inf"), dtype=torch.float32, device="cuda")
    out = torch.empty((S, H, d), dtype=torch.float16, device="cuda")
    bounds = b2a.chunk_bounds(k.shape[0], P)
    for c, (lo, hi) in enumerate(bounds):
        b2a.attn_fwd_accumulate(qd, kd[lo:hi], vd[lo:hi], o_acc, lse_acc, out if c == P - 1 else None,
                                scale=scale)
    b2a.check_status()
    return host(o_acc), host(lse_acc), host(out)


@pytest.mark.parametrize("kernel", [AUTO, SINGLE, PAIR], indirect=True)
@pytest.mark.parametrize("S,H,d,P,qs", [(1000, 2, 128, 3, 1.0), (777, 1, 64, 4, 1.0), (5, 2, 128, 8, 1.0),
                                        (300, 2, 128, 1, 1.0), (1500, 2, 128, 5, 4.0), (640, 3, 64, 7, 4.0)])
def test_ring_matches_oracle(b2a, kernel, S, H, d, P, qs):
    q, k, v = W.qkv(S, H, d, seed=S + P, q_sigma=qs)
    scale = 1 / math.sqrt(d)
    o_acc, lse_acc, out = ring_on_gpu(b2a, q, k, v, P, scale)
    ref, ref_lse = OA.attention(q, k, v, scale)
    assert_out_close(out.astype(np.float64), ref, f"ring out S={S} d={d} P={P}")
    assert_lse_close(lse_acc, ref_lse)
    o_r, l_r = OC.ring_attention(q, k, v, scale, P)
    assert_out_close(o_acc, o_r, f"ring o_acc S={S} d={d} P={P}")
    assert_lse_close(lse_acc, l_r)


def test_ring_equals_partials_and_merge(b2a):
    q, k, v = W.qkv(1200, 2, 128, seed=22, q_sigma=3.0)
    P = 4
    o_acc, lse_acc, out = ring_on_gpu(b2a, q, k, v, P, 0.1)
    out2, lse2 = b2a.attn_chunked(dev(q), dev(k), dev(v), P, scale=0.1)
    b2a.check_status()
    assert_out_close(out.astype(np.float64), host(out2).astype(np.float64), "ring vs merge")
    assert_lse_close(lse_acc, host(lse2), "ring vs merge lse")


def test_ring_empty_steps(b2a):
    q, k, v = W.qkv(300, 2, 64, seed=23)
    qd, kd, vd = dev(q), dev(k), dev(v)
    S, H, d = q.shape
    o_acc = torch.full((S, H, d), float("nan"), dtype=torch.float32, device="cuda")
    lse_acc = torch.full((H, S), float("-inf"), dtype=torch.float32, device="cuda")
    out = torch.empty((S, H, d), dtype=torch.float16, device="cuda")
    # an empty step before any key: nothing seen, out is all zeros
    b2a.attn_fwd_accumulate(qd, kd[:0], vd[:0], o_acc, lse_acc, out, scale=0.125)
    b2a.check_status()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse_acc))
    # one real step, then an empty one that must change nothing but write out
    b2a.attn_fwd_accumulate(qd, kd, vd, o_acc, lse_acc, None, scale=0.125)
    before_o, before_l = o_acc.clone(), lse_acc.clone()
    b2a.attn_fwd_accumulate(qd, kd[:0], vd[:0], o_acc, lse_acc, out, scale=0.125)
    b2a.check_status()
    assert torch.equal(o_acc, before_o) and torch.equal(lse_acc, before_l)
    assert torch.equal(out, before_o.half())
    ref, ref_lse = OA.attention(q, k, v, 0.125)
    assert_out_close(host(out).astype(np.float64), ref, "ring with empty steps")
    assert_lse_close(host(lse_acc), ref_lse)


def test_ring_workload_sampled(b2a):
    # the 8-chunk ring over the 32k, Q ~ N(0, 4^2) workload: sampled rows
    # against the oracle, every element against the GPU's monolithic result
    w = W.SEQ32K
    q, k, v = W.workload_qkv(w)
    rows = [W.sample_rows(w.S, w.P, h, seed=w.seed) for h in range(w.H)]
    ref, ref_lse = OA.attention(q, k, v, w.scale, rows=rows)
    qd, kd, vd = dev(q), dev(k), dev(v)
    out, lse = b2a.attn_ring(qd, kd, vd, w.P, scale=w.scale)
    mono, mono_lse = b2a.attn_fwd(qd, kd, vd, scale=w.scale)
    b2a.check_status()
    oh, lh = host(out), host(lse)
    got = np.stack([oh[rows[h], h, :] for h in range(w.H)], axis=1).astype(np.float64)
    got_lse = np.stack([lh[h, rows[h]] for h in range(w.H)]).astype(np.float64)
    assert_out_close(got, ref, "32k ring sampled")
    assert_lse_close(got_lse, ref_lse)
    assert_out_close(oh.astype(np.float64), host(mono).astype(np.float64), "32k ring vs mono")
    assert_lse_close(lh, host(mono_lse), "32k ring vs mono lse")
