"""Per-rank shapes of the context-parallel variants, on one GPU, against the
FP64 oracle and against the unsharded CUDA result.

* AllGather-KV (the sample's own hint: K/V gathered, Q local -- "Multi-Device
  Attention Inference with TensorRT", What is hint.json?): rank r keeps query
  rows [r*S/P, (r+1)*S/P) and attends to every key (``attn_fwd_gathered_kv``).
* Ulysses (TensorRT 11.0 multi-device article, the three context-parallel
  implementations): after the all-to-all a rank holds every row for H/P
  heads; on one device that is ``attn_fwd`` on a head slice of [S, H, d]
  (pointer offset, row stride H*d).

Each query row meets the same key tiles in the same order whichever rank
computes it, so the ranks' outputs put together equal the unsharded output
bit for bit (the pages report the 2-GPU result at seq 8192 bit-identical to
the 1-GPU one: "TensorRT Multi-Device (multi-GPU) support", Validation).
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from parity import assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu

SINGLE, PAIR, AUTO = 1, 2, 0


@pytest.fixture(scope="module")
def b2a():
    import long_context_bidirectional_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


@pytest.fixture
def kernel(b2a, request):
    b2a.set_attn_kernel(request.param)
    yield request.param
    b2a.set_attn_kernel(b2a.ATTN_KERNEL_AUTO)


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def host(t):
    return t.detach().cpu().numpy()


@pytest.mark.parametrize("kernel", [SINGLE, PAIR], indirect=True)
@pytest.mark.parametrize("Sq,Skv,d", [(200, 700, 128), (1000, 64, 128), (129, 1, 128), (333, 1000, 64)])
def test_gathered_kv_small_and_ragged(b2a, kernel, Sq, Skv, d):
    q, k, v = W.qkv(Sq, 2, d, seed=Sq * 3 + Skv, Skv=Skv, q_sigma=2.0)
    scale = 1 / math.sqrt(d)
    out, lse = b2a.attn_fwd_gathered_kv(dev(q), dev(k), dev(v), scale=scale)
    b2a.check_status()
    ref, ref_lse = OA.attention(q, k, v, scale)
    assert_out_close(host(out).astype(np.float64), ref, f"gathered-kv Sq={Sq} Skv={Skv} d={d}")
    assert_lse_close(host(lse), ref_lse)


@pytest.mark.parametrize("kernel", [AUTO, SINGLE, PAIR], indirect=True)
@pytest.mark.parametrize("S,H,P", [(8192, 4, 2), (3000, 2, 3)])
def test_gathered_kv_ranks_equal_unsharded(b2a, kernel, S, H, P):
    q, k, v = W.qkv(S, H, 128, seed=S + P)
    qd, kd, vd = dev(q), dev(k), dev(v)
    full, full_lse = b2a.attn_fwd(qd, kd, vd)
    parts, lses = [], []
    for lo, hi in b2a.chunk_bounds(S, P):
        o, l = b2a.attn_fwd_gathered_kv(qd[lo:hi], kd, vd)
        parts.append(o)
        lses.append(l)
    b2a.check_status()
    assert torch.equal(torch.cat(parts), full)
    assert torch.equal(torch.cat(lses, dim=1), full_lse)


@pytest.mark.parametrize("S,H,P", [(8192, 8, 4), (1000, 6, 3)])
def test_ulysses_head_slices_equal_unsharded(b2a, S, H, P):
    q, k, v = W.qkv(S, H, 128, seed=S + H)
    qd, kd, vd = dev(q), dev(k), dev(v)
    full, full_lse = b2a.attn_fwd(qd, kd, vd)
    out = torch.zeros_like(full)
    lse = torch.empty_like(full_lse)
    hp = H // P
    for r in range(P):
        hs = slice(r * hp, (r + 1) * hp)
        # views into the [S, H, d] tensors: row stride H*d, hp heads
        o_r, l_r = b2a.attn_fwd(qd[:, hs], kd[:, hs], vd[:, hs], out=out[:, hs])
        lse[hs] = l_r
    b2a.check_status()
    assert torch.equal(out, full)
    assert torch.equal(lse, full_lse)


def test_gathered_kv_workload_rank_sampled(b2a):
    # rank 3 of 8 on the 32k, Q ~ N(0, 4^2) workload: 4096 query rows x 32768 keys
    w = W.SEQ32K
    q, k, v = W.workload_qkv(w)
    lo, hi = b2a.chunk_bounds(w.S, 8)[3]
    qr = np.ascontiguousarray(q[lo:hi])
    rows = [W.sample_rows(hi - lo, 1, h, seed=w.seed) for h in range(w.H)]
    ref, ref_lse = OA.attention(qr, k, v, w.scale, rows=rows)
    out, lse = b2a.attn_fwd_gathered_kv(dev(qr), dev(k), dev(v), scale=w.scale)
    b2a.check_status()
    oh, lh = host(out), host(lse)
    got = np.stack([oh[rows[h], h, :] for h in range(w.H)], axis=1).astype(np.float64)
    got_lse = np.stack([lh[h, rows[h]] for h in range(w.H)]).astype(np.float64)
    assert_out_close(got, ref, "32k gathered-kv rank 3/8 sampled")
    assert_lse_close(got_lse, ref_lse)


# ------------------------------------------------- (S, B, hidden) layout --

@pytest.mark.parametrize("S,B,H,d", [(700, 3, 2, 128), (300, 2, 3, 64), (1, 4, 1, 128)])
def test_batched_layout(b2a, S, B, H, d):
    rng = np.random.default_rng(S + B)
    q, k, v = (rng.standard_normal((S, B, H, d), dtype=np.float32).astype(np.float16) for _ in range(3))
    scale = 1 / math.sqrt(d)
    out, lse = b2a.attn_fwd_batched(dev(q), dev(k), dev(v), scale=scale)
    b2a.check_status()
    oh, lh = host(out), host(lse)
    for b in range(B):
        ref, ref_lse = OA.attention(q[:, b], k[:, b], v[:, b], scale)
        assert_out_close(oh[:, b].astype(np.float64), ref, f"batch {b} of {B}")
        assert_lse_close(lh[b], ref_lse)
    # each batch equals a contiguous single-batch call bit for bit
    o1, l1 = b2a.attn_fwd(dev(np.ascontiguousarray(q[:, B - 1])), dev(np.ascontiguousarray(k[:, B - 1])),
                          dev(np.ascontiguousarray(v[:, B - 1])), scale=scale)
    b2a.check_status()
    np.testing.assert_array_equal(oh[:, B - 1], host(o1))
    np.testing.assert_array_equal(lh[B - 1], host(l1))


def test_sample_default_seq56320_sampled(b2a):
    w = W.SEQ56K
    q, k, v = W.workload_qkv(w)
    rows = [W.sample_rows(w.S, 1, h, seed=w.seed) for h in range(w.H)]
    ref, ref_lse = OA.attention(q, k, v, w.scale, rows=rows)
    out, lse = b2a.attn_fwd(dev(q), dev(k), dev(v), scale=w.scale)
    b2a.check_status()
    oh, lh = host(out), host(lse)
    got = np.stack([oh[rows[h], h, :] for h in range(w.H)], axis=1).astype(np.float64)
    got_lse = np.stack([lh[h, rows[h]] for h in range(w.H)]).astype(np.float64)
    assert_out_close(got, ref, "s56320 sampled")
    assert_lse_close(got_lse, ref_lse)
