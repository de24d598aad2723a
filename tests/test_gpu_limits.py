"""CUDA path at the edges of its size limits, against the FP64 oracle.

* 65535 heads, the largest grid.y a launch takes (the host rejects 65536),
  at short sequence lengths (one partial tile and a ragged second one),
  compared on 16 heads at each end.
* A 131072-token sequence (four times the pages' longest), compared on
  sampled rows per head including both ends.
* The largest chunk count the merge takes (P = 64) through the one-launch
  partials and the merge.
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from parity import assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def b2a():
    import long_context_bidirectional_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


@pytest.mark.parametrize("S,d", [(1, 64), (3, 64), (130, 128)])
def test_largest_head_count(b2a, S, d):
    # Heads are independent: the compared heads (16 at each end) hold the
    # seeded workload inputs, the other 65503 seeded device-side filler.
    H = 65535
    heads = np.r_[0:16, H - 16:H]
    q, k, v = W.qkv(S, len(heads), d, seed=S + d, q_sigma=2.0)
    g = torch.Generator(device="cuda").manual_seed(S + d)
    qd, kd, vd = (torch.randn((S, H, d), generator=g, device="cuda").half() for _ in range(3))
    idx = torch.from_numpy(heads).cuda()
    for t, x in ((qd, q), (kd, k), (vd, v)):
        t[:, idx] = dev(x)
    scale = 1 / math.sqrt(d)
    out, lse = b2a.attn_fwd(qd, kd, vd, scale=scale)
    b2a.check_status()
    ref, ref_lse = OA.attention(q, k, v, scale)
    assert_out_close(out[:, idx].cpu().numpy().astype(np.float64), ref, f"H=65535 S={S} d={d}")
    assert_lse_close(lse[idx].cpu().numpy(), ref_lse)


def test_head_count_past_the_grid_limit_is_refused(b2a):
    q = torch.zeros((1, 65536, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(b2a.B2AError):
        b2a.attn_fwd(q, q, q)


def test_sequence_of_131072_tokens_sampled(b2a):
    S, H, d = 131072, 4, 128
    q, k, v = W.qkv(S, H, d, seed=5)
    scale = 1 / math.sqrt(d)
    out, lse = b2a.attn_fwd(dev(q), dev(k), dev(v), scale=scale)
    b2a.check_status()
    rows = [W.sample_rows(S, 1, h, seed=5, n=128) for h in range(H)]
    ref, ref_lse = OA.attention(q, k, v, scale, rows=rows)
    oh, lh = out.cpu().numpy(), lse.cpu().numpy()
    got = np.stack([oh[rows[h], h] for h in range(H)], axis=1).astype(np.float64)
    got_lse = np.stack([lh[h, rows[h]] for h in range(H)], axis=0)
    assert_out_close(got, ref, "S=131072 sampled")
    assert_lse_close(got_lse, ref_lse)


def test_largest_chunk_count_partials_and_merge(b2a):
    S, H, d, P = 4096, 2, 128, 64   # 64 chunks of 64 keys
    q, k, v = W.qkv(S, H, d, seed=64)
    scale = 1 / math.sqrt(d)
    out, lse = b2a.attn_chunked(dev(q), dev(k), dev(v), P, scale=scale)
    b2a.check_status()
    ref, ref_lse = OA.attention(q, k, v, scale)
    assert_out_close(out.cpu().numpy().astype(np.float64), ref, "P=64 partials + merge")
    assert_lse_close(lse.cpu().numpy(), ref_lse)
