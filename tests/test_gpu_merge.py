"""CUDA LSE merge against the FP64 oracle merge on random partials."""
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
    return m


@pytest.mark.parametrize("P,S,H,d,empty", [
    (1, 64, 2, 64, ()), (2, 300, 3, 128, ()), (3, 257, 1, 64, (1,)), (8, 1000, 4, 128, (0, 7)),
    (5, 33, 32, 128, (0, 1, 2, 3)), (64, 40, 2, 64, (10,)),
])
def test_merge_random_partials(b2a, P, S, H, d, empty):
    o, lse = W.merge_operands(P, S, H, d, seed=P * 1000 + S, empty_chunks=empty)
    ref, ref_lse = OC.merge(o, lse)
    out, lse_out = b2a.attn_merge(torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda())
    b2a.check_status()
    assert_out_close(out.cpu().numpy().astype(np.float64), ref, "merge out")
    assert_lse_close(lse_out.cpu().numpy(), ref_lse)


def test_merge_all_empty_rows(b2a):
    o, lse = W.merge_operands(3, 20, 2, 64, seed=3, empty_chunks=(0, 1, 2))
    out, lse_out = b2a.attn_merge(torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda())
    b2a.check_status()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse_out))


def test_merge_full_size_sampled(b2a):
    # the S=32768, P=8 merge of the ring-emulation workload, checked on rows
    P, S, H, d = 8, 32768, 32, 128
    o, lse = W.merge_operands(P, S, H, d, seed=21)
    out, lse_out = b2a.attn_merge(torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda())
    b2a.check_status()
    rows = W.sample_rows(S, P, 0, seed=21)
    ref, ref_lse = OC.merge(o[:, rows], lse[:, :, rows])
    assert_out_close(out.cpu().numpy()[rows].astype(np.float64), ref, "merge 32k sampled")
    assert_lse_close(lse_out.cpu().numpy()[:, rows], ref_lse)


@pytest.mark.parametrize("P,dtype", [(5, "f32"), (9, "f32"), (9, "f16")])
def test_merge_many_pair_groups_per_block(b2a, P, dtype):
    # 155400 (row, head) pairs = 607 groups of 256, the last one partial (8
    # pairs): every block of the persistent merge (two per SM) walks two or
    # three groups with its weights double-buffered across them, and P = 9
    # streams its chunks in two batches; all pairs against the oracle
    S, H, d = 4200, 37, 64
    o, lse = W.merge_operands(P, S, H, d, seed=P + 77, empty_chunks=(1,))
    if dtype == "f16":
        o = o.astype(np.float16)
        out, lse_out = b2a.attn_merge_f16(torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda())
    else:
        out, lse_out = b2a.attn_merge(torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda())
    b2a.check_status()
    ref, ref_lse = OC.merge(o, lse)
    assert_out_close(out.cpu().numpy().astype(np.float64), ref, f"merge {dtype} P={P}, 607 pair groups")
    assert_lse_close(lse_out.cpu().numpy(), ref_lse)
