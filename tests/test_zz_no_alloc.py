"""attn_block_fwd_static: the self-attention block for callers that cannot
allocate device memory (their intermediates live in the library's static
device array).  Called through the C ABI and compared with attn_block_fwd,
which takes caller workspaces, on two calls in a row with different inputs;
and with the FP64 oracle's block, at a small size (all rows) and at the
largest size the array holds (sampled rows), where the attention output
ends on the array's last byte.

This file is collected last on purpose: if it fails, a run that stops at
the first failure has already run every other test.
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import stack as OS
from parity import MAX_ABS, REL_FRO, assert_out_close, fp16_ulp, metrics, record

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def b2a():
    import long_context_bidirectional_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _inputs(S, H, d, seed):
    g = torch.Generator().manual_seed(seed)
    h = H * d
    x = torch.randn(S, h, generator=g).half().cuda()
    w_qkv = (torch.randn(3 * h, h, generator=g) * 0.02).half().cuda()
    w_o = (torch.randn(h, h, generator=g) * 0.02).half().cuda()
    return x, w_qkv, w_o


def _static_block(b2a, x, w_qkv, w_o, H, d):
    S = x.shape[0]
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream().cuda_stream
    st = b2a.lib.attn_block_fwd_static(x.data_ptr(), w_qkv.data_ptr(), w_o.data_ptr(), y.data_ptr(),
                                       S, H, d, 1.0 / math.sqrt(d), stream)
    assert st == 0, b2a.lib.b2a_status_string(st)
    return y


def test_static_scratch_block_matches_workspace_block_twice(b2a):
    S, H, d = 1000, 16, 128
    for seed in (1, 2):                     # two calls in a row share the static array
        x, w_qkv, w_o = _inputs(S, H, d, seed)
        got = _static_block(b2a, x, w_qkv, w_o, H, d)
        want = b2a.attn_block_fwd(x, w_qkv, w_o, H, d, scale=1.0 / math.sqrt(d))
        b2a.check_status()
        assert_out_close(got.cpu().numpy().astype(np.float64), want.cpu().numpy().astype(np.float64),
                         f"static-scratch block, call with seed {seed}")


def _check_vs_oracle(got, ref, what):
    # both sides round at the same tensor boundaries: one fp16 ulp allowed
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    worst = float(np.max(np.abs(got - ref) / np.maximum(MAX_ABS, fp16_ulp(ref))))
    _, rf = metrics(got, ref)
    record(what, "elem_bound", worst, 1.0)
    record(what, "rel_fro", rf, REL_FRO)
    assert worst <= 1.0 and rf <= REL_FRO, f"{what}: worst {worst:.2f} of bound, rel_fro={rf:.3e}"


def test_static_scratch_block_matches_the_oracle(b2a):
    S, H, d = 1000, 4, 64
    x, w_qkv, w_o = _inputs(S, H, d, 3)
    got = _static_block(b2a, x, w_qkv, w_o, H, d)
    ry, _, _ = OS.block(x.cpu().numpy(), w_qkv.cpu().numpy(), w_o.cpu().numpy(), H, d, 1.0 / math.sqrt(d))
    _check_vs_oracle(got.cpu().numpy(), ry, "static-scratch block S=1000 vs oracle")


def test_static_scratch_block_at_its_size_limit(b2a):
    # S*H*d = 8388608: qkv fills the first 48 MiB, the attention output the
    # last 16 MiB of the 64 MiB array
    w = W.STACK6_S2048
    assert w.S * w.H * w.d == 8388608
    x16 = W.stack_x(w)
    w_qkv16, w_o16 = W.stack_weights(w, 0)
    x, w_qkv, w_o = (torch.from_numpy(t).cuda() for t in (x16, w_qkv16, w_o16))
    rows = W.sample_rows(w.S, 1, 0, seed=11)
    rows = np.unique(np.concatenate([rows, np.arange(w.S - 16, w.S)]))   # the array's last rows
    ry, _, _ = OS.block_rows(x16, w_qkv16, w_o16, w.H, w.d, w.scale, rows)
    for call in range(2):
        got = _static_block(b2a, x, w_qkv, w_o, w.H, w.d).cpu().numpy()
        _check_vs_oracle(got[rows], ry, f"static-scratch block at the limit, call {call + 1}")


def test_static_scratch_block_rejects_sizes_beyond_its_array(b2a):
    # 8*S*H*d bytes of intermediates must fit in 64 MiB: S*H*d <= 8388608
    H, d = 32, 128
    S = 8388608 // (H * d) + 1
    st = b2a.lib.attn_block_fwd_static(0x10000, 0x10000, 0x10000, 0x10000, S, H, d, 0.1, None)
    assert st == 2  # B2A_ERR_UNSUPPORTED, nothing enqueued
