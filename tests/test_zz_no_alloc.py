"""attn_block_fwd_static: the self-attention block for callers that cannot
allocate device memory (their intermediates live in the library's static
device array).  Called through the C ABI and compared with attn_block_fwd,
which takes caller workspaces, on two calls in a row with different inputs.

This file is collected last on purpose: if it fails, a run that stops at
the first failure has already run every other test.
"""
import math

import numpy as np
import pytest
import torch

from parity import assert_out_close

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


def test_static_scratch_block_rejects_sizes_beyond_its_array(b2a):
    # 8*S*H*d bytes of intermediates must fit in 64 MiB: S*H*d <= 8388608
    H, d = 32, 128
    S = 8388608 // (H * d) + 1
    st = b2a.lib.attn_block_fwd_static(0x10000, 0x10000, 0x10000, 0x10000, S, H, d, 0.1, None)
    assert st == 2  # B2A_ERR_UNSUPPORTED, nothing enqueued
