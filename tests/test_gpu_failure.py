"""Failure detection on the GPU without a fault.

Every wait in the kernels is bounded; one that runs out sets a device status
word and its kernel returns, so the context stays usable.  The self-test
kernel makes such a wait run out on purpose (a barrier that nothing arrives
on) with a 50 ms limit; the host must then see B2A_ERR_TIMEOUT exactly once,
and work launched after the status is read must run normally.
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


def test_expired_wait_is_reported_once_and_context_survives(b2a):
    b2a.check_status()   # start clean
    result = b2a.selftest_wait_timeout(50)
    with pytest.raises(b2a.B2AError) as exc:
        b2a.check_status()
    assert exc.value.status == 4  # B2A_ERR_TIMEOUT
    assert result.cpu().tolist() == [1, 1]
    b2a.check_status()   # cleared by the read above
    # the context is usable: an attention call afterwards matches the oracle
    q, k, v = W.qkv(300, 2, 128, seed=40)
    out, lse = b2a.attn_fwd(torch.from_numpy(q).cuda(), torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    b2a.check_status()
    ref, ref_lse = OA.attention(q, k, v, 1 / math.sqrt(128))
    assert_out_close(out.cpu().numpy().astype(np.float64), ref, "after timeout")
    assert_lse_close(lse.cpu().numpy(), ref_lse)


def test_selftest_rejects_bad_limits(b2a):
    for ms in (0, -5, 2001):
        with pytest.raises(b2a.B2AError):
            b2a.selftest_wait_timeout(ms)
