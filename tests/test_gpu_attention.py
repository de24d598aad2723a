"""CUDA attention (monolithic, partial + merge) against the FP64 oracle.

Small and ragged shapes compare every element; the full-size workloads
compare 256 sampled query rows per head (all d outputs plus the LSE) and,
for the chunked form, every element against the CUDA monolithic result (the
pages' sharded-vs-unsharded check, "TensorRT Multi-Device (multi-GPU)
support", Validation).
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


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def host(t):
    return t.detach().cpu().numpy()


def run_mono(b2a, q, k, v, scale):
    out, lse = b2a.attn_fwd(dev(q), dev(k), dev(v), scale=scale)
    b2a.check_status()
    return host(out).astype(np.float64), host(lse).astype(np.float64)


def run_chunked(b2a, q, k, v, scale, P, partial_dtype=torch.float32):
    out, lse = b2a.attn_chunked(dev(q), dev(k), dev(v), P, scale=scale, partial_dtype=partial_dtype)
    b2a.check_status()
    return host(out).astype(np.float64), host(lse).astype(np.float64)


# ------------------------------------------------------------ small / ragged --

SHAPES = [
    (1, 1, 64), (3, 2, 64), (64, 1, 128), (127, 2, 128), (128, 1, 64), (129, 2, 128),
    (255, 1, 64), (256, 2, 64), (257, 3, 128), (384, 2, 128), (1000, 2, 64), (1000, 1, 128),
]


@pytest.mark.parametrize("S,H,d", SHAPES)
def test_monolithic_small_and_ragged(b2a, S, H, d):
    q, k, v = W.qkv(S, H, d, seed=S + 7 * H + d)
    scale = 1 / math.sqrt(d)
    out, lse = run_mono(b2a, q, k, v, scale)
    ref, ref_lse = OA.attention(q, k, v, scale)
    assert_out_close(out, ref, f"out S={S} H={H} d={d}")
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("S,H,d,P", [(256, 2, 64, 2), (1000, 2, 128, 3), (129, 1, 64, 7),
                                     (5, 2, 128, 8), (700, 2, 128, 1)])
def test_chunked_small_and_ragged(b2a, S, H, d, P):
    q, k, v = W.qkv(S, H, d, seed=100 + S + P)
    scale = 1 / math.sqrt(d)
    out, lse = run_chunked(b2a, q, k, v, scale, P)
    ref, ref_lse = OA.attention(q, k, v, scale)
    assert_out_close(out, ref, f"chunked out S={S} P={P}")
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("d", [64, 128])
def test_peaked_softmax_forces_rescales(b2a, d):
    # Q ~ N(0, 4^2): logits std ~4, the running max keeps growing past the
    # lazy-rescale threshold across key tiles.
    q, k, v = W.qkv(1500, 2, d, seed=5, q_sigma=4.0)
    scale = 1 / math.sqrt(d)
    out, lse = run_mono(b2a, q, k, v, scale)
    ref, ref_lse = OA.attention(q, k, v, scale)
    assert_out_close(out, ref, "peaked out")
    assert_lse_close(lse, ref_lse)
    # keys sorted by their logit with query row 0 of head 0: that row's running
    # max rises tile after tile, so it rescales repeatedly
    order = np.argsort(k[:, 0, :].astype(np.float64) @ q[0, 0, :].astype(np.float64))
    ks, vs = np.ascontiguousarray(k[order]), np.ascontiguousarray(v[order])
    out2, lse2 = run_mono(b2a, q, ks, vs, scale)
    ref2, ref_lse2 = OA.attention(q, ks, vs, scale)
    assert_out_close(out2, ref2, "rising-max out")
    assert_lse_close(lse2, ref_lse2)


@pytest.mark.parametrize("d", [64, 128])
def test_single_key_and_constant_values(b2a, d):
    q, k, v = W.qkv(300, 2, d, seed=9, Skv=1)
    o, l = b2a.attn_fwd_partial(dev(q), dev(k), dev(v), scale=0.125)
    b2a.check_status()
    np.testing.assert_allclose(host(o), np.repeat(v.astype(np.float32), 300, axis=0), atol=1e-6)
    s0 = 0.125 * np.einsum("ihe,he->hi", q.astype(np.float64), k[0].astype(np.float64))
    assert_lse_close(host(l), s0)
    # constant V rows -> output equals that row
    q, k, v = W.qkv(500, 2, 128, seed=10)
    v[:] = v[0:1]
    out, _ = run_mono(b2a, q, k, v, 1 / math.sqrt(128))
    assert_out_close(out, np.repeat(v[0:1].astype(np.float64), 500, axis=0), "constant v")


@pytest.mark.parametrize("Sq,Skv,d", [(200, 700, 128), (1000, 64, 128), (300, 1, 128), (130, 515, 64)])
def test_partial_query_and_key_counts_differ(b2a, Sq, Skv, d):
    # one rank's queries against a gathered (or a single ring step's) K/V
    q, k, v = W.qkv(Sq, 2, d, seed=Sq + Skv, Skv=Skv)
    scale = 1 / math.sqrt(d)
    o, l = b2a.attn_fwd_partial(dev(q), dev(k), dev(v), scale=scale)
    b2a.check_status()
    ref, ref_lse = OA.attention(q, k, v, scale)
    assert_out_close(host(o), ref, f"partial Sq={Sq} Skv={Skv}")
    assert_lse_close(host(l), ref_lse)


def test_empty_chunk_partial(b2a):
    q, _, _ = W.qkv(77, 2, 64, seed=11)
    qd = dev(q)
    o, l = b2a.attn_fwd_partial(qd, qd[:0], qd[:0], scale=0.1)
    b2a.check_status()
    assert torch.all(o == 0) and torch.all(torch.isneginf(l))


def test_strided_fused_qkv_views(b2a):
    S, H, d = 600, 2, 128
    h = H * d
    rng = np.random.default_rng(12)
    qkv = rng.standard_normal((S, 3 * h), dtype=np.float32).astype(np.float16)
    t = dev(qkv)
    q = t[:, 0:h].view(S, H, d)   # row stride 3h
    k = t[:, h:2 * h].view(S, H, d)
    v = t[:, 2 * h:3 * h].view(S, H, d)
    out_buf = torch.zeros((S, 2 * h), dtype=torch.float16, device="cuda")
    out_view = out_buf[:, h:].view(S, H, d)  # row stride 2h
    b2a.attn_fwd(q, k, v, out=out_view, scale=1 / math.sqrt(d))
    b2a.check_status()
    ref, _ = OA.attention(qkv[:, 0:h].reshape(S, H, d), qkv[:, h:2 * h].reshape(S, H, d),
                          qkv[:, 2 * h:].reshape(S, H, d), 1 / math.sqrt(d))
    assert_out_close(host(out_view).astype(np.float64), ref, "strided out")
    assert torch.all(out_buf[:, :h] == 0), "wrote outside the output view"


def test_repeat_calls_are_deterministic(b2a):
    q, k, v = W.qkv(700, 2, 128, seed=13)
    a, la = run_mono(b2a, q, k, v, 0.09)
    b, lb = run_mono(b2a, q, k, v, 0.09)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(la, lb)


# --------------------------------------------------------------- workloads --

def test_tiny_workload_full(b2a):
    w = W.TINY
    q, k, v = W.workload_qkv(w)
    ref, ref_lse = OA.attention(q, k, v, w.scale)
    out, lse = run_mono(b2a, q, k, v, w.scale)
    assert_out_close(out, ref, "tiny mono")
    assert_lse_close(lse, ref_lse)
    out2, lse2 = run_chunked(b2a, q, k, v, w.scale, w.P)
    assert_out_close(out2, ref, "tiny chunked")
    assert_lse_close(lse2, ref_lse)
    out3, lse3 = run_chunked(b2a, q, k, v, w.scale, w.P, torch.float16)
    assert_out_close(out3, ref, "tiny chunked, fp16 partials")
    assert_lse_close(lse3, ref_lse)


def test_seq8k_workload_full(b2a):
    w = W.SEQ8K
    q, k, v = W.workload_qkv(w)
    ref, ref_lse = OA.attention(q, k, v, w.scale)
    out, lse = run_mono(b2a, q, k, v, w.scale)
    assert_out_close(out, ref, "8k mono")
    assert_lse_close(lse, ref_lse)
    out2, lse2 = run_chunked(b2a, q, k, v, w.scale, w.P)
    assert_out_close(out2, ref, "8k chunked")
    assert_lse_close(lse2, ref_lse)
    out3, lse3 = run_chunked(b2a, q, k, v, w.scale, w.P, torch.float16)
    assert_out_close(out3, ref, "8k chunked, fp16 partials")
    assert_lse_close(lse3, ref_lse)


def _sampled_check(b2a, w, P):
    q, k, v = W.workload_qkv(w)
    rows = [W.sample_rows(w.S, max(P, 1), h, seed=w.seed) for h in range(w.H)]
    ref, ref_lse = OA.attention(q, k, v, w.scale, rows=rows)
    qd, kd, vd = dev(q), dev(k), dev(v)
    out, lse = b2a.attn_fwd(qd, kd, vd, scale=w.scale)
    b2a.check_status()
    out_h, lse_h = host(out), host(lse)
    got = np.stack([out_h[rows[h], h, :] for h in range(w.H)], axis=1).astype(np.float64)
    got_lse = np.stack([lse_h[h, rows[h]] for h in range(w.H)]).astype(np.float64)
    assert_out_close(got, ref, f"{w.name} mono sampled")
    assert_lse_close(got_lse, ref_lse)
    if P > 1:
        out2, lse2 = b2a.attn_chunked(qd, kd, vd, P, scale=w.scale)
        b2a.check_status()
        o2h, l2h = host(out2), host(lse2)
        got2 = np.stack([o2h[rows[h], h, :] for h in range(w.H)], axis=1).astype(np.float64)
        got2_lse = np.stack([l2h[h, rows[h]] for h in range(w.H)]).astype(np.float64)
        assert_out_close(got2, ref, f"{w.name} chunked sampled")
        assert_lse_close(got2_lse, ref_lse)
        # sharded vs unsharded on every element
        assert_out_close(o2h.astype(np.float64), out_h.astype(np.float64), f"{w.name} chunked vs mono")
        assert_lse_close(l2h, lse_h, f"{w.name} chunked vs mono lse")
        del out2, lse2
        # the FP16 split-reduction form
        out3, lse3 = b2a.attn_chunked(qd, kd, vd, P, scale=w.scale, partial_dtype=torch.float16)
        b2a.check_status()
        o3h, l3h = host(out3), host(lse3)
        got3 = np.stack([o3h[rows[h], h, :] for h in range(w.H)], axis=1).astype(np.float64)
        got3_lse = np.stack([l3h[h, rows[h]] for h in range(w.H)]).astype(np.float64)
        assert_out_close(got3, ref, f"{w.name} chunked fp16 partials sampled")
        assert_lse_close(got3_lse, ref_lse)
        assert_out_close(o3h.astype(np.float64), out_h.astype(np.float64), f"{w.name} fp16 partials vs mono")
        assert_lse_close(l3h, lse_h, f"{w.name} fp16 partials vs mono lse")


def test_seq32k_qsigma4_workload_sampled(b2a):
    _sampled_check(b2a, W.SEQ32K, W.SEQ32K.P)


def test_seq64k_workload_sampled(b2a):
    _sampled_check(b2a, W.SEQ64K, 1)


def test_seq8k_h64_workload_full(b2a):
    # hidden 8192 (64 heads x 128) at S=8192: every row of every head
    w = W.SEQ8K_H64
    q, k, v = W.workload_qkv(w)
    ref, ref_lse = OA.attention(q, k, v, w.scale)
    out, lse = run_mono(b2a, q, k, v, w.scale)
    assert_out_close(out, ref, "8k h64 mono")
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("S", [1000, 4500])
def test_host_entry_point_end_to_end(b2a, S):
    # S = 4500: the P = 1 path copies and computes the query rows in 4 blocks
    # (row-strided LSE copies), the chunked path copies each key chunk
    # while the previous chunk's partial runs
    H, d = 2, 128
    q, k, v = W.qkv(S, H, d, seed=14)
    scale = 1 / math.sqrt(d)
    ref, ref_lse = OA.attention(q, k, v, scale)
    for P in (1, 3, 8):
        ws = torch.empty(b2a.host_workspace_bytes(S, H, d, P), dtype=torch.uint8, device="cuda")
        qh, kh, vh = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
        out = torch.empty((S, H, d), dtype=torch.float16).pin_memory()
        lse = torch.empty((H, S), dtype=torch.float32).pin_memory()
        b2a.attn_fwd_host(qh, kh, vh, out, lse, ws, P=P, scale=scale)
        b2a.check_status()
        assert_out_close(out.numpy().astype(np.float64), ref, f"host S={S} P={P}")
        assert_lse_close(lse.numpy(), ref_lse)
    # two calls back to back on one stream, no sync between: the second's
    # copies must wait for the first's use of the shared workspace
    ws = torch.empty(b2a.host_workspace_bytes(S, H, d, 4), dtype=torch.uint8, device="cuda")
    outs = [torch.empty((S, H, d), dtype=torch.float16).pin_memory() for _ in range(2)]
    lses = [torch.empty((H, S), dtype=torch.float32).pin_memory() for _ in range(2)]
    q2 = q.copy()
    q2[:, 0] = q[:, 1]  # a different second call
    ref2, ref2_lse = OA.attention(q2, k, v, scale)
    kh, vh = torch.from_numpy(k).pin_memory(), torch.from_numpy(v).pin_memory()
    qhs = [torch.from_numpy(qq).pin_memory() for qq in (q, q2)]   # alive until the sync below
    for i, P in enumerate((1, 4)):
        b2a.attn_fwd_host(qhs[i], kh, vh, outs[i], lses[i], ws, P=P, scale=scale)
    b2a.check_status()
    assert_out_close(outs[0].numpy().astype(np.float64), ref, "host back-to-back 1")
    assert_out_close(outs[1].numpy().astype(np.float64), ref2, "host back-to-back 2")
    assert_lse_close(lses[1].numpy(), ref2_lse)
    # two streams, a workspace each, several rounds with no sync in between:
    # the calls share the library's copy streams and overlap each other
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    wss = [torch.empty(b2a.host_workspace_bytes(S, H, d, P), dtype=torch.uint8, device="cuda") for P in (1, 4)]
    for _ in range(3):
        for i, P in enumerate((1, 4)):
            b2a.attn_fwd_host(qhs[i], kh, vh, outs[i], lses[i], wss[i], P=P, scale=scale, stream=streams[i])
    torch.cuda.synchronize()
    b2a.check_status()
    assert_out_close(outs[0].numpy().astype(np.float64), ref, "host two streams 1")
    assert_lse_close(lses[0].numpy(), ref_lse)
    assert_out_close(outs[1].numpy().astype(np.float64), ref2, "host two streams 2")
    assert_lse_close(lses[1].numpy(), ref2_lse)
