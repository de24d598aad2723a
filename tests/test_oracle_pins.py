"""Pins for the FP64 oracle, checked against things other than itself.

Each test fixes the oracle to a closed form, an invariant of non-causal
softmax attention, a brute-force double loop, a library routine, or a
hand-derived golden case (``tests/golden/hand_attention.json``).  Together
they catch a dropped scale, a missing max-subtraction, a transposed operand,
a wrong log base, a sign error in the merge and a mis-split QKV.
"""
import json
import math
import os
import struct

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import chunked as C
from oracle import stack as ST
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_attention.json")


def rand_qkv(S, H, d, seed, Skv=None, sigma=1.0):
    rng = np.random.default_rng(seed)
    Skv = S if Skv is None else Skv
    q = rng.standard_normal((S, H, d)) * sigma
    k = rng.standard_normal((Skv, H, d))
    v = rng.standard_normal((Skv, H, d))
    return q, k, v


# ---------------------------------------------------------------- golden ----

def test_hand_derived_golden_cases():
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    assert len(cases) >= 4
    for c in cases:
        q = np.array(c["q"], dtype=np.float64)[:, None, :]
        k = np.array(c["k"], dtype=np.float64)[:, None, :]
        v = np.array(c["v"], dtype=np.float64)[:, None, :]
        out, lse = A.attention(q, k, v, c["scale"])
        np.testing.assert_allclose(out[:, 0, :], np.array(c["out"]), rtol=0, atol=1e-12,
                                   err_msg=c["name"])
        np.testing.assert_allclose(lse[0], np.array(c["lse"]), rtol=0, atol=1e-12,
                                   err_msg=c["name"])


# ------------------------------------------------------------ invariants ----

@pytest.mark.parametrize("d", [3, 64])
def test_constant_v_gives_that_row(d):
    q, k, _ = rand_qkv(37, 2, d, seed=1, sigma=3.0)
    v0 = np.random.default_rng(2).standard_normal((1, 2, d))
    v = np.repeat(v0, k.shape[0], axis=0)
    out, _ = A.attention(q, k, v, 1 / math.sqrt(d))
    np.testing.assert_allclose(out, np.repeat(v0, q.shape[0], axis=0), rtol=0, atol=1e-14)


def test_single_key_gives_v_and_its_logit():
    q, k, v = rand_qkv(11, 3, 8, seed=3, Skv=1)
    scale = 0.37
    out, lse = A.attention(q, k, v, scale)
    np.testing.assert_allclose(out, np.repeat(v, 11, axis=0), rtol=0, atol=1e-14)
    for h in range(3):
        s0 = scale * np.array([sum(q[i, h, e] * k[0, h, e] for e in range(8)) for i in range(11)])
        np.testing.assert_allclose(lse[h], s0, rtol=0, atol=1e-13)


def test_softmax_rows_sum_to_one_and_reproduce_output():
    q, k, v = rand_qkv(50, 2, 16, seed=4, sigma=4.0)
    out, _ = A.attention(q, k, v, 0.25)
    for h in range(2):
        p = A.probabilities(q, k, 0.25, h)
        assert np.all(p >= 0)
        np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
        np.testing.assert_allclose(p @ v[:, h, :], out[:, h, :], rtol=0, atol=1e-12)


def test_key_permutation_invariance_and_query_equivariance():
    q, k, v = rand_qkv(40, 2, 8, seed=5, Skv=33)
    out, lse = A.attention(q, k, v, 0.5)
    pk = np.random.default_rng(6).permutation(33)
    out2, lse2 = A.attention(q, k[pk], v[pk], 0.5)
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-12)
    pq = np.random.default_rng(7).permutation(40)
    out3, lse3 = A.attention(q[pq], k, v, 0.5)
    np.testing.assert_allclose(out3, out[pq], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse3, lse[:, pq], rtol=0, atol=1e-12)


def test_lse_bounds():
    q, k, v = rand_qkv(30, 2, 8, seed=8, Skv=45, sigma=5.0)
    scale = 0.3
    _, lse = A.attention(q, k, v, scale)
    for h in range(2):
        s = scale * np.einsum("ie,je->ij", q[:, h], k[:, h])
        mx = s.max(axis=1)
        assert np.all(lse[h] >= mx - 1e-12)
        assert np.all(lse[h] <= mx + math.log(45) + 1e-12)


def test_empty_key_set():
    q, k, v = rand_qkv(5, 2, 4, seed=9, Skv=0)
    out, lse = A.attention(q, k, v, 1.0)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_row_selection_matches_full():
    q, k, v = rand_qkv(64, 2, 8, seed=10)
    out, lse = A.attention(q, k, v, 0.4)
    rows = np.array([0, 5, 63, 17])
    o2, l2 = A.attention(q, k, v, 0.4, rows=rows)
    np.testing.assert_array_equal(o2, out[rows])
    np.testing.assert_array_equal(l2, lse[:, rows])
    per_head = [np.array([1, 2]), np.array([60, 3])]
    o3, l3 = A.attention(q, k, v, 0.4, rows=per_head)
    for h in range(2):
        np.testing.assert_array_equal(o3[:, h], out[per_head[h], h])
        np.testing.assert_array_equal(l3[h], lse[h, per_head[h]])


# ----------------------------------------------------------- brute force ----

def brute_force(q, k, v, scale):
    """Pure-Python double loop, no max subtraction (inputs keep logits small)."""
    S, H, d = q.shape
    Skv = k.shape[0]
    out = [[[0.0] * d for _ in range(H)] for _ in range(S)]
    lse = [[0.0] * S for _ in range(H)]
    for h in range(H):
        for i in range(S):
            w = []
            for j in range(Skv):
                dot = 0.0
                for e in range(d):
                    dot += float(q[i, h, e]) * float(k[j, h, e])
                w.append(math.exp(scale * dot))
            tot = sum(w)
            for e in range(d):
                out[i][h][e] = sum(w[j] * float(v[j, h, e]) for j in range(Skv)) / tot
            lse[h][i] = math.log(tot)
    return np.array(out), np.array(lse)


@pytest.mark.parametrize("S,Skv,H,d", [(1, 1, 1, 4), (7, 13, 2, 5), (64, 64, 1, 8), (16, 3, 2, 12)])
def test_brute_force_small(S, Skv, H, d):
    q, k, v = rand_qkv(S, H, d, seed=S * 100 + Skv, Skv=Skv)
    scale = 1 / math.sqrt(d)
    out, lse = A.attention(q, k, v, scale)
    bo, bl = brute_force(q, k, v, scale)
    np.testing.assert_allclose(out, bo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, bl, rtol=0, atol=1e-12)


def test_closed_forms_one_and_two_keys():
    rng = np.random.default_rng(11)
    q = rng.standard_normal((3, 1, 6))
    k = rng.standard_normal((2, 1, 6))
    v = rng.standard_normal((2, 1, 6))
    scale = 0.7
    # S_kv = 1: o = v_0
    o1, _ = A.attention(q, k[:1], v[:1], scale)
    np.testing.assert_allclose(o1[:, 0], np.repeat(v[:1, 0], 3, axis=0), atol=1e-15)
    # S_kv = 2: o = sigmoid(s1 - s2) v1 + sigmoid(s2 - s1) v2, lse = ln(e^s1 + e^s2)
    o2, l2 = A.attention(q, k, v, scale)
    for i in range(3):
        s1 = scale * float(np.dot(q[i, 0], k[0, 0]))
        s2 = scale * float(np.dot(q[i, 0], k[1, 0]))
        sig = 1.0 / (1.0 + math.exp(-(s1 - s2)))
        np.testing.assert_allclose(o2[i, 0], sig * v[0, 0] + (1 - sig) * v[1, 0], atol=1e-14)
        np.testing.assert_allclose(l2[0, i], max(s1, s2) + math.log1p(math.exp(-abs(s1 - s2))),
                                   atol=1e-14)


# -------------------------------------------------------- library routine ----

@pytest.mark.parametrize("S,H,d", [(256, 2, 64), (300, 3, 128), (2048, 1, 64)])
def test_matches_torch_sdpa_float64(S, H, d):
    q, k, v = W.qkv(S, H, d, seed=12)
    scale = 1 / math.sqrt(d)
    out, lse = A.attention(q, k, v, scale)
    tq = torch.from_numpy(q.astype(np.float64)).permute(1, 0, 2)[None]
    tk = torch.from_numpy(k.astype(np.float64)).permute(1, 0, 2)[None]
    tv = torch.from_numpy(v.astype(np.float64)).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale)
    np.testing.assert_allclose(out, ref[0].permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
    ref_lse = torch.logsumexp(scale * (tq[0] @ tk[0].transpose(1, 2)), dim=-1)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-12)


# --------------------------------------------------------- chunk + merge ----

@pytest.mark.parametrize("P", [1, 2, 3, 4, 7, 8, 61])
def test_chunked_equals_monolithic(P):
    q, k, v = rand_qkv(29, 2, 8, seed=13, Skv=61, sigma=4.0)
    out, lse = A.attention(q, k, v, 0.35)
    o2, l2 = C.chunked_attention(q, k, v, 0.35, P)
    np.testing.assert_allclose(o2, out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, lse, rtol=0, atol=1e-12)


def test_chunk_bounds_cover_keys_once():
    for S, P in [(10, 3), (7, 7), (3, 5), (32768, 8)]:
        b = C.chunk_bounds(S, P)
        assert b[0][0] == 0 and b[-1][1] == S
        assert all(b[i][1] == b[i + 1][0] for i in range(P - 1))
        assert all(hi >= lo for lo, hi in b)


def test_more_chunks_than_keys_leaves_empty_chunks_harmless():
    q, k, v = rand_qkv(6, 1, 4, seed=14, Skv=3)
    out, lse = A.attention(q, k, v, 1.0)
    o_parts, lse_parts = C.partials(q, k, v, 1.0, 5)
    assert np.isneginf(lse_parts).any()
    o2, l2 = C.merge(o_parts, lse_parts)
    np.testing.assert_allclose(o2, out, atol=1e-12)
    np.testing.assert_allclose(l2, lse, atol=1e-12)


def test_merge_closed_form_two_partials():
    rng = np.random.default_rng(15)
    o = rng.standard_normal((2, 4, 1, 3))
    lse = rng.standard_normal((2, 1, 4)) * 3
    om, lm = C.merge(o, lse)
    for s in range(4):
        a, b = lse[0, 0, s], lse[1, 0, s]
        np.testing.assert_allclose(lm[0, s], math.log(math.exp(a) + math.exp(b)), atol=1e-13)
        want = (math.exp(a) * o[0, s, 0] + math.exp(b) * o[1, s, 0]) / (math.exp(a) + math.exp(b))
        np.testing.assert_allclose(om[s, 0], want, atol=1e-13)


def test_merge_identities():
    rng = np.random.default_rng(16)
    o = rng.standard_normal((1, 5, 2, 3))
    lse = rng.standard_normal((1, 2, 5))
    om, lm = C.merge(o, lse)
    np.testing.assert_array_equal(om, o[0])
    np.testing.assert_allclose(lm, lse[0], atol=1e-15)
    # two identical partials: same output, lse + ln 2
    om2, lm2 = C.merge(np.concatenate([o, o]), np.concatenate([lse, lse]))
    np.testing.assert_allclose(om2, o[0], atol=1e-15)
    np.testing.assert_allclose(lm2, lse[0] + math.log(2), atol=1e-14)
    # an all-empty row stays empty
    lse_e = np.full((2, 2, 5), -np.inf)
    om3, lm3 = C.merge(np.zeros((2, 5, 2, 3)), lse_e)
    assert np.all(om3 == 0) and np.all(np.isneginf(lm3))


# ------------------------------------------------------------ ring step ----

def test_accumulate_hand_case():
    # lse 0 = ln 2 and ln 6: the new lse is ln 8, the weights 2/8 and 6/8
    o_acc = np.array([[[1.0, -2.0]]])              # [S=1, H=1, d=2]
    o_c = np.array([[[5.0, 4.0]]])
    o, lse = C.accumulate(o_acc, np.array([[math.log(2)]]), o_c, np.array([[math.log(6)]]))
    np.testing.assert_allclose(lse, [[math.log(8)]], atol=1e-15)
    np.testing.assert_allclose(o, [[[0.25 * 1 + 0.75 * 5, 0.25 * -2 + 0.75 * 4]]], atol=1e-15)


def test_accumulate_empty_sides():
    rng = np.random.default_rng(17)
    o_c = rng.standard_normal((3, 2, 4))
    lse_c = rng.standard_normal((2, 3))
    junk = np.full((3, 2, 4), np.nan)
    # nothing seen yet: the chunk's result, whatever o_acc holds
    o, lse = C.accumulate(junk, np.full((2, 3), -np.inf), o_c, lse_c)
    np.testing.assert_array_equal(o, o_c)
    np.testing.assert_array_equal(lse, lse_c)
    # an empty chunk leaves the running result alone
    o2, l2 = C.accumulate(o_c, lse_c, junk, np.full((2, 3), -np.inf))
    np.testing.assert_array_equal(o2, o_c)
    np.testing.assert_array_equal(l2, lse_c)
    # both empty: still empty
    o3, l3 = C.accumulate(junk, np.full((2, 3), -np.inf), junk, np.full((2, 3), -np.inf))
    assert np.all(np.isneginf(l3)) and np.all(o3 == 0)


@pytest.mark.parametrize("P", [1, 2, 3, 7, 61, 70])
def test_ring_steps_equal_monolithic(P):
    # includes more chunks than keys (empty steps)
    q, k, v = rand_qkv(23, 2, 8, seed=18, Skv=61, sigma=4.0)
    out, lse = A.attention(q, k, v, 0.35)
    o2, l2 = C.ring_attention(q, k, v, 0.35, P)
    np.testing.assert_allclose(o2, out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, lse, rtol=0, atol=1e-12)


def test_ring_step_order_does_not_matter():
    # non-causal: folding the chunks in any order reaches the same result
    q, k, v = rand_qkv(9, 1, 6, seed=19, Skv=40, sigma=3.0)
    o_parts, lse_parts = C.partials(q, k, v, 0.5, 5)
    fwd = (np.zeros((9, 1, 6)), np.full((1, 9), -np.inf))
    rev = (np.zeros((9, 1, 6)), np.full((1, 9), -np.inf))
    for p in range(5):
        fwd = C.accumulate(*fwd, o_parts[p], lse_parts[p])
        rev = C.accumulate(*rev, o_parts[4 - p], lse_parts[4 - p])
    np.testing.assert_allclose(fwd[0], rev[0], atol=1e-13)
    np.testing.assert_allclose(fwd[1], rev[1], atol=1e-13)
    om, lm = C.merge(o_parts, lse_parts)
    np.testing.assert_allclose(fwd[0], om, atol=1e-13)
    np.testing.assert_allclose(fwd[1], lm, atol=1e-13)


def test_fp16_partials_round_to_nearest_even():
    # fp16 spacing at 1 is 2^-10: 1 + 2^-11 is a tie and goes to the even
    # neighbour 1; 1 + 3*2^-11 ties between odd 1 + 2^-10 and even 1 + 2^-9;
    # below 2^-14 the spacing is 2^-24 (subnormals)
    got = C.fp16_partials(np.array([1 + 2 ** -11, 1 + 3 * 2 ** -11, -(1 + 2 ** -11), 3 * 2 ** -25, 0.1]))
    assert got.dtype == np.float16
    want = [1.0, 1 + 2 ** -9, -1.0, 2 ** -23, struct.unpack("<e", struct.pack("<e", 0.1))[0]]
    assert [float(x) for x in got] == want


def test_fp16_partials_single_chunk_is_the_rounded_output():
    # one chunk has weight exactly 1: the merge returns the stored fp16 values
    q, k, v = rand_qkv(7, 2, 8, seed=31, Skv=23, sigma=2.0)
    o_parts, lse_parts = C.partials(q, k, v, 0.4, 1)
    o16 = C.fp16_partials(o_parts)
    om, lm = C.merge(o16, lse_parts)
    np.testing.assert_array_equal(om, o16[0].astype(np.float64))
    np.testing.assert_array_equal(lm, lse_parts[0])


def test_fp16_partials_error_within_half_ulp_of_the_partials():
    # the merge weights are >= 0 and sum to 1, so rounding each partial by at
    # most half an fp16 ulp moves the merged value by at most the largest
    # such half ulp among the chunks; the lse does not change at all
    q, k, v = rand_qkv(40, 3, 16, seed=37, Skv=90, sigma=3.0)
    o_parts, lse_parts = C.partials(q, k, v, 0.25, 6)
    exact, lse_e = C.merge(o_parts, lse_parts)
    o16 = C.fp16_partials(o_parts)
    got, lse_g = C.merge(o16, lse_parts)
    half_ulp = np.spacing(np.abs(o16).astype(np.float16)).astype(np.float64) / 2
    bound = half_ulp.max(axis=0)
    err = np.abs(got - exact)
    assert np.all(err <= bound * (1 + 1e-9) + 1e-15)
    assert err.max() > 0                       # the rounding did happen
    np.testing.assert_array_equal(lse_g, lse_e)
    # fp16-exact partials merge exactly as the fp64 merge does
    np.testing.assert_array_equal(C.merge(o16.astype(np.float64), lse_parts)[0], got)


# ----------------------------------------------------------------- stack ----

def test_rmsnorm_closed_forms():
    # a constant vector c*1: mean square c^2, so with eps = 0 the result is sign(c) * g
    g = np.array([0.5, -2.0, 3.0, 1.0])
    np.testing.assert_allclose(ST.rmsnorm(np.full(4, -3.0), g, 0.0), -g, atol=1e-15)
    # (3, 4) has mean square 12.5: y = (3, 4) / sqrt(12.5 + eps)
    y = ST.rmsnorm(np.array([3.0, 4.0]), np.ones(2), 0.5)
    np.testing.assert_allclose(y, np.array([3.0, 4.0]) / math.sqrt(13.0), atol=1e-15)
    # with eps = 0 and g = 1 every normalised vector has mean square 1,
    # and scaling the input by c > 0 changes nothing
    rng = np.random.default_rng(24)
    x = rng.standard_normal((5, 7, 16)) * 3
    yn = ST.rmsnorm(x, np.ones(16), 0.0)
    np.testing.assert_allclose(np.mean(yn * yn, axis=-1), 1.0, atol=1e-13)
    np.testing.assert_allclose(ST.rmsnorm(4.5 * x, np.ones(16), 0.0), yn, atol=1e-13)
    # eps shrinks the mean square to ms / (ms + eps)
    ms = np.mean(x * x, axis=-1)
    ye = ST.rmsnorm(x, np.ones(16), 0.25)
    np.testing.assert_allclose(np.mean(ye * ye, axis=-1), ms / (ms + 0.25), atol=1e-13)


def test_qkv_qknorm_against_python_loops():
    rng = np.random.default_rng(25)
    S, H, d, K = 3, 2, 4, 5
    x = rng.standard_normal((S, K)).astype(np.float16)
    w = rng.standard_normal((3 * H * d, K)).astype(np.float16)
    gq = rng.standard_normal(d).astype(np.float16)
    gk = rng.standard_normal(d).astype(np.float16)
    eps = 1e-3
    got = ST.qkv_qknorm(x, w, gq, gk, H, d, eps)
    h = H * d
    for s in range(S):
        row = [sum(float(x[s, c]) * float(w[n, c]) for c in range(K)) for n in range(3 * h)]
        for sec, g in ((0, gq), (1, gk)):
            for hh in range(H):
                seg = row[sec * h + hh * d: sec * h + (hh + 1) * d]
                r = math.sqrt(sum(t * t for t in seg) / d + eps)
                for e in range(d):
                    want = np.float16(seg[e] / r * float(g[e]))
                    assert got[s, sec * h + hh * d + e] == want
        for n in range(2 * h, 3 * h):   # v is left as projected
            assert got[s, n] == np.float16(row[n])


def test_round16_matches_ieee_half_from_struct():
    vals = [0.1, 1 / 3, 2049.0, 2051.0, 65504.0, -7.123456, 1e-5, 3.0e-8, 1.0 + 2 ** -11]
    got = ST.round16(np.array(vals))
    for x, g in zip(vals, got):
        want = struct.unpack("<e", struct.pack("<e", x))[0]
        assert float(g) == want, (x, float(g), want)


def test_linear_matches_python_dot_products():
    rng = np.random.default_rng(17)
    x = rng.standard_normal((9, 13)).astype(np.float16)
    w = rng.standard_normal((5, 13)).astype(np.float16)
    y = ST.linear(x, w)
    for i in range(9):
        for j in range(5):
            want = sum(float(x[i, e]) * float(w[j, e]) for e in range(13))
            assert abs(y[i, j] - want) < 1e-12


def _tiny_stack(S=24, H=2, d=4, seed=18):
    rng = np.random.default_rng(seed)
    h = H * d
    x = rng.standard_normal((S, h)).astype(np.float16)
    w_qkv = (rng.standard_normal((3 * h, h)) * 0.3).astype(np.float16)
    w_o = (rng.standard_normal((h, h)) * 0.3).astype(np.float16)
    return x, w_qkv, w_o, H, d


def test_block_zero_out_proj_is_identity():
    x, w_qkv, w_o, H, d = _tiny_stack()
    y, _, _ = ST.block(x, w_qkv, np.zeros_like(w_o), H, d, 0.5)
    np.testing.assert_array_equal(y, x)


def test_block_zero_key_weights_give_mean_of_values_and_split_order():
    x, w_qkv, w_o, H, d = _tiny_stack()
    h = H * d
    w = w_qkv.copy()
    w[h:2 * h] = 0                      # K = 0 -> every logit 0 -> uniform weights
    _, qkv, a = ST.block(x, w, w_o, H, d, 0.5)
    v = qkv[:, 2 * h:3 * h].astype(np.float64)
    want = ST.round16(np.repeat(v.mean(axis=0, keepdims=True), x.shape[0], axis=0))
    np.testing.assert_array_equal(a, want)
    # only head 1 has nonzero V columns -> head 0's output is exactly zero
    w2 = w.copy()
    w2[2 * h:2 * h + d] = 0
    _, _, a2 = ST.block(x, w2, w_o, H, d, 0.5)
    assert np.all(a2[:, :d] == 0) and np.any(a2[:, d:] != 0)


def test_block_identity_out_proj_adds_attention():
    x, w_qkv, _, H, d = _tiny_stack()
    h = H * d
    y, _, a = ST.block(x, w_qkv, np.eye(h, dtype=np.float16), H, d, 0.5)
    np.testing.assert_array_equal(y, ST.round16(x.astype(np.float64) + a.astype(np.float64)))


def test_block_rows_matches_full_block():
    x, w_qkv, w_o, H, d = _tiny_stack(S=40)
    y, qkv, a = ST.block(x, w_qkv, w_o, H, d, 0.5)
    rows = np.array([0, 7, 39, 20])
    y2, qkv2, a2 = ST.block_rows(x, w_qkv, w_o, H, d, 0.5, rows)
    np.testing.assert_array_equal(qkv2, qkv[rows])
    np.testing.assert_array_equal(a2, a[rows])
    np.testing.assert_array_equal(y2, y[rows])


def test_stack_chains_blocks():
    x, w_qkv, w_o, H, d = _tiny_stack()
    outs = ST.stack(x, [(w_qkv, w_o), (w_qkv, w_o)], H, d, 0.5)
    y1, _, _ = ST.block(x, w_qkv, w_o, H, d, 0.5)
    y2, _, _ = ST.block(y1, w_qkv, w_o, H, d, 0.5)
    np.testing.assert_array_equal(outs[1][0], y2)


# ------------------------------------------------------------ generators ----

def test_generators_are_seeded_and_shaped():
    q, k, v = W.qkv(16, 2, 8, seed=0, q_sigma=4.0)
    q2, k2, v2 = W.qkv(16, 2, 8, seed=0, q_sigma=4.0)
    assert q.dtype == np.float16 and q.shape == (16, 2, 8)
    np.testing.assert_array_equal(q, q2)
    np.testing.assert_array_equal(v, v2)
    assert 2.5 < float(np.std(q.astype(np.float64))) < 5.5
    rows = W.sample_rows(32768, 8, head=3)
    assert len(rows) == 256 and rows[0] == 0 and rows[-1] == 32767
    assert 4095 in rows and 4096 in rows and np.all(np.diff(rows) > 0)
