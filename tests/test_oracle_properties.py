"""Property checks of the FP64 oracle over random small shapes (CPU).

For any shape, chunk count (empty chunks and more chunks than keys
included) and scale: the exact merge of the chunk partials is monolithic
attention; folding the chunks in with the two-term ring step, in any order,
reaches the same result; the fp16-stored partials move the merge by at most
half an fp16 ulp of the partials; and the output lies in the convex hull of
the value rows (softmax weights are a probability vector).
"""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import attention as A
from oracle import chunked as C


shapes = st.tuples(st.integers(1, 12), st.integers(0, 40), st.integers(1, 3), st.integers(1, 8),
                   st.integers(1, 45), st.floats(0.05, 2.0), st.integers(0, 2 ** 31 - 1))


def make(S, Skv, H, d, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((S, H, d)) * 2.0
    k = rng.standard_normal((Skv, H, d))
    v = rng.standard_normal((Skv, H, d))
    return q, k, v


@settings(max_examples=60, deadline=None)
@given(shapes)
def test_merge_of_partials_is_attention(args):
    S, Skv, H, d, P, scale, seed = args
    q, k, v = make(S, Skv, H, d, seed)
    o, lse = A.attention(q, k, v, scale)
    op, lp = C.partials(q, k, v, scale, P)
    om, lm = C.merge(op, lp)
    if Skv == 0:
        assert np.all(om == 0) and np.all(np.isneginf(lm))
        return
    np.testing.assert_allclose(om, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lm, lse, rtol=0, atol=1e-12)


@settings(max_examples=40, deadline=None)
@given(shapes, st.randoms(use_true_random=False))
def test_ring_steps_in_any_order_equal_the_merge(args, rnd):
    S, Skv, H, d, P, scale, seed = args
    q, k, v = make(S, Skv, H, d, seed)
    op, lp = C.partials(q, k, v, scale, P)
    om, lm = C.merge(op, lp)
    order = list(range(P))
    rnd.shuffle(order)
    acc = (np.full((S, H, d), np.nan), np.full((H, S), -np.inf))   # unseen rows: o ignored
    for c in order:
        acc = C.accumulate(*acc, op[c], lp[c])
    seen = ~np.isneginf(lm)
    np.testing.assert_array_equal(np.isneginf(acc[1]), ~seen)
    np.testing.assert_allclose(acc[1][seen], lm[seen], rtol=0, atol=1e-12)
    np.testing.assert_allclose(acc[0], om, rtol=0, atol=1e-12)


@settings(max_examples=40, deadline=None)
@given(shapes)
def test_fp16_partials_stay_within_half_an_ulp(args):
    S, Skv, H, d, P, scale, seed = args
    q, k, v = make(S, Skv, H, d, seed)
    op, lp = C.partials(q, k, v, scale, P)
    exact, _ = C.merge(op, lp)
    o16 = C.fp16_partials(op)
    got, _ = C.merge(o16, lp)
    bound = (np.spacing(np.abs(o16).astype(np.float16)).astype(np.float64) / 2).max(axis=0)
    assert np.all(np.abs(got - exact) <= bound * (1 + 1e-9) + 1e-15)


@settings(max_examples=40, deadline=None)
@given(shapes)
def test_output_lies_in_the_hull_of_the_values(args):
    S, Skv, H, d, _, scale, seed = args
    if Skv == 0:
        return
    q, k, v = make(S, Skv, H, d, seed)
    o, lse = A.attention(q, k, v, scale)
    lo = v.min(axis=0)[None]                      # per head and column
    hi = v.max(axis=0)[None]
    assert np.all(o >= lo - 1e-12) and np.all(o <= hi + 1e-12)
    # lse between the largest logit and that plus ln(Skv)
    s = np.einsum("shd,khd->hsk", q, k) * scale
    mx = s.max(axis=2)
    assert np.all(lse >= mx - 1e-12) and np.all(lse <= mx + np.log(Skv) + 1e-12)
