"""Property-based pins of the fp64 oracle (hypothesis, CPU): facts that hold for every shape
and input, checked on random small cases against a library routine (torch's
scaled_dot_product_attention in float64), a closed form, or the definition of the
selection rule. Shapes include no full video block, ragged video tails, no sinks, odd block
counts on the 128-query route and every ratio from one block to all of them."""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle.spark_oracle as orc
from block_sparse_video_mean_b200.inputs import make_qkv
from tests.test_oracle_pins import lse64, sdpa64

SETTINGS = dict(max_examples=25, deadline=None, suppress_health_check=[HealthCheck.too_slow])


def head(nv, ns, d, seed):
    Q, K, V = make_qkv(1, 1, nv, ns, d, seed=seed)
    return tuple(orc.to_f64(t[0, 0]) for t in (Q, K, V))


@settings(**SETTINGS)
@given(nb=st.integers(0, 5), tail=st.integers(0, 63), ns=st.integers(0, 20),
       d=st.sampled_from([8, 16, 32]), q_tile=st.sampled_from([64, 128]),
       seed=st.integers(0, 2**16))
def test_full_density_without_compression_is_dense_attention(nb, tail, ns, d, q_tile, seed):
    nv = nb * 64 + tail
    if nv + ns == 0:
        return
    q, k, v = head(nv, ns, d, seed)
    scale = 1.0 / np.sqrt(d)
    O, L, _ = orc.forward_head(q, k, v, ns, "topk", 1.0, compressed=False, q_tile=q_tile)
    np.testing.assert_allclose(O, sdpa64(q, k, v, scale), rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, lse64(q, k, scale), rtol=0, atol=1e-12)


@settings(**SETTINGS)
@given(n=st.integers(1, 40), data=st.data())
def test_topk_row_is_the_k_largest_with_ties_to_the_lower_index(n, data):
    # scores from a small integer set, so that ties are common
    s = np.array(data.draw(st.lists(st.integers(-3, 3), min_size=n, max_size=n)), dtype=np.float64)
    k = data.draw(st.integers(1, n))
    sel = orc.select_topk_row(s, k)
    assert len(sel) == k and np.all(np.diff(sel) > 0)
    rest = np.setdiff1d(np.arange(n), sel)
    for j in rest:
        for i in sel:
            # every kept score beats every dropped one, or ties it from a lower index
            assert s[i] > s[j] or (s[i] == s[j] and i < j)


@settings(**SETTINGS)
@given(n=st.integers(1, 40), data=st.data())
def test_topk_selections_are_nested_in_k(n, data):
    s = np.array(data.draw(st.lists(st.integers(-3, 3), min_size=n, max_size=n)), dtype=np.float64)
    k1 = data.draw(st.integers(1, n))
    k2 = data.draw(st.integers(k1, n))
    assert set(orc.select_topk_row(s, k1)) <= set(orc.select_topk_row(s, k2))


@settings(**SETTINGS)
@given(n=st.integers(1, 40), thr=st.floats(-3, 3), data=st.data())
def test_tau_row_keeps_exactly_the_scores_above_the_threshold(n, thr, data):
    s = np.array(data.draw(st.lists(st.floats(-3, 3), min_size=n, max_size=n)), dtype=np.float64)
    sel = orc.select_tau_row(s, thr)
    assert list(sel) == [j for j in range(n) if s[j] > thr]


@settings(**SETTINGS)
@given(nb=st.integers(1, 6), tail=st.integers(0, 63), ns=st.integers(0, 10),
       d=st.sampled_from([8, 16]), seed=st.integers(0, 2**16),
       sel=st.sampled_from([("topk", 0.2), ("topk", 0.5), ("tau", 0.5), ("tau", -0.5)]),
       q_tile=st.sampled_from([64, 128]))
def test_queries_equal_to_the_anchor_get_dense_attention(nb, tail, ns, d, seed, sel, q_tile):
    """The compressed entry of a block carries, for the anchor query, exactly the block's
    mass and mass-weighted value, so a query equal to the anchor (the mean of the full video
    blocks' queries) gets dense attention at any selection; the bias never falls below
    log 64 (Jensen)."""
    rng = np.random.default_rng(seed)
    nv = nb * 64
    a = rng.standard_normal(d)
    delta = rng.standard_normal((nv // 2, d)) * 1.3
    delta[::5] = 0.0                                   # some rows are exactly the anchor
    qv = np.concatenate([a + delta, a - delta])[rng.permutation(nv)]
    q = np.concatenate([qv, rng.standard_normal((tail + ns, d))])   # ragged tail, sinks
    N = nv + tail + ns
    k = rng.standard_normal((N, d)) + 0.5 * np.repeat(rng.standard_normal((N // 64 + 1, d)), 64, 0)[:N]
    v = rng.standard_normal((N, d))
    O, L, info = orc.forward_head(q, k, v, ns, sel[0], sel[1], compressed=True, q_tile=q_tile)
    P = info["pooled"]
    np.testing.assert_allclose(P.anchor, a, rtol=0, atol=1e-13)
    assert np.all(P.beta >= np.log(64.0) - 1e-12)
    scale = 1.0 / np.sqrt(d)
    rows = np.nonzero(np.all(np.abs(q[:nv] - a) < 1e-15, axis=1))[0]
    assert rows.size > 0
    np.testing.assert_allclose(O[rows], sdpa64(q, k, v, scale)[rows], rtol=0, atol=1e-11)
    np.testing.assert_allclose(L[rows], lse64(q, k, scale)[rows], rtol=0, atol=1e-11)


@settings(**SETTINGS)
@given(nb=st.integers(0, 9), q_tile=st.sampled_from([64, 128]))
def test_query_tiles_cover_the_video_rows_once_in_order(nb, q_tile):
    nt = orc.n_tiles(nb, q_tile)
    assert nt == (nb if q_tile == 64 else (nb + 1) // 2)
    rows = [orc.tile_rows(t, nb * 64, q_tile) for t in range(nt)]
    flat = np.concatenate(rows) if rows else np.zeros(0, dtype=np.int64)
    assert np.array_equal(flat, np.arange(nb * 64))
    assert all(len(r) == q_tile for r in rows[:-1])
