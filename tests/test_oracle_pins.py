"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test checks the oracle against a library routine on a special case that reduces
to it (torch's scaled_dot_product_attention in float64), a closed form, an invariant
of the method, or a hand-derived fixture under tests/golden/. The mutation tests at
the end plant plausible mistakes in the oracle and check that a pin catches them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle.spark_oracle as orc
from block_sparse_video_mean_b200.inputs import make_qkv, random_orthogonal

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sdpa64(q, k, v, scale):
    """Dense softmax attention of every row, by torch's library routine in float64."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(a))[None, None] for a in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale)
    return o[0, 0].numpy()


def lse64(q, k, scale):
    return torch.logsumexp(torch.from_numpy(q @ k.T * scale), dim=1).numpy()


def head(nv, ns, d, seed=0, amp=0.5):
    Q, K, V = make_qkv(1, 1, nv, ns, d, seed=seed, amp=amp)
    return tuple(orc.to_f64(t[0, 0]) for t in (Q, K, V))


# ----------------------------------------------------------------- attention core

@pytest.mark.parametrize("nv,ns,d", [(256, 16, 64), (320, 0, 32), (256 + 37, 5, 64), (30, 8, 16)])
def test_full_density_no_compression_is_dense_attention(nv, ns, d):
    """Keep ratio 1.0 with the compressed branch off is dense softmax attention for every
    row (video, ragged tail and sink rows)."""
    q, k, v = head(nv, ns, d, seed=3)
    scale = 1 / math.sqrt(d)
    O, L, _ = orc.forward_head(q, k, v, ns, "topk", 1.0, compressed=False)
    np.testing.assert_allclose(O, sdpa64(q, k, v, scale), atol=1e-12, rtol=0)
    np.testing.assert_allclose(L, lse64(q, k, scale), atol=1e-12, rtol=0)


@pytest.mark.parametrize("mode,param", [("topk", 0.25), ("topk", 0.1), ("tau", 0.5)])
def test_constant_key_blocks_make_compression_exact(mode, param):
    """When every key of a video block is the same vector, the pooled entry with the
    log-mass bias carries exactly the block's attention mass and value, so the split
    forward equals dense attention at any density."""
    nv, ns, d = 512, 24, 64
    q, k, v = head(nv, ns, d, seed=5)
    kb = k[:nv].reshape(-1, 64, d)
    kb[:] = kb[:, :1, :]
    k[:nv] = kb.reshape(nv, d)
    O, L, info = orc.forward_head(q, k, v, ns, mode, param, compressed=True)
    scale = 1 / math.sqrt(d)
    np.testing.assert_allclose(O, sdpa64(q, k, v, scale), atol=1e-10, rtol=0)
    np.testing.assert_allclose(L, lse64(q, k, scale), atol=1e-10, rtol=0)
    pooled = info["pooled"]
    np.testing.assert_allclose(pooled.beta, math.log(64), atol=1e-12)
    np.testing.assert_allclose(pooled.vtil, v[:nv].reshape(-1, 64, d).mean(1), atol=1e-12)


def test_anchor_query_rows_are_exact():
    """A query equal to the anchor sees, through each compressed entry, exactly the mass
    and the mass-weighted value of the block it stands for; its output is the dense one
    at any density. The other rows must differ (the branch is an approximation)."""
    rng = np.random.default_rng(7)
    nv, ns, d = 640, 16, 32
    a = rng.standard_normal(d)
    delta = rng.standard_normal((nv // 2, d)) * 1.3
    delta[::9] = 0.0                                   # some rows are exactly the anchor
    q = np.concatenate([a + delta, a - delta])         # mean of the video rows is a
    q = q[rng.permutation(nv)]
    q = np.concatenate([q, rng.standard_normal((ns, d))])
    k = rng.standard_normal((nv + ns, d)) + 0.4 * np.repeat(rng.standard_normal((nv // 64 + 1, d)), 64, 0)[: nv + ns]
    v = rng.standard_normal((nv + ns, d))
    O, L, info = orc.forward_head(q, k, v, ns, "topk", 0.2, compressed=True)
    np.testing.assert_allclose(info["pooled"].anchor, a, atol=1e-13)
    scale = 1 / math.sqrt(d)
    ref = sdpa64(q, k, v, scale)
    lref = lse64(q, k, scale)
    rows = np.nonzero(np.all(np.abs(q[:nv] - a) < 1e-15, axis=1))[0]
    assert rows.size >= 8
    np.testing.assert_allclose(O[rows], ref[rows], atol=1e-11, rtol=0)
    np.testing.assert_allclose(L[rows], lref[rows], atol=1e-11, rtol=0)
    others = np.setdiff1d(np.arange(nv), rows)
    assert np.abs(O[others] - ref[others]).max() > 1e-3


def test_log_mass_identity_at_the_anchor():
    """exp(a . kbar_b * scale + beta_b) is the block's total anchor mass sum_j exp(s_j)."""
    q, k, v = head(1024, 32, 64, seed=11)
    scale = 0.125
    P = orc.pool_head(q, k, v, 32, scale)
    kb = k[:1024].reshape(16, 64, 64)
    mass = np.exp((kb @ q[:1024].mean(0)) * scale).sum(axis=1)
    np.testing.assert_allclose(np.exp(P.kbar @ P.anchor * scale + P.beta), mass, rtol=1e-13)
    # the bias is the Jensen gap plus log(64): never below log(64)
    assert np.all(P.beta >= math.log(64) - 1e-12)


def test_pooled_means_and_anchor():
    rng = np.random.default_rng(1)
    nb, d = 6, 16
    rows = rng.standard_normal((nb, d))
    q = np.repeat(rows, 64, axis=0)                    # every block holds one repeated query
    k = np.repeat(rows[::-1], 64, axis=0)
    P = orc.pool_head(q, k, q, 0)
    np.testing.assert_allclose(P.qbar, rows, atol=1e-14)
    np.testing.assert_allclose(P.kbar, rows[::-1], atol=1e-14)
    np.testing.assert_allclose(P.anchor, rows.mean(0), atol=1e-14)


@pytest.mark.parametrize("compressed", [True, False])
@pytest.mark.parametrize("pool_mode", ["reweight", "mean"])
def test_constant_values_give_constant_output(compressed, pool_mode):
    """Softmax weights sum to one over both branches, so V = c everywhere gives O = c."""
    q, k, v = head(384, 20, 32, seed=2)
    c = np.linspace(-1, 2, 32)
    v[:] = c
    O, _, _ = orc.forward_head(q, k, v, 20, "topk", 0.3, compressed=compressed, pool_mode=pool_mode)
    np.testing.assert_allclose(O, np.broadcast_to(c, O.shape), atol=1e-12)


def test_mean_pool_branch_closed_form():
    """Plain mean pooling: vtil = block mean of v, beta = log 64; with constant key
    blocks it is exact as well (Jensen's gap vanishes)."""
    q, k, v = head(256, 8, 32, seed=4)
    P = orc.pool_head(q, k, v, 8, mode="mean")
    np.testing.assert_allclose(P.vtil, v[:256].reshape(4, 64, 32).mean(1), atol=1e-14)
    np.testing.assert_allclose(P.beta, math.log(64), atol=0)


def test_empty_row_outputs_zero():
    """tau so high that nothing is kept, no sinks, no compressed branch: O = 0, LSE = -inf."""
    q, k, v = head(256, 0, 32, seed=6)
    O, L, info = orc.forward_head(q, k, v, 0, "tau", 50.0, compressed=False)
    assert all(len(s) == 0 for s in info["sel"])
    assert np.all(O == 0) and np.all(np.isneginf(L))


# ----------------------------------------------------------------- selection

def _golden_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


def test_topk_hand_derived_fixture():
    for ln in _golden_rows("topk_tiny.txt"):
        k, s, e = (p.strip() for p in ln.split("|"))
        got = orc.select_topk_row(np.array([float(x) for x in s.split(",")]), int(k))
        assert got.tolist() == [int(x) for x in e.split(",")], ln


def test_topk_count_fixture():
    for ln in _golden_rows("topk_count.txt"):
        r, nb, k = ln.split()
        assert orc.topk_count(float(r), int(nb)) == int(k), ln


def test_topk_selection_invariants():
    """Every kept score is >= every dropped one; equal scores are kept lowest index first."""
    rng = np.random.default_rng(0)
    for _ in range(50):
        nb = int(rng.integers(1, 90))
        s = np.round(rng.standard_normal(nb), 1)      # coarse rounding forces ties
        k = int(rng.integers(1, nb + 1))
        sel = orc.select_topk_row(s, k)
        assert len(sel) == k and np.all(np.diff(sel) > 0)
        drop = np.setdiff1d(np.arange(nb), sel)
        if drop.size:
            assert s[sel].min() >= s[drop].max()
            t = s[sel].min()
            if np.any(s[drop] == t):                   # a tie at the boundary
                assert np.nonzero(s == t)[0][: (s[sel] == t).sum()].tolist() == sel[s[sel] == t].tolist()


def test_tau_moments_closed_form():
    """mu = scale * (sum qbar) . (sum kbar) / nb^2 and E[S^2] = scale^2 tr(Mq Mk) / nb^2."""
    q, k, v = head(64 * 40, 0, 32, seed=9)
    scale = 1 / math.sqrt(32)
    P = orc.pool_head(q, k, v, 0, scale)
    S = orc.block_scores(P.qbar, P.kbar, scale)
    mu, sigma = orc.tau_stats(S)
    nb = P.qbar.shape[0]
    mu_cf = scale * P.qbar.sum(0) @ P.kbar.sum(0) / nb ** 2
    es2 = scale ** 2 * np.trace((P.qbar.T @ P.qbar) @ (P.kbar.T @ P.kbar)) / nb ** 2
    assert abs(mu - mu_cf) < 1e-13
    assert abs(sigma - math.sqrt(es2 - mu_cf ** 2)) < 1e-12


def test_tau_kept_fraction_matches_pages_and_gaussian_tail():
    """On block-correlated synthetic data the block scores are close to Gaussian, so
    tau = 1.0 / 1.5 / 2.0 keeps about the upper-tail mass; the pages quote ~16/7/2.7%."""
    Q, K, V = make_qkv(1, 2, 64 * 300, 0, 128, seed=0)
    fr = {}
    for h in range(2):
        q, k, v = (orc.to_f64(t[0, h]) for t in (Q, K, V))
        P = orc.pool_head(q, k, v, 0)
        S = orc.block_scores(P.qbar, P.kbar, 1 / math.sqrt(128))
        for ln in _golden_rows("tau_kept_fraction.txt"):
            tau, pages, tail = (float(x) for x in ln.split())
            kept = 100.0 * (S > orc.tau_threshold(S, tau)).mean()
            fr.setdefault(tau, []).append(kept)
            assert abs(kept - tail) < 1.0, (tau, kept, tail)
            assert abs(kept - pages) < 1.5, (tau, kept, pages)
    assert fr[1.0][0] > fr[1.5][0] > fr[2.0][0]


def test_topk_tau_scale_invariance():
    """Selections do not depend on the softmax scale (top-k) and on a common scaling of
    K (tau works in sigma units)."""
    q, k, v = head(64 * 30, 0, 32, seed=12)
    a = orc.forward_head(q, k, v, 0, "topk", 0.2, scale=0.1)[2]["sel"]
    b = orc.forward_head(q, k, v, 0, "topk", 0.2, scale=0.7)[2]["sel"]
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    c = orc.forward_head(q, k, v, 0, "tau", 1.2)[2]["sel"]
    d = orc.forward_head(q, 3.0 * k, v, 0, "tau", 1.2)[2]["sel"]
    assert all(np.array_equal(x, y) for x, y in zip(c, d))


# ----------------------------------------------------------------- Spark-Reblock

def _check_partition(perm, nv):
    assert sorted(perm.tolist()) == list(range(nv))
    leaves = perm.reshape(-1, 64)
    assert np.all(np.diff(leaves, axis=1) > 0)            # ascending inside a leaf
    assert np.all(np.diff(leaves[:, 0]) > 0)              # leaves by smallest index


@pytest.mark.parametrize("nb", [1, 2, 3, 5, 8, 13])
def test_reblock_leaves_are_exact_blocks(nb):
    q, k, v = head(64 * nb, 10, 32, seed=nb)
    rb = orc.reblock_head(q, k, 10)
    _check_partition(rb.perm, 64 * nb)
    assert rb.labels.shape[0] == orc.n_levels(nb) + 1
    _, counts = np.unique(rb.labels[-1], return_counts=True)
    assert np.all(counts == 64)


def _partition_sets(perm):
    return sorted(tuple(x) for x in perm.reshape(-1, 64).tolist())


def test_reblock_invariances():
    """The partition depends only on the Mahalanobis cosines q_i^T M q_j: unchanged when K
    is scaled, and when Q and K are rotated together by an orthogonal matrix."""
    q, k, v = head(64 * 12, 0, 32, seed=21)
    base = _partition_sets(orc.reblock_head(q, k, 0).perm)
    assert _partition_sets(orc.reblock_head(q, 3.7 * k, 0).perm) == base
    assert _partition_sets(orc.reblock_head(2.5 * q, k, 0).perm) == base
    R = random_orthogonal(32, 5).numpy()
    assert _partition_sets(orc.reblock_head(q @ R, k @ R, 0).perm) == base


def test_whitening_is_mahalanobis_cosine():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((50, 8))
    k = rng.standard_normal((400, 8)) @ rng.standard_normal((8, 8))
    M = orc.key_second_moment(k)
    x = orc.whiten(q, M)
    qMq = q @ M @ q.T
    nrm = np.sqrt(np.diag(qMq))
    np.testing.assert_allclose(x @ x.T, qMq / np.outer(nrm, nrm), atol=1e-12)


def test_reblock_two_clusters_split_first():
    """Two well separated groups of query directions go to different children at level 0."""
    rng = np.random.default_rng(8)
    d = 16
    e = np.eye(d)
    q = np.concatenate([e[0] + 0.05 * rng.standard_normal((192, d)),
                        e[1] + 0.05 * rng.standard_normal((192, d))])
    idx = rng.permutation(384)
    q = q[idx]
    k = rng.standard_normal((384, d))
    rb = orc.reblock_head(q, k, 0)
    groupA = set(np.nonzero(idx < 192)[0].tolist())
    left = set(np.nonzero(rb.labels[1] == 0)[0].tolist())
    assert left == groupA or left == set(range(384)) - groupA


def test_reblock_arc_hand_derived():
    """Queries on a short arc of a circle with an isotropic key second moment: the
    principal direction runs along the arc, so the leaves are the consecutive runs of
    64 angles, whatever the token order (hand-derived; no eigen solver involved)."""
    rng = np.random.default_rng(4)
    n, d = 512, 8
    theta = np.sort(rng.uniform(0.0, 0.6, n))
    q = np.zeros((n, d))
    q[:, 0], q[:, 1] = np.cos(theta), np.sin(theta)
    shuffle = rng.permutation(n)
    q = q[shuffle]
    Qo, _ = np.linalg.qr(rng.standard_normal((n, d)))
    k = Qo * math.sqrt(n)                                   # k^T k / n = I exactly
    rb = orc.reblock_head(q, k, 0)
    rank = np.argsort(np.argsort(theta[shuffle]))           # position of each token on the arc
    expect = sorted(tuple(sorted(np.nonzero(rank // 64 == g)[0].tolist())) for g in range(8))
    assert _partition_sets(rb.perm) == expect


def test_reblock_odd_node_sign_convention():
    """m = 3: the left child takes the 64 lowest projections, with the eigenvector
    signed so that the projections have a non-negative third central moment."""
    rng = np.random.default_rng(5)
    n, d = 192, 4
    t = np.concatenate([rng.uniform(-1, 0.3, 150), rng.uniform(2.0, 6.0, 42)])  # long + tail
    q = np.zeros((n, d))
    q[:, 0] = 1.0
    q[:, 1] = 0.05 * t
    q[:, 2:] = 1e-4 * rng.standard_normal((n, 2))
    k = np.eye(d)[np.arange(n) % d] * 2.0
    rb = orc.reblock_head(q, k, 0)
    sp = rb.splits[(0, 0)]
    assert sp.skew >= 0
    assert set(sp.left.tolist()) == set(np.argsort(t)[:64].tolist())


def test_reblock_m2_split_matches_svd():
    """For a two-block node the split is the median of the projection on the top right
    singular vector of the centred whitened data (numpy SVD, another routine than eigh)."""
    q, k, v = head(128, 0, 16, seed=30)
    rb = orc.reblock_head(q, k, 0)
    x = orc.whiten(q, orc.key_second_moment(k))
    _, _, Vt = np.linalg.svd(x - x.mean(0))
    p = x @ Vt[0]
    low = set(np.argsort(p)[:64].tolist())
    left = set(rb.splits[(0, 0)].left.tolist())
    assert left == low or left == set(range(128)) - low


def test_reblock_forward_outputs_in_original_order():
    """With reblocking at full density and no compression the forward is still dense
    attention, row for row in the original order."""
    q, k, v = head(64 * 6, 12, 32, seed=13)
    O, L, info = orc.forward_head(q, k, v, 12, "topk", 1.0, compressed=False, reblock=True)
    np.testing.assert_allclose(O, sdpa64(q, k, v, 1 / math.sqrt(32)), atol=1e-12)


# ----------------------------------------------------------------- planted mistakes

def test_planted_beta_sign_error_is_caught(monkeypatch):
    real = orc.pool_head

    def bad(*a, **kw):
        P = real(*a, **kw)
        P.beta = -P.beta
        return P
    monkeypatch.setattr(orc, "pool_head", bad)
    with pytest.raises(AssertionError):
        test_constant_key_blocks_make_compression_exact("topk", 0.25)


def test_planted_missing_scale_is_caught(monkeypatch):
    monkeypatch.setattr(orc, "default_scale", lambda d, s=None: 1.0)
    with pytest.raises(AssertionError):
        test_full_density_no_compression_is_dense_attention(256, 16, 64)


def test_planted_unweighted_summary_is_caught(monkeypatch):
    real = orc.pool_head

    def bad(q, k, v, n_sink, scale=None, block=64, mode="reweight", q_tile=64, *extra_args):
        P = real(q, k, v, n_sink, scale, block, mode, q_tile, *extra_args)
        nb = P.kbar.shape[0]
        P.vtil = v[: nb * block].reshape(nb, block, -1).mean(1)
        return P
    monkeypatch.setattr(orc, "pool_head", bad)
    with pytest.raises(AssertionError):
        test_anchor_query_rows_are_exact()


def test_planted_unsorted_split_is_caught(monkeypatch):
    """Splitting by token order instead of by projection must break the arc pin."""
    real = orc.split_node

    def bad(x, members, block=64):
        sp = real(x, members, block)
        members = np.sort(np.asarray(members))
        cut = len(sp.left)
        return orc.Split(members[:cut], members[cut:], sp.split_value, sp.proj, sp.gap, sp.skew)
    monkeypatch.setattr(orc, "split_node", bad)
    with pytest.raises(AssertionError):
        test_reblock_arc_hand_derived()


def test_planted_wrong_whitening_side_is_caught(monkeypatch):
    """Whitening with the queries' own second moment instead of the keys' must break the
    Mahalanobis-cosine pin."""
    monkeypatch.setattr(orc, "key_second_moment", lambda kv: np.eye(kv.shape[1]))
    with pytest.raises(AssertionError):
        test_whitening_is_mahalanobis_cosine_via_reblock()


def test_whitening_is_mahalanobis_cosine_via_reblock():
    """The partition of a node of two blocks equals the one computed from the
    Mahalanobis Gram matrix G_ij = q_i^T M q_j / (|q_i|_M |q_j|_M): the top eigenvector of
    the doubly centred G gives the same projections up to sign (kernel-PCA identity)."""
    rng = np.random.default_rng(31)
    d = 12
    q = rng.standard_normal((128, d)) * np.linspace(0.3, 3.0, d)
    k = rng.standard_normal((128, d)) @ rng.standard_normal((d, d))
    rb = orc.reblock_head(q, k, 0)
    M = k.T @ k / 128.0
    G = q @ M @ q.T
    nrm = np.sqrt(np.diag(G))
    G = G / np.outer(nrm, nrm)
    J = np.eye(128) - 1.0 / 128
    w, U = np.linalg.eigh(J @ G @ J)
    p = U[:, -1]
    low = set(np.argsort(p)[:64].tolist())
    left = set(rb.splits[(0, 0)].left.tolist())
    assert left == low or left == set(range(128)) - low


# --------------------------------------------------------------------------- branch fidelity
# [Spark-H3] "What Spark-Attn changes": the compressed branch stands in for the blocks the
# exact branch drops, and Spark-Reweight replaces the plain mean-pooled entry because
# mean pooling gives exp(E[x]) where the softmax needs E[exp(x)]. On seeded synthetic
# heads the oracle must order the three forwards by their distance to dense attention:
# no compressed branch > mean-pooled branch > reweighted branch.
@pytest.mark.parametrize("nv,ns,d,ratio,amp,seed,q_offset", [
    (64 * 48, 32, 64, 0.1, 0.5, 0, 0.0),
    (64 * 48, 32, 64, 0.2, 0.5, 1, 0.0),
    (64 * 48, 32, 64, 0.1, 1.0, 3, 0.0),
    (64 * 48, 32, 64, 0.1, 0.5, 5, 1.0),   # queries with a mean direction: beta far from log 64
    (64 * 48, 0, 128, 0.2, 0.5, 6, 1.0),
])
def test_compressed_branch_fidelity_ordering(nv, ns, d, ratio, amp, seed, q_offset):
    Q, K, V = make_qkv(1, 1, nv, ns, d, seed=seed, amp=amp, q_offset=q_offset)
    q, k, v = (orc.to_f64(t[0, 0]) for t in (Q, K, V))
    dense, _, _ = orc.forward_head(q, k, v, ns, "topk", 1.0, False)
    err = {}
    for name, comp, pm in (("none", False, "reweight"), ("mean", True, "mean"),
                           ("reweight", True, "reweight")):
        o, _, _ = orc.forward_head(q, k, v, ns, "topk", ratio, comp, pool_mode=pm)
        err[name] = np.linalg.norm(o[:nv] - dense[:nv]) / np.linalg.norm(dense[:nv])
    assert err["reweight"] < err["mean"] < err["none"], err


def test_offset_queries_move_beta_away_from_log64():
    """The query-offset input family exercises Spark-Reweight: with a mean query direction
    the anchor is long, the anchor scores inside a block spread, and the log-mass bias
    beta_b = lse_b - a . kbar_b * scale (>= log 64 by Jensen) departs from log 64 by O(1);
    without the offset it stays within a few hundredths of it."""
    for q_offset, lo, hi in ((0.0, 0.0, 0.05), (1.0, 0.2, 2.0)):
        Q, K, V = make_qkv(1, 1, 64 * 64, 16, 128, seed=8, q_offset=q_offset)
        q, k, v = (orc.to_f64(t[0, 0]) for t in (Q, K, V))
        P = orc.pool_head(q, k, v, 16, 1 / math.sqrt(128))
        excess = P.beta - math.log(64)
        assert np.all(excess >= -1e-12)
        assert lo <= float(excess.mean()) <= hi, (q_offset, float(excess.mean()))


# --------------------------------------------------------------------------- keys' own partition
def test_reblock_kv_full_density_is_dense_attention():
    """With the keys on a partition of their own (and the queries on theirs), density 1.0
    without the compressed branch is still dense softmax attention in the original order:
    K and V must follow one permutation and O must be scattered back by the queries'."""
    q, k, v = head(64 * 10, 24, 32, seed=31)
    scale = 1 / math.sqrt(32)
    O, L, info = orc.forward_head(q, k, v, 24, "topk", 1.0, compressed=False, reblock=True,
                                  reblock_kv=True)
    assert not np.array_equal(info["reblock"].perm, info["reblock_k"].perm)
    np.testing.assert_allclose(O, sdpa64(q, k, v, scale), atol=1e-12, rtol=0)
    np.testing.assert_allclose(L, lse64(q, k, scale), atol=1e-12, rtol=0)


def test_reblock_kv_partition_is_the_swapped_partition_and_invariant():
    """The keys' partition is the queries' construction with the roles swapped: leaves of 64
    keys, unchanged when Q is scaled and when Q and K are rotated together."""
    q, k, v = head(64 * 12, 0, 32, seed=22)
    _, _, info = orc.forward_head(q, k, v, 0, "topk", 0.5, reblock=True, reblock_kv=True)
    pk = info["reblock_k"].perm
    assert sorted(pk.tolist()) == list(range(64 * 12))
    base = _partition_sets(pk)
    assert _partition_sets(orc.reblock_head(k, 3.1 * q, 0).perm) == base
    R = random_orthogonal(32, 6).numpy()
    assert _partition_sets(orc.reblock_head(k @ R, q @ R, 0).perm) == base


# ----------------------------------------------------------------- 128-query x 64-key route

@pytest.mark.parametrize("nv,ns,d", [(448, 16, 64), (512 + 21, 7, 32)])
def test_q128_full_density_no_compression_is_dense_attention(nv, ns, d):
    """On the 128-query route (odd nb: the last tile holds one block; a ragged tail and
    sinks follow), keep ratio 1.0 without compression is dense attention for every row."""
    q, k, v = head(nv, ns, d, seed=11)
    scale = 1 / math.sqrt(d)
    O, L, info = orc.forward_head(q, k, v, ns, "topk", 1.0, compressed=False, q_tile=128)
    assert len(info["sel"]) == orc.n_tiles(nv // 64, 128)
    np.testing.assert_allclose(O, sdpa64(q, k, v, scale), atol=1e-12, rtol=0)
    np.testing.assert_allclose(L, lse64(q, k, scale), atol=1e-12, rtol=0)


def test_q128_tile_scores_are_means_of_block_scores():
    """Pooling is linear: a tile's score against key block j is the mean of its blocks'
    scores (the last tile of an odd nb is one block)."""
    nv, ns, d = 7 * 64, 8, 64
    q, k, v = head(nv, ns, d, seed=12)
    scale = 1 / math.sqrt(d)
    P64 = orc.pool_head(q, k, v, ns, scale)
    P128 = orc.pool_head(q, k, v, ns, scale, q_tile=128)
    S64 = orc.block_scores(P64.qbar, P64.kbar, scale)
    S128 = orc.block_scores(P128.qbar, P128.kbar, scale)
    assert S128.shape == (4, 7)
    want = np.stack([S64[0:2].mean(0), S64[2:4].mean(0), S64[4:6].mean(0), S64[6]])
    np.testing.assert_allclose(S128, want, atol=1e-13, rtol=0)
    np.testing.assert_array_equal(P128.kbar, P64.kbar)
    np.testing.assert_array_equal(P128.anchor, P64.anchor)


@pytest.mark.parametrize("mode,param,nb", [("topk", 0.2, 7), ("topk", 0.5, 6), ("tau", 0.5, 8)])
def test_q128_route_equals_block_route_when_block_pairs_repeat(mode, param, nb):
    """When the second block of every tile repeats the first one's queries, a tile pools to
    the same query as each of its blocks, selects the same key blocks and gives every row
    the output of the 64-query route (for tau, with nb even, the score moments agree too)."""
    ns, d = 12, 64
    q, k, v = head(nb * 64, ns, d, seed=13)
    for b in range(1, nb, 2):
        q[b * 64:(b + 1) * 64] = q[(b - 1) * 64:b * 64]
    O64, L64, i64 = orc.forward_head(q, k, v, ns, mode, param, compressed=True)
    O128, L128, i128 = orc.forward_head(q, k, v, ns, mode, param, compressed=True, q_tile=128)
    for t, sel in enumerate(i128["sel"]):
        np.testing.assert_array_equal(sel, i64["sel"][2 * t])
    np.testing.assert_allclose(O128, O64, atol=1e-12, rtol=0)
    np.testing.assert_allclose(L128, L64, atol=1e-12, rtol=0)


@pytest.mark.parametrize("mode,param", [("topk", 0.25), ("tau", 0.5)])
def test_q128_constant_key_blocks_make_compression_exact(mode, param):
    """The constant-key-block special case on the 128-query route: the pooled entries
    carry each unselected block exactly, so the forward is dense attention."""
    nv, ns, d = 5 * 64, 20, 64
    q, k, v = head(nv, ns, d, seed=14)
    kb = k[:nv].reshape(-1, 64, d)
    kb[:] = kb[:, :1, :]
    k[:nv] = kb.reshape(nv, d)
    O, L, info = orc.forward_head(q, k, v, ns, mode, param, compressed=True, q_tile=128)
    scale = 1 / math.sqrt(d)
    np.testing.assert_allclose(O, sdpa64(q, k, v, scale), atol=1e-10, rtol=0)
    np.testing.assert_allclose(L, lse64(q, k, scale), atol=1e-10, rtol=0)


def test_planted_end_aligned_last_tile_is_caught(monkeypatch):
    """A last tile aligned to the end of the video rows (overlapping the tile before it,
    instead of holding one block) breaks the linearity pin."""
    def end_aligned(t, nv, q_tile=64):
        hi = min((t + 1) * q_tile, nv)
        return np.arange(max(hi - q_tile, 0), hi)
    monkeypatch.setattr(orc, "tile_rows", end_aligned)
    with pytest.raises(AssertionError):
        test_q128_tile_scores_are_means_of_block_scores()


# --------------------------------------------------------------------------- extra tokens
# [Core-node] "Block-sparse attention: one node, three backends": extra_tokens adds the
# highest-scoring tokens beyond the selected blocks. Reading: a per-head budget of E tokens
# ranked by the anchor score s_j = a . k_j * scale (ties to the lower index); they join
# every video query's exact branch, and each compressed entry summarises only its block's
# remaining tokens (no entry when all 64 are extra).

def _anchor_head(nv=640, ns=16, d=32, seed=7):
    """Queries whose mean is a known anchor a, some rows exactly a (as in the anchor pin)."""
    rng = np.random.default_rng(seed)
    a = rng.standard_normal(d)
    delta = rng.standard_normal((nv // 2, d)) * 1.3
    delta[::9] = 0.0
    q = np.concatenate([a + delta, a - delta])
    q = q[rng.permutation(nv)]
    q = np.concatenate([q, rng.standard_normal((ns, d))])
    k = rng.standard_normal((nv + ns, d)) + 0.4 * np.repeat(rng.standard_normal((nv // 64 + 1, d)), 64, 0)[: nv + ns]
    v = rng.standard_normal((nv + ns, d))
    return q, k, v, a


@pytest.mark.parametrize("E,pool_mode", [(1, "reweight"), (37, "reweight"), (200, "reweight"),
                                         (64 * 3 + 5, "reweight"), (37, "mean")])
def test_extra_tokens_keep_anchor_rows_exact(E, pool_mode):
    """Mass bookkeeping: for a query equal to the anchor every entry of the reweighted
    branch carries exactly the mass and mass-weighted value of the tokens it stands for,
    and the extra tokens are exact, so anchor rows still get dense attention whatever
    tokens were taken out of the blocks (a recomputation over the wrong token set, or an
    extra token counted twice, breaks this). The mean-pool branch is not exact there;
    its entries must stand for |R_b| tokens at the pooled logit (closed form below)."""
    q, k, v, a = _anchor_head()
    nv, ns, d = 640, 16, 32
    scale = 1 / math.sqrt(d)
    O, L, info = orc.forward_head(q, k, v, ns, "topk", 0.2, compressed=True, extra_tokens=E,
                                  pool_mode=pool_mode)
    P = info["pooled"]
    assert P.extra.shape == (E,) and np.all(np.diff(P.extra) > 0)
    s = k[:nv] @ a * scale
    # the extra set: the E largest anchor scores
    assert s[P.extra].min() >= np.sort(s)[::-1][E - 1]
    keep = np.ones(nv, bool)
    keep[P.extra] = False
    for b in range(nv // 64):
        r = keep[b * 64:(b + 1) * 64]
        if pool_mode == "mean" and r.any():
            assert math.isclose(P.beta[b], math.log(r.sum()), rel_tol=0, abs_tol=1e-14)
            np.testing.assert_allclose(P.vtil[b], v[b * 64:(b + 1) * 64][r].mean(0), atol=1e-14)
        if pool_mode == "reweight" and r.any():
            mass = np.exp(s[b * 64:(b + 1) * 64][r]).sum()
            np.testing.assert_allclose(np.exp(P.kc[b] @ a * scale + P.beta[b]), mass, rtol=1e-13)
        if not r.any():
            assert P.beta[b] == -np.inf
    if pool_mode == "reweight":
        ref = sdpa64(q, k, v, scale)
        rows = np.nonzero(np.all(np.abs(q[:nv] - a) < 1e-15, axis=1))[0]
        np.testing.assert_allclose(O[rows], ref[rows], atol=1e-11, rtol=0)
        np.testing.assert_allclose(L[rows], lse64(q, k, scale)[rows], atol=1e-11, rtol=0)


def test_extra_tokens_covering_a_block_equal_selecting_it():
    """When the E = 64 highest anchor scores are exactly the tokens of one block b (its keys
    are shifted along the anchor), taking them as extra tokens gives the same forward as
    adding b to every query block's selection without extra tokens."""
    nv, ns, d = 64 * 12, 20, 32
    q, k, v = head(nv, ns, d, seed=41)
    a = q[:nv].mean(0)
    b = 7
    k[b * 64:(b + 1) * 64] += 6.0 * a / np.linalg.norm(a)
    O1, L1, info = orc.forward_head(q, k, v, ns, "topk", 0.25, compressed=True, extra_tokens=64)
    np.testing.assert_array_equal(info["extra"], np.arange(b * 64, (b + 1) * 64))
    assert info["pooled"].beta[b] == -np.inf
    sel = [np.union1d(s_, [b]) for s_ in info["sel"]]
    assert any(b not in s_ for s_ in info["sel"])
    O2, L2, _ = orc.forward_head(q, k, v, ns, "topk", 0.25, compressed=True, sel_override=sel)
    np.testing.assert_allclose(O1, O2, atol=1e-12, rtol=0)
    np.testing.assert_allclose(L1, L2, atol=1e-12, rtol=0)


@pytest.mark.parametrize("compressed", [True, False])
def test_all_tokens_extra_is_dense_attention(compressed):
    """E >= the number of video tokens makes every key exact: dense attention for every row."""
    nv, ns, d = 64 * 6 + 13, 9, 32
    q, k, v = head(nv, ns, d, seed=2)
    O, L, info = orc.forward_head(q, k, v, ns, "topk", 0.2, compressed=compressed, extra_tokens=10 ** 6)
    scale = 1 / math.sqrt(d)
    assert info["extra"].shape == (64 * 6,)
    np.testing.assert_allclose(O, sdpa64(q, k, v, scale), atol=1e-12, rtol=0)
    np.testing.assert_allclose(L, lse64(q, k, scale), atol=1e-12, rtol=0)


def test_extra_token_ties_go_to_the_lower_index():
    """Hand-derived: keys 5 and 200 are the same vector, the largest anchor score; with a
    budget of one token the lower index is taken, with two both are."""
    nv, d = 64 * 4, 16
    rng = np.random.default_rng(3)
    a = rng.standard_normal(d)
    k = rng.standard_normal((nv, d)) * 0.1
    k[5] = k[200] = 3.0 * a
    s = k @ a
    np.testing.assert_array_equal(orc.select_extra_tokens(s, 1), [5])
    np.testing.assert_array_equal(orc.select_extra_tokens(s, 2), [5, 200])
    assert orc.select_extra_tokens(s, 0).size == 0


def test_extra_tokens_zero_changes_nothing():
    q, k, v = head(64 * 10, 12, 32, seed=9)
    O0, L0, _ = orc.forward_head(q, k, v, 12, "tau", 0.8, compressed=True)
    O1, L1, info = orc.forward_head(q, k, v, 12, "tau", 0.8, compressed=True, extra_tokens=0)
    assert info["extra"].size == 0
    np.testing.assert_array_equal(O0, O1)
    np.testing.assert_array_equal(L0, L1)


@pytest.mark.parametrize("q_offset", [0.0, 1.0])
def test_extra_tokens_bring_the_forward_closer_to_dense(q_offset):
    """Fidelity: taking the highest-scoring tokens out of the compressed entries into the
    exact branch moves the output toward dense attention, with and without the compressed
    branch."""
    nv, ns, d = 64 * 40, 16, 64
    Q, K, V = make_qkv(1, 1, nv, ns, d, seed=12, q_offset=q_offset)
    q, k, v = (orc.to_f64(t[0, 0]) for t in (Q, K, V))
    dense, _, _ = orc.forward_head(q, k, v, ns, "topk", 1.0, False)
    for comp in (True, False):
        err = []
        for E in (0, 256, 1024):
            o, _, _ = orc.forward_head(q, k, v, ns, "topk", 0.1, comp, extra_tokens=E)
            err.append(np.linalg.norm(o[:nv] - dense[:nv]) / np.linalg.norm(dense[:nv]))
        assert err[0] > err[1] > err[2], (comp, err)


def test_planted_extra_token_counted_twice_is_caught(monkeypatch):
    """An extra token inside a selected block attended a second time must break the
    anchor-row pin."""
    real = orc.attn_video_block

    def bad(q, k, v, n_sink, i, sel, pooled, scale=None, block=64, q_tile=64, extra=None):
        o, l = real(q, k, v, n_sink, i, sel, pooled, scale, block, q_tile, None)
        if extra is None or len(extra) == 0:
            return o, l
        # recompute with every extra token appended, duplicates included
        sel = np.asarray(sel, dtype=np.int64)
        nv = orc.n_blocks(q.shape[0], n_sink, block) * block
        rows = np.concatenate([np.arange(b * block, (b + 1) * block) for b in sel]
                              + [np.asarray(extra, dtype=np.int64), np.arange(nv, q.shape[0])])
        qi = q[orc.tile_rows(i, nv, q_tile)]
        lg = (qi @ k[rows].T) * scale
        unsel = np.setdiff1d(np.arange(nv // block), sel)
        unsel = unsel[np.isfinite(pooled.beta[unsel])]
        lg = np.concatenate([lg, (qi @ pooled.kc[unsel].T) * scale + pooled.beta[unsel]], axis=1)
        vals = np.concatenate([v[rows], pooled.vtil[unsel]], axis=0)
        return orc._softmax_out(lg, vals)
    monkeypatch.setattr(orc, "attn_video_block", bad)
    with pytest.raises(AssertionError):
        test_extra_tokens_keep_anchor_rows_exact(200, "reweight")


def test_planted_entry_over_the_whole_block_is_caught(monkeypatch):
    """Keeping the whole-block summary after taking tokens out (mass counted twice) must
    break the anchor-row pin."""
    real = orc.pool_head

    def bad(q, k, v, n_sink, scale=None, block=64, mode="reweight", q_tile=64, extra=0, extra_override=None):
        P = real(q, k, v, n_sink, scale, block, mode, q_tile, extra, extra_override)
        P0 = real(q, k, v, n_sink, scale, block, mode, q_tile, 0, None)
        P.kc, P.vtil, P.beta, P.lse = P0.kc, P0.vtil, P0.beta, P0.lse
        return P
    monkeypatch.setattr(orc, "pool_head", bad)
    with pytest.raises(AssertionError):
        test_extra_tokens_keep_anchor_rows_exact(200, "reweight")
