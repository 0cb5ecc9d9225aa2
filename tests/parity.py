"""Comparison helpers for the GPU-vs-oracle parity tests (selection tie windows and the
output tolerances)."""
import math

import numpy as np

import oracle.spark_oracle as orc

TIE = 1e-4          # scores closer than this to the cut count as ties
MAX_ABS = 1e-2      # output max |o - r|
MEAN_REL = 5e-3     # output sum |o - r| / sum |r|
LSE_ABS = 5e-3      # natural-log LSE, |l - r|


def gpu_rows(idx, cnt):
    """List of ascending index arrays (the kept sets) from the device's idx/cnt of one
    head; the device writes each row in its sweep order (see sweep_start)."""
    idx = np.asarray(idx)
    cnt = np.asarray(cnt)
    return [np.sort(idx[i, : cnt[i]].astype(np.int64)) for i in range(cnt.shape[0])]


def sweep_start(i, nb, sweep):
    """First block position of row i's sweep order: floor((i mod sweep) * nb / sweep)
    rounded down to a multiple of 32 (sweep = query tiles the attention kernel runs at
    once: 2 per SM for 64-query tiles, 1 per SM for 128-query tiles)."""
    return ((i % sweep) * nb // sweep) & ~31


def check_sweep_order(row, i, nb, sweep):
    """True when a device row lists its kept blocks ascending from the first one at or
    above sweep_start(i), then the ones below it, ascending."""
    row = np.asarray(row, dtype=np.int64)
    s = np.sort(row)
    st = sweep_start(i, nb, sweep)
    return np.array_equal(row, np.concatenate([s[s >= st], s[s < st]]))


def check_selection_row(gsel, s_row, mode, param, thr=None):
    """True when the device's kept set equals the oracle's up to near-ties; returns
    (ok, n_differing)."""
    gsel = np.asarray(gsel, dtype=np.int64)
    if np.any(np.diff(gsel) <= 0):
        return False, -1
    nb = s_row.shape[0]
    if mode == "topk":
        k = orc.topk_count(param, nb)
        ref = orc.select_topk_row(s_row, k)
        cut = np.sort(s_row)[::-1][k - 1]
        if gsel.shape[0] != k:
            return False, -1
    else:
        ref = orc.select_tau_row(s_row, thr)
        cut = thr
    diff = np.setxor1d(ref, gsel)
    if diff.size == 0:
        return True, 0
    return bool(np.all(np.abs(s_row[diff] - cut) < TIE)), int(diff.size)


def check_output(o, r, what=""):
    o = np.asarray(o, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    assert o.shape == r.shape, (o.shape, r.shape)
    err = np.abs(o - r)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.abs(r).sum())
    mean_rel = float(err.sum() / denom) if denom > 0 else float(err.sum())
    assert max_abs <= MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {MAX_ABS}"
    assert mean_rel <= MEAN_REL, f"{what}: mean-rel {mean_rel:.3e} > {MEAN_REL}"
    return max_abs, mean_rel


def check_lse(l, r, what=""):
    l = np.asarray(l, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    inf = np.isneginf(r)
    assert np.array_equal(np.isneginf(l), inf), what
    if (~inf).any():
        d = float(np.abs(l[~inf] - r[~inf]).max())
        assert d <= LSE_ABS, f"{what}: LSE max-abs {d:.3e}"


def default_scale(d):
    return 1.0 / math.sqrt(d)


GAP_TIE = 1e-4      # relative eigengap below which a node's direction is ill-defined
SKEW_TIE = 1e-6     # |third moment| / sigma^3 below which the sign of v is ambiguous


def replay_reblock_tree(x, tree, levels, nodes=None):
    """Node replay: for every node of the device's tree (its token set given by the labels
    at `level`, split into the labels 2c / 2c + 1 at level + 1) the oracle recomputes the
    split in fp64 from the same membership. Returns (n_checked, n_skipped_as_ties); raises
    AssertionError on a disagreement outside the tie windows. `nodes` limits the check to
    a list of (level, label)."""
    checked = skipped = 0
    todo = nodes
    if todo is None:
        todo = [(lev, int(c)) for lev in range(levels) for c in np.unique(tree[lev])]
    for lev, c in todo:
        members = np.nonzero(tree[lev] == c)[0]
        if members.size <= 64:
            continue
        left_dev = set(np.nonzero(tree[lev + 1][members] == 2 * c)[0].tolist())
        left_dev = set(members[list(left_dev)].tolist())
        assert len(left_dev) == (members.size // 64 // 2) * 64, (lev, c, len(left_dev))
        sp = orc.split_node(x, members)
        if sp.gap < GAP_TIE:
            skipped += 1
            continue
        cut = len(left_dev)
        cands = [(set(sp.left.tolist()), 1.0, sp.split_value)]
        if abs(sp.skew) < SKEW_TIE:
            # the other orientation: the lowest projections after flipping the sign
            pf = -np.array([sp.proj[t] for t in members.tolist()])
            order = np.lexsort((members, pf))
            split_f = 0.5 * (pf[order[cut - 1]] + pf[order[cut]])
            cands.append((set(members[order[:cut]].tolist()), -1.0, split_f))
        ok = False
        for cand, sg, split in cands:
            diff = cand ^ left_dev
            if all(abs(sg * sp.proj[t] - split) < TIE for t in diff):
                ok = True
                break
        assert ok, (lev, c, len(cands[0][0] ^ left_dev))
        checked += 1
    return checked, skipped


def check_partition(perm, nv):
    perm = np.asarray(perm)
    assert sorted(perm.tolist()) == list(range(nv))
    leaves = perm.reshape(-1, 64)
    assert np.all(np.diff(leaves, axis=1) > 0)
    assert np.all(np.diff(leaves[:, 0]) > 0)
