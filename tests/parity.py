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
    """List of ascending index arrays from the device's idx/cnt of one head."""
    idx = np.asarray(idx)
    cnt = np.asarray(cnt)
    return [idx[i, : cnt[i]].astype(np.int64) for i in range(cnt.shape[0])]


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
