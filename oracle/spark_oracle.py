"""fp64 CPU oracle of the block-sparse video attention forward (Spark-Attn split).

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.
It shares no code with the CUDA library and never calls it.

Everything here is plain numpy in float64 on bf16 inputs converted exactly, one
(batch, head) at a time, written in the order the method states its steps. A numpy
matmul / eigh / lexsort serves as a library step where noted; there is no blocking,
fusion or reordering beyond what the definitions below state.

Sources (cited by page title and section):

* [Spark-H3] "Spark-H3: speeding up MiniMax-H3 in ComfyUI with block-sparse attention"
  (comfyui-wiki news, 2026-10-11). Section "What Spark-Attn changes": the exact /
  compressed two-branch split; the Spark-Reblock bullet (Mahalanobis cosine under the
  opposite side's second moment, hierarchical splits until every leaf holds the block
  size, O(N log N)); the Spark-Reweight bullet (weighted value summary + log-mass bias,
  one anchor per head = mean of the video queries) and the figure caption after it
  (mean pooling gives exp(E[x]) < E[exp(x)]; the bias restores the expected exponent).
  Section "Workflows": topk_mode=topk_ratio, reblock_layout=q_reuse_k.
* [Core-node] "ComfyUI adds a core sparse-attention node and the Comfy Compiler"
  (comfyui-wiki news, 2026-09-08). Section "Block-sparse attention: one node, three
  backends": Sol-Attn per-head adaptive threshold tau in units of the block-score
  sigma (tau 1.0 / 1.5 / 2.0 keep about 16% / 7% / 2.7%); top-k keep_percent (SLA);
  sink_conditioning attends packed text/audio/reference rows exactly.
* [H3-Opt] "H3 Optimizations" node-pack README. Section "Nodes": text, reference,
  audio, non-video queries and mixed boundary tiles stay dense.

Readings where the pages are silent (each the plainest one the rest supports):

* video rows come first, the ``n_sink`` sink rows last; blocks are consecutive runs of
  64 video rows. A ragged tail of fewer than 64 video rows is handled exactly like sink
  rows (dense queries, always-attended keys, never pooled or scored);
* block score S[i, j] = qbar_i . kbar_j * scale, scale = 1/sqrt(d);
* top-k keeps k = min(nb, max(1, ceil(ratio * nb - 1e-9))) blocks per query block,
  ranked by (score descending, block index ascending);
* tau keeps S[i, j] > mu_h + tau * sigma_h, with mu_h and sigma_h (population) over all
  nb^2 scores of the head; there is no per-row floor, so a row may keep nothing;
* the compressed branch covers every unselected video block of the query block (sinks
  are never compressed) with logit q . kbar_b * scale + beta_b and value vtil_b, where
  s_j = a . k_j * scale, vtil_b = sum_j softmax_b(s)_j v_j and
  beta_b = logsumexp_b(s) - a . kbar_b * scale; the entry carries the whole block's mass;
* the plain mean-pool compressed branch (the baseline Spark-Reweight replaces) uses
  vtil_b = mean_b v and beta_b = log(64): the entry stands for 64 tokens that all take
  the pooled logit;
* sink queries attend densely to every key, with no compressed branch;
* a query row with no entry at all returns O = 0 and LSE = -inf;
* Reblock: M = mean over video keys of k k^T; x_i = L^T q_i / |L^T q_i| with M = L L^T
  (Cholesky); a node of m blocks takes the leading eigenvector v of the centred
  covariance of its x, signs v so that the third central moment of the projections is
  >= 0, orders its tokens by (x . v, token index) and sends the first floor(m/2)*64 to
  the left child; leaves are ordered by their smallest token index and hold their
  tokens in ascending order. Keys reuse the query partition (q_reuse_k).
* extra tokens ([Core-node] "Block-sparse attention: one node, three backends": an
  advanced option adds the highest-scoring tokens beyond the selected blocks, to stay
  close to dense attention; the pages give neither the score nor the count's unit):
  a per-head budget of E tokens, scored by the anchor score s_j = a . k_j * scale (the
  per-token score the compressed branch already uses), ranked by (s desc, token index
  asc) over the head's video keys. Every video query attends the extra tokens exactly
  (those inside its selected blocks once, as part of the block); the compressed entry of
  an unselected block then stands only for the block's remaining tokens R_b: its key
  mean, value summary and log-mass bias are those of R_b (the mean-pool branch: mean
  value of R_b, beta = log |R_b|), and a block whose 64 tokens are all extra has no
  entry. Block scores (the selection) keep the whole-block means; sink queries stay
  dense;
* the 128-query x 64-key route ([H3-Opt] section "Manual Sparse Sage recovery": the
  sparse fallback backends consume a 128Q x 64KV route): a query tile is two consecutive video blocks
  (the last tile holds one block when nb is odd); its pooled query is the mean of the
  tile's queries, it is scored against the 64-token key blocks and keeps
  k = topk_count(ratio, nb) of them (tau: mu and sigma over all tile x block scores);
  every query of the tile attends to the tile's selection. Keys, the anchor and the
  compressed branch do not change.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

BLOCK = 64


# --------------------------------------------------------------------------- helpers

def to_f64(t) -> np.ndarray:
    """Exact conversion of a torch tensor (bf16/fp32/...) to a float64 numpy array."""
    import torch  # local: the oracle needs torch only to read tensors
    return t.detach().to("cpu", torch.float64).numpy()


def default_scale(d: int, scale: float | None = None) -> float:
    return 1.0 / math.sqrt(d) if (scale is None or scale <= 0) else float(scale)


def n_blocks(n_rows: int, n_sink: int, block: int = BLOCK) -> int:
    """Number of full video blocks; the rest of the rows are dense (sinks, ragged tail)."""
    return max(n_rows - n_sink, 0) // block


# --------------------------------------------------------------------------- pooling

@dataclass
class Pooled:
    qbar: np.ndarray    # [nt, d] mean query of each query tile (a block unless q_tile = 128)
    kbar: np.ndarray    # [nb, d] mean key of each block (block scores)
    vtil: np.ndarray    # [nb, d] value summary of each block's compressed entry
    beta: np.ndarray    # [nb]    log-mass bias of each entry (-inf: the block has no entry)
    anchor: np.ndarray  # [d]     per-head anchor (mean video query)
    lse: np.ndarray     # [nb]    logsumexp of the anchor scores of each entry's tokens
    kc: np.ndarray = None      # [nb, d] key mean of each entry's tokens (kbar without extra tokens)
    extra: np.ndarray = None   # [E]  extra token indices, ascending (empty without extra tokens)


def n_tiles(nb: int, q_tile: int = BLOCK, block: int = BLOCK) -> int:
    """Query tiles of the route: ceil(nb * block / q_tile) (the last may be shorter)."""
    return -(-nb * block // q_tile)


def tile_rows(t: int, nv: int, q_tile: int = BLOCK) -> np.ndarray:
    """Video rows of query tile t."""
    return np.arange(t * q_tile, min((t + 1) * q_tile, nv))


def anchor_scores(k_video, anchor, scale) -> np.ndarray:
    """s_j = a . k_j * scale for every video key j."""
    return (k_video @ anchor) * scale


def select_extra_tokens(s, n_extra) -> np.ndarray:
    """The n_extra video keys with the highest anchor scores, ranked by (s desc, index asc);
    returned ascending."""
    n_extra = int(min(max(n_extra, 0), s.shape[0]))
    if n_extra == 0:
        return np.zeros(0, dtype=np.int64)
    j = np.arange(s.shape[0])
    return np.sort(np.lexsort((j, -s))[:n_extra]).astype(np.int64)


def pool_head(q, k, v, n_sink, scale=None, block=BLOCK, mode="reweight", q_tile=BLOCK,
              extra=0, extra_override=None) -> Pooled:
    """Mean pooling, anchor and Spark-Reweight summaries of one head.

    [Spark-H3] "What Spark-Attn changes", Spark-Reweight bullet and the figure caption:
    one anchor per head (the mean of the video queries) scores every key of a block;
    the value summary is the softmax-weighted mean under those scores, and the log-mass
    bias makes exp(a . kbar_b * scale + beta_b) equal the block's total mass
    sum_j exp(s_j). ``mode="mean"`` gives the plain mean-pool branch instead.
    ``q_tile`` = 128 pools the queries over the tiles of the 128-query route (qbar has
    one row per tile); keys and the compressed branch keep 64-token blocks.
    ``extra`` > 0 takes that many extra tokens (``extra_override``: a given token list
    instead) out of their blocks' compressed entries, which then summarise the remaining
    tokens of each block only (see the module header).
    """
    d = q.shape[1]
    scale = default_scale(d, scale)
    nb = n_blocks(q.shape[0], n_sink, block)
    nv = nb * block
    qb = q[:nv].reshape(nb, block, d)
    kb = k[:nv].reshape(nb, block, d)
    vb = v[:nv].reshape(nb, block, d)
    if q_tile == block:
        qbar = qb.mean(axis=1)
    else:
        qbar = np.stack([q[tile_rows(t, nv, q_tile)].mean(axis=0)
                         for t in range(n_tiles(nb, q_tile, block))]) if nb else np.zeros((0, d))
    kbar = kb.mean(axis=1)
    anchor = q[:nv].mean(axis=0) if nv else np.zeros(d)
    s = anchor_scores(k[:nv], anchor, scale).reshape(nb, block)  # [nb, block]
    if extra_override is not None:
        xt = np.sort(np.asarray(extra_override, dtype=np.int64))
    else:
        xt = select_extra_tokens(s.reshape(-1), extra)
    if mode not in ("reweight", "mean"):
        raise ValueError(mode)
    if xt.size == 0:
        if nb:
            smax = s.max(axis=1, keepdims=True)
            lse = smax[:, 0] + np.log(np.exp(s - smax).sum(axis=1))
        else:
            lse = np.zeros(0)
        if mode == "reweight":
            w = np.exp(s - lse[:, None])                        # softmax inside each block
            vtil = np.einsum("bj,bjd->bd", w, vb)
            beta = lse - (kbar @ anchor) * scale
        else:
            vtil = vb.mean(axis=1)
            beta = np.full(nb, math.log(block))
        return Pooled(qbar, kbar, vtil, beta, anchor, lse, kbar.copy(), xt)
    # with extra tokens: each block's entry summarises its remaining tokens R_b
    keep = np.ones(nv, dtype=bool)
    keep[xt] = False
    keep = keep.reshape(nb, block)
    kc = np.zeros((nb, d))
    vtil = np.zeros((nb, d))
    lse = np.full(nb, -np.inf)
    beta = np.full(nb, -np.inf)
    for b in range(nb):
        r = keep[b]
        if not r.any():
            continue                                            # every token is extra: no entry
        kc[b] = kb[b][r].mean(axis=0)
        sr = s[b][r]
        m = sr.max()
        lse[b] = m + math.log(np.exp(sr - m).sum())
        if mode == "reweight":
            vtil[b] = np.exp(sr - lse[b]) @ vb[b][r]
            beta[b] = lse[b] - float(kc[b] @ anchor) * scale
        else:
            vtil[b] = vb[b][r].mean(axis=0)
            beta[b] = math.log(int(r.sum()))
    return Pooled(qbar, kbar, vtil, beta, anchor, lse, kc, xt)


# --------------------------------------------------------------------------- scoring / selection

def block_scores(qbar, kbar, scale, rows=None) -> np.ndarray:
    """S[i, j] = qbar_i . kbar_j * scale (rows i of ``rows``, all j)."""
    qs = qbar if rows is None else qbar[np.asarray(rows)]
    return (qs @ kbar.T) * scale


def topk_count(ratio: float, nb: int) -> int:
    """Blocks kept per query block at keep ratio ``ratio`` ([Core-node], top-k bullet)."""
    if nb <= 0:
        return 0
    return int(min(nb, max(1, math.ceil(float(ratio) * nb - 1e-9))))


def select_topk_row(s_row, k) -> np.ndarray:
    """The k largest scores of one row, ranked by (score desc, index asc); returned ascending."""
    j = np.arange(s_row.shape[0])
    order = np.lexsort((j, -s_row))      # primary key: -score, secondary: index
    return np.sort(order[:k])


def tau_stats(S_full) -> tuple[float, float]:
    """Per-head mean and population standard deviation of all nb^2 block scores."""
    mu = float(S_full.mean())
    sigma = float(np.sqrt(((S_full - mu) ** 2).mean()))
    return mu, sigma


def tau_threshold(S_full, tau) -> float:
    """[Core-node] Sol-Attn bullet: per-head threshold tau sigma above the score mean."""
    mu, sigma = tau_stats(S_full)
    return mu + float(tau) * sigma


def select_tau_row(s_row, thr) -> np.ndarray:
    return np.nonzero(s_row > thr)[0]


def select_head(qbar, kbar, scale, mode, param, rows=None):
    """Selected block lists of one head: a list of ascending int arrays, one per row."""
    rows = np.arange(qbar.shape[0]) if rows is None else np.asarray(rows)
    if mode == "topk":
        k = topk_count(param, kbar.shape[0])
        S = block_scores(qbar, kbar, scale, rows)
        return [select_topk_row(S[r], k) for r in range(len(rows))]
    if mode == "tau":
        thr = tau_threshold(block_scores(qbar, kbar, scale), param)
        S = block_scores(qbar, kbar, scale, rows)
        return [select_tau_row(S[r], thr) for r in range(len(rows))]
    raise ValueError(mode)


# --------------------------------------------------------------------------- attention

def _softmax_out(logits, vals):
    """o = softmax(logits) @ vals and LSE = logsumexp(logits), row by row."""
    nq = logits.shape[0]
    if logits.shape[1] == 0:
        return np.zeros((nq, vals.shape[1])), np.full(nq, -np.inf)
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    l = p.sum(axis=1, keepdims=True)
    return (p @ vals) / l, (m + np.log(l))[:, 0]


def attn_video_block(q, k, v, n_sink, i, sel, pooled: Pooled | None, scale=None, block=BLOCK,
                     q_tile=BLOCK, extra=None):
    """Output rows of video query tile i (block i unless ``q_tile`` = 128), in the order of q.

    [Spark-H3] "What Spark-Attn changes": the exact branch attends to the keys of the
    selected blocks, the compressed branch covers every other video block with one
    pooled entry each; [Core-node] sink_conditioning: every sink key is attended
    exactly, and extra_tokens adds the head's extra tokens (``extra``, token indices) to
    the exact branch. All logits share one softmax (one log-sum-exp merge).
    """
    d = q.shape[1]
    scale = default_scale(d, scale)
    nb = n_blocks(q.shape[0], n_sink, block)
    nv = nb * block
    qi = q[tile_rows(i, nv, q_tile)]
    sel = np.asarray(sel, dtype=np.int64)
    # extra tokens outside the selected blocks (those inside are attended as part of it)
    xt = np.zeros(0, dtype=np.int64) if extra is None else np.asarray(extra, dtype=np.int64)
    xt = xt[~np.isin(xt // block, sel)]
    key_rows = np.concatenate([np.arange(b * block, (b + 1) * block) for b in sel]
                              + [xt, np.arange(nv, q.shape[0])]).astype(np.int64)
    logits = (qi @ k[key_rows].T) * scale
    vals = v[key_rows]
    if pooled is not None:
        unsel = np.setdiff1d(np.arange(nb), sel)
        unsel = unsel[np.isfinite(pooled.beta[unsel])]          # blocks left with an entry
        kc = pooled.kbar if pooled.kc is None else pooled.kc
        logits = np.concatenate([logits, (qi @ kc[unsel].T) * scale + pooled.beta[unsel]], axis=1)
        vals = np.concatenate([vals, pooled.vtil[unsel]], axis=0)
    return _softmax_out(logits, vals)


def attn_dense_rows(q, k, v, rows, scale=None):
    """Dense softmax attention of query rows ``rows`` over every key ([H3-Opt] "Nodes")."""
    scale = default_scale(q.shape[1], scale)
    return _softmax_out((q[np.asarray(rows)] @ k.T) * scale, v)


def attention_head(q, k, v, n_sink, sel_lists, pooled=None, scale=None, block=BLOCK,
                   qblocks=None, dense_rows=True, q_tile=BLOCK, extra=None):
    """O [N, d] and LSE [N] of one head; rows not computed are NaN.

    ``sel_lists[i]`` is the selected block list of video query tile i (all tiles when
    ``qblocks`` is None, else the tiles listed in ``qblocks``, in that order).
    """
    N, d = q.shape
    nb = n_blocks(N, n_sink, block)
    O = np.full((N, d), np.nan)
    L = np.full(N, np.nan)
    blocks = range(n_tiles(nb, q_tile, block)) if qblocks is None else qblocks
    for t, i in enumerate(blocks):
        o, l = attn_video_block(q, k, v, n_sink, i, sel_lists[t], pooled, scale, block, q_tile, extra)
        rows = tile_rows(i, nb * block, q_tile)
        O[rows] = o
        L[rows] = l
    if dense_rows and N > nb * block:
        rows = np.arange(nb * block, N)
        o, l = attn_dense_rows(q, k, v, rows, scale)
        O[rows] = o
        L[rows] = l
    return O, L


# --------------------------------------------------------------------------- Spark-Reblock

def key_second_moment(k_video) -> np.ndarray:
    """M = mean_j k_j k_j^T over the video keys ("the opposite side's second moment")."""
    return (k_video.T @ k_video) / max(k_video.shape[0], 1)


def whiten(q_video, M) -> np.ndarray:
    """Unit vectors x_i = L^T q_i / |L^T q_i| with M = L L^T, so x_i . x_j is the
    Mahalanobis cosine q_i^T M q_j / (|q_i|_M |q_j|_M) ([Spark-H3] Spark-Reblock bullet).
    A query with zero M-norm maps to the zero vector. When M is not positive definite the
    factor of M + 1e-6 tr(M)/d I is used, and the identity when that fails too."""
    d = M.shape[0]
    try:
        L = np.linalg.cholesky(M)
    except np.linalg.LinAlgError:
        try:
            L = np.linalg.cholesky(M + 1e-6 * np.trace(M) / d * np.eye(d))
        except np.linalg.LinAlgError:
            L = np.eye(d)   # degenerate keys (e.g. all zero): plain cosine
    x = q_video @ L
    nrm = np.linalg.norm(x, axis=1, keepdims=True)
    return np.divide(x, nrm, out=np.zeros_like(x), where=nrm > 0)


@dataclass
class Split:
    left: np.ndarray        # token indices sent to the left child (ascending)
    right: np.ndarray
    split_value: float      # projection at the boundary (mean of the two straddling values)
    proj: dict = field(repr=False, default_factory=dict)  # token -> projection
    gap: float = 1.0        # relative eigengap (lambda1 - lambda2) / lambda1
    skew: float = 0.0       # third central moment of the projections / sigma^3 (after signing)


def split_node(x, members, block=BLOCK) -> Split:
    """One bisection of a node of m = len(members)/block blocks.

    Leading eigenvector of the node's centred covariance (numpy eigh), signed so the
    projections' third central moment is >= 0; tokens ordered by (projection, token
    index); the first floor(m/2) blocks of that order form the left child.
    """
    members = np.asarray(members, dtype=np.int64)
    n = members.shape[0]
    m = n // block
    xs = x[members]
    xc = xs - xs.mean(axis=0)
    C = (xc.T @ xc) / n
    w, V = np.linalg.eigh(C)
    v = V[:, -1]
    gap = float((w[-1] - w[-2]) / w[-1]) if w[-1] > 0 else 0.0
    p = xs @ v
    pc = p - p.mean()
    m3 = float((pc ** 3).mean())
    sd = float(np.sqrt((pc ** 2).mean()))
    if m3 < 0:
        p = -p
        m3 = -m3
    order = np.lexsort((members, p))
    cut = (m // 2) * block
    left = np.sort(members[order[:cut]])
    right = np.sort(members[order[cut:]])
    split_value = 0.5 * (p[order[cut - 1]] + p[order[cut]])
    return Split(left, right, split_value, dict(zip(members.tolist(), p.tolist())), gap,
                 m3 / sd ** 3 if sd > 0 else 0.0)


def n_levels(nb: int) -> int:
    """Bisection levels until every node holds one block: ceil(log2(nb))."""
    return 0 if nb <= 1 else int(math.ceil(math.log2(nb)))


@dataclass
class ReblockResult:
    perm: np.ndarray        # [nv] perm[p] = original token index at permuted position p
    labels: np.ndarray      # [levels+1, nv] node label of every token at every level
    splits: dict            # (level, label) -> Split


def reblock_head(q, k, n_sink, block=BLOCK) -> ReblockResult:
    """Spark-Reblock partition of one head ([Spark-H3] Spark-Reblock bullet; the
    q_reuse_k layout of "Workflows" reuses this partition for the keys).

    Level-synchronous bisection: at every level a node with label c and m > 1 blocks
    sends its left part to label 2c and its right part to 2c + 1; a leaf moves to 2c.
    """
    nb = n_blocks(q.shape[0], n_sink, block)
    nv = nb * block
    x = whiten(q[:nv], key_second_moment(k[:nv]))
    L = n_levels(nb)
    labels = np.zeros((L + 1, nv), dtype=np.int64)
    splits = {}
    for lev in range(L):
        cur = labels[lev]
        nxt = 2 * cur
        for c in np.unique(cur):
            members = np.nonzero(cur == c)[0]
            if members.shape[0] > block:
                sp = split_node(x, members, block)
                splits[(lev, int(c))] = sp
                nxt[sp.right] = 2 * c + 1
        labels[lev + 1] = nxt
    return ReblockResult(canonical_perm(labels[L]), labels, splits)


def canonical_perm(leaf_labels) -> np.ndarray:
    """Leaves ordered by their smallest token index, tokens ascending inside a leaf."""
    leaf_labels = np.asarray(leaf_labels)
    groups = {}
    for t, c in enumerate(leaf_labels.tolist()):
        groups.setdefault(c, []).append(t)
    leaves = sorted(groups.values(), key=lambda g: g[0])
    return np.array([t for g in leaves for t in g], dtype=np.int64)


def apply_perm(x, perm, n_sink, block=BLOCK):
    """Rows p < nv of the result are x[perm[p]]; dense rows are copied unchanged."""
    nb = n_blocks(x.shape[0], n_sink, block)
    out = x.copy()
    out[: nb * block] = x[np.asarray(perm)]
    return out


# --------------------------------------------------------------------------- full forward

def forward_head(q, k, v, n_sink, mode="topk", param=0.1, compressed=True, scale=None,
                 block=BLOCK, reblock=False, qblocks=None, sel_override=None,
                 pool_mode="reweight", perm_override=None, reblock_kv=False,
                 perm_k_override=None, q_tile=BLOCK, extra_tokens=0, extra_override=None):
    """The whole forward of one head, in the original token order.

    Returns (O [N, d], LSE [N], info) where info holds the selection lists, the pooled
    summaries and, when ``reblock``, the Reblock result. ``sel_override`` replaces the
    oracle's own selection (used when a near-tie lets the GPU legitimately pick another
    block). ``qblocks`` restricts the video query blocks computed (others are NaN).
    ``reblock_kv``: the keys get a partition of their own (the same bisection on the
    keys, whitened by the queries' second moment) instead of reusing the queries'
    (the alternative to q_reuse_k in [Spark-H3] "Workflows"); K and V follow it.
    ``q_tile`` = 128: the 128-query route (``qblocks`` then lists query tiles).
    ``extra_tokens``: the per-head budget of extra tokens (``extra_override``: the token
    list to use instead of the oracle's own, e.g. when a near-tie lets the device take
    another token); the tokens are indices of the (reblocked) video rows.
    """
    if q_tile not in (BLOCK, 2 * BLOCK) or block != BLOCK:
        raise ValueError("q_tile must be 64 or 128 with 64-token blocks")
    d = q.shape[1]
    scale = default_scale(d, scale)
    info = {}
    if reblock:
        if perm_override is not None:
            rb = ReblockResult(np.asarray(perm_override, dtype=np.int64), None, {})
        else:
            rb = reblock_head(q, k, n_sink, block)
        info["reblock"] = rb
        qp = apply_perm(q, rb.perm, n_sink, block)
        if reblock_kv:
            if perm_k_override is not None:
                rbk = ReblockResult(np.asarray(perm_k_override, dtype=np.int64), None, {})
            else:
                rbk = reblock_head(k, q, n_sink, block)  # keys partitioned, whitened by queries
            info["reblock_k"] = rbk
            kp, vp = (apply_perm(t, rbk.perm, n_sink, block) for t in (k, v))
        else:
            kp, vp = (apply_perm(t, rb.perm, n_sink, block) for t in (k, v))
    else:
        qp, kp, vp = q, k, v
    pooled = pool_head(qp, kp, vp, n_sink, scale, block, pool_mode, q_tile, extra_tokens, extra_override)
    info["pooled"] = pooled
    info["extra"] = pooled.extra
    nb = pooled.kbar.shape[0]
    rows = np.arange(pooled.qbar.shape[0]) if qblocks is None else np.asarray(qblocks)
    if sel_override is not None:
        sel = sel_override
    else:
        sel = select_head(pooled.qbar, pooled.kbar, scale, mode, param, rows)
    info["sel"] = sel
    O, L = attention_head(qp, kp, vp, n_sink, sel, pooled if compressed else None, scale,
                          block, qblocks=rows, q_tile=q_tile, extra=pooled.extra)
    if reblock:
        nv = nb * block
        O2, L2 = O.copy(), L.copy()
        O2[rb.perm] = O[:nv]
        L2[rb.perm] = L[:nv]
        O, L = O2, L2
    return O, L, info
