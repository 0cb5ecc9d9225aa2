"""GPU parity of the extra tokens ("ComfyUI adds a core sparse-attention node...", section
"Block-sparse attention: one node, three backends": extra_tokens adds the highest-scoring
tokens beyond the selected blocks).

The device's extra tokens must be the oracle's (the E largest anchor scores, ties to the
lower index) up to tokens whose fp64 score lies within the tie window of the E-th score;
where they differ there, the oracle takes the device's set. The rewritten compressed
entries (value summary, log-mass bias; no entry for a block whose 64 tokens are all extra)
and every output element are then compared with the oracle, on both query routes, with
the compressed branch on and off, and in front of Reblock."""
import math

import numpy as np
import pytest
import torch

import oracle.spark_oracle as orc
from block_sparse_video_mean_b200.inputs import make_qkv
from tests.parity import TIE, check_lse, check_output, check_selection_row, gpu_rows

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def spark():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_video_mean_b200.spark as spark
    spark.load()
    return spark


def check_extra_set(dev, s, E):
    """The device's extra tokens against the oracle's, up to near-ties; returns the set the
    oracle should use (the device's)."""
    dev = np.asarray(dev, dtype=np.int64)
    n = min(E, s.shape[0])
    assert dev.shape == (n,) and np.all(np.diff(dev) > 0) and dev.min() >= 0 and dev.max() < s.shape[0]
    ref = orc.select_extra_tokens(s, E)
    diff = np.setxor1d(ref, dev)
    if diff.size:
        cut = np.sort(s)[::-1][n - 1]
        assert np.all(np.abs(s[diff] - cut) < TIE), diff
    return dev


def compare_extra_head(spark, plan, Q, K, V, b, h, ns, cfg, qblocks=None, dense=True):
    q, k, v = (orc.to_f64(t[b, h]) for t in (Q, K, V))
    d = q.shape[1]
    scale = 1.0 / math.sqrt(d)
    nb = plan.nb
    perm = None
    if cfg.reblock:
        perm = plan.rb["perm"][b, h].cpu().numpy().astype(np.int64)
        q, k, v = (orc.apply_perm(t, perm, ns) for t in (q, k, v))
    P0 = orc.pool_head(q, k, v, ns, scale, 64, cfg.pool_mode, cfg.q_tile)
    s = orc.anchor_scores(k[: nb * 64], P0.anchor, scale)
    xs = check_extra_set(plan.extra_rows()[b, h].cpu().numpy(), s, cfg.extra_tokens)
    P = orc.pool_head(q, k, v, ns, scale, 64, cfg.pool_mode, cfg.q_tile, extra_override=xs)
    if cfg.compressed:
        gb = plan.pool["beta"][b, h].cpu().double().numpy()
        assert np.array_equal(np.isneginf(gb), np.isneginf(P.beta))
        fin = np.isfinite(P.beta)
        np.testing.assert_allclose(gb[fin], P.beta[fin], atol=2e-5, rtol=0)
        gv = plan.pool["v_summ"][b, h].cpu().double().numpy()
        np.testing.assert_allclose(gv[fin], P.vtil[fin], atol=2e-5, rtol=0)
    sel = gpu_rows(plan.idx[b, h].cpu().numpy(), plan.cnt[b, h].cpu().numpy())
    thr = orc.tau_threshold(orc.block_scores(P.qbar, P.kbar, scale), cfg.param) if cfg.mode == "tau" else None
    blocks = np.arange(P.qbar.shape[0]) if qblocks is None else np.asarray(qblocks)
    S = orc.block_scores(P.qbar, P.kbar, scale, blocks)
    for t, i in enumerate(blocks):
        assert check_selection_row(sel[i], S[t], cfg.mode, cfg.param, thr)[0], (b, h, i)
    Og = plan.O[b, h].float().cpu().numpy()
    Lg = plan.lse[b, h].cpu().numpy()
    pooled = P if cfg.compressed else None
    for i in blocks:
        o, l = orc.attn_video_block(q, k, v, ns, i, sel[i], pooled, scale, 64, cfg.q_tile, xs)
        rows = orc.tile_rows(i, nb * 64, cfg.q_tile)
        if perm is not None:
            rows = perm[rows]
        check_output(Og[rows], o, f"head {b},{h} tile {i}")
        check_lse(Lg[rows], l, f"head {b},{h} tile {i}")
    N = q.shape[0]
    if dense and N > nb * 64:
        rows = np.arange(nb * 64, N)
        o, l = orc.attn_dense_rows(q, k, v, rows, scale)
        check_output(Og[rows], o, f"head {b},{h} dense rows")
        check_lse(Lg[rows], l, f"head {b},{h} dense rows")


SMALL = [
    # d, n_video, n_sink, mode, param, compressed, pool_mode, extra, q_tile, q_offset
    (64, 1024, 32, "topk", 0.1, True, "reweight", 37, 64, 0.0),
    (128, 64 * 40, 100, "topk", 0.2, True, "reweight", 200, 64, 1.0),
    (128, 64 * 33 + 17, 64, "topk", 0.1, True, "mean", 64 * 3 + 5, 64, 0.0),
    (64, 64 * 50, 0, "tau", 1.0, True, "reweight", 500, 64, 1.0),
    (128, 64 * 40, 30, "tau", 1.5, False, "reweight", 130, 64, 0.0),
    (128, 64 * 40, 30, "topk", 0.1, True, "reweight", 200, 128, 1.0),
    (64, 64 * 21, 8, "topk", 0.25, True, "reweight", 64 * 21 + 100, 128, 0.0),  # every token extra
    (64, 64 * 31, 12, "topk", 0.1, False, "reweight", 64, 128, 0.0),
]


@pytest.mark.parametrize("d,nv,ns,mode,param,compressed,pool_mode,extra,q_tile,q_offset", SMALL)
def test_extra_tokens_every_element(spark, d, nv, ns, mode, param, compressed, pool_mode, extra, q_tile,
                                    q_offset):
    Q, K, V = make_qkv(1, 2, nv, ns, d, seed=17, q_offset=q_offset)
    cfg = spark.ForwardConfig(mode, param, compressed, pool_mode, q_tile=q_tile, extra_tokens=extra)
    plan = spark.SparkAttention(1, 2, nv + ns, d, ns, cfg, DEV)
    plan.run(Q.to(DEV), K.to(DEV), V.to(DEV))
    torch.cuda.synchronize()
    assert spark.device_error() == 0
    for h in range(2):
        compare_extra_head(spark, plan, Q, K, V, 0, h, ns, cfg)


def test_extra_tokens_behind_reblock(spark):
    Q, K, V = make_qkv(1, 2, 64 * 24, 20, 64, seed=23, q_offset=1.0)
    cfg = spark.ForwardConfig("topk", 0.15, True, reblock=True, extra_tokens=150)
    plan = spark.SparkAttention(1, 2, 64 * 24 + 20, 64, 20, cfg, DEV)
    plan.run(Q.to(DEV), K.to(DEV), V.to(DEV))
    torch.cuda.synchronize()
    assert spark.device_error() == 0
    for h in range(2):
        compare_extra_head(spark, plan, Q, K, V, 0, h, 20, cfg)


def test_extra_tokens_host_forward_is_bitwise_the_device_forward(spark):
    Q, K, V = make_qkv(2, 3, 64 * 30 + 9, 24, 128, seed=5, q_offset=1.0)
    cfg = spark.ForwardConfig("tau", 1.2, True, extra_tokens=321)
    plan = spark.SparkAttention(2, 3, Q.shape[2], 128, 24, cfg, DEV)
    O, L = plan.run(Q.to(DEV), K.to(DEV), V.to(DEV))
    torch.cuda.synchronize()
    hO = torch.empty(Q.shape, dtype=torch.bfloat16).pin_memory()
    hL = torch.empty(L.shape, dtype=torch.float32).pin_memory()
    plan.run_host(Q.pin_memory(), K.pin_memory(), V.pin_memory(), hO, hL, heads_per_group=2)
    torch.cuda.synchronize()
    assert spark.device_error() == 0
    assert torch.equal(hO, O.cpu()) and torch.equal(hL, L.cpu())


def test_extra_tokens_full_size_sampled(spark):
    B, H, nv, ns, d = 1, 3, 175680, 512, 128
    Q, K, V = make_qkv(B, H, nv, ns, d, seed=2, device=DEV, q_offset=1.0)
    cfg = spark.ForwardConfig("topk", 0.1, True, extra_tokens=512)
    plan = spark.SparkAttention(B, H, nv + ns, d, ns, cfg, DEV)
    plan.run(Q, K, V)
    torch.cuda.synchronize()
    assert spark.device_error() == 0
    Qc, Kc, Vc = Q.cpu(), K.cpu(), V.cpu()
    rng = np.random.default_rng(0)
    for h in (0, H - 1):
        blocks = np.unique(np.concatenate([[0, plan.nb - 1], rng.choice(plan.nb, 6, replace=False)]))
        compare_extra_head(spark, plan, Qc, Kc, Vc, 0, h, ns, cfg, qblocks=blocks, dense=(h == 0))
