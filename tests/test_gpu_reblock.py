"""GPU parity of Spark-Reblock: the device partition against the fp64 oracle (exactly when
no node sits near a tie, by node replay otherwise), the gathered Q/K/V, and the reblocked
forward in the original token order."""
import math

import numpy as np
import pytest
import torch

import oracle.spark_oracle as orc
from block_sparse_video_mean_b200.inputs import make_qkv
from tests.parity import (check_lse, check_output, check_partition, gpu_rows,
                          replay_reblock_tree)

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def spark():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_video_mean_b200.spark as spark
    spark.load()
    return spark


@pytest.mark.parametrize("d,nb,ns,H", [(64, 1, 8, 1), (64, 2, 0, 2), (128, 3, 16, 2), (64, 5, 3, 2),
                                       (128, 13, 40, 2), (64, 40, 10, 1), (128, 70, 64, 1)])
def test_reblock_small(spark, d, nb, ns, H):
    nv = 64 * nb
    Q, K, V = make_qkv(1, H, nv, ns, d, seed=nb)
    out = spark.reblock(Q.to(DEV), K.to(DEV), V.to(DEV), ns, tree=True)
    torch.cuda.synchronize()
    assert spark.device_error() == 0
    L = orc.n_levels(nb)
    for h in range(H):
        q, k, v = (orc.to_f64(t[0, h]) for t in (Q, K, V))
        perm = out["perm"][0, h].cpu().numpy()
        check_partition(perm, nv)
        tree = out["tree"][0, h].cpu().numpy()
        assert tree.shape == (L + 1, nv) and np.all(tree[0] == 0)
        x = orc.whiten(q[:nv], orc.key_second_moment(k[:nv]))
        replay_reblock_tree(x, tree, L)
        ref = orc.reblock_head(q, k, ns)
        # no node near a tie in the oracle's own tree -> identical partition
        near = any(sp.gap < 1e-3 or min(abs(p - sp.split_value) for p in sp.proj.values()) < 1e-4
                   for sp in ref.splits.values())
        if not near:
            assert np.array_equal(perm, ref.perm)
        # gathered rows
        for name, T in (("Qp", Q), ("Kp", K), ("Vp", V)):
            got = out[name][0, h].cpu()
            exp = torch.cat([T[0, h][torch.from_numpy(perm).long()], T[0, h][nv:]])
            assert torch.equal(got, exp), name


def test_reblocked_forward_in_original_order(spark):
    nb, ns, d = 30, 20, 128
    Q, K, V = make_qkv(1, 2, 64 * nb, ns, d, seed=11)
    cfg = spark.ForwardConfig("topk", 0.2, True, reblock=True)
    plan = spark.SparkAttention(1, 2, Q.shape[2], d, ns, cfg, DEV)
    O, Lse = plan.run(Q.to(DEV), K.to(DEV), V.to(DEV))
    torch.cuda.synchronize()
    assert spark.device_error() == 0
    for h in range(2):
        q, k, v = (orc.to_f64(t[0, h]) for t in (Q, K, V))
        perm = plan.rb["perm"][0, h].cpu().numpy()
        sel = gpu_rows(plan.idx[0, h].cpu().numpy(), plan.cnt[0, h].cpu().numpy())
        ref, lref, _ = orc.forward_head(q, k, v, ns, "topk", 0.2, True, reblock=True,
                                        perm_override=perm, sel_override=sel)
        check_output(O[0, h].float().cpu().numpy(), ref, f"head {h}")
        check_lse(Lse[0, h].cpu().numpy(), lref, f"head {h}")


def test_reblock_repeat_is_deterministic(spark):
    Q, K, V = make_qkv(1, 2, 64 * 90, 8, 128, seed=3, device=DEV)
    a = spark.reblock(Q, K, V, 8, tree=True)
    pa, ta = a["perm"].clone(), a["tree"].clone()
    b = spark.reblock(Q, K, V, 8, tree=True)
    torch.cuda.synchronize()
    assert torch.equal(pa, b["perm"]) and torch.equal(ta, b["tree"])


@pytest.mark.slow
def test_reblock_full_size_sampled(spark):
    """1344x768, 240 frames: 61 x 84 x 48 = 245,952 video tokens + 512 sinks, 24 heads; the
    launch configuration of the reblocked forward. Replays the root and a sample of nodes
    at every level of two heads and checks sampled output blocks."""
    B, H, nv, ns, d = 1, 24, 245952, 512, 128
    Q, K, V = make_qkv(B, H, nv, ns, d, seed=0, device=DEV)
    cfg = spark.ForwardConfig("topk", 0.1, True, reblock=True)
    plan = spark.SparkAttention(B, H, nv + ns, d, ns, cfg, DEV)
    plan.rb["tree"] = torch.empty((B, H, plan.levels + 1, nv), dtype=torch.int32, device=DEV)
    O, Lse = plan.run(Q, K, V)
    torch.cuda.synchronize()
    assert spark.device_error() == 0
    rng = np.random.default_rng(0)
    for h in (0, H - 1):
        perm = plan.rb["perm"][0, h].cpu().numpy()
        check_partition(perm, nv)
        tree = plan.rb["tree"][0, h].cpu().numpy()
        q, k, v = (orc.to_f64(t[0, h].cpu()) for t in (Q, K, V))
        x = orc.whiten(q[:nv], orc.key_second_moment(k[:nv]))
        nodes = []
        for lev in range(plan.levels):
            labels = np.unique(tree[lev])
            nodes += [(lev, int(c)) for c in rng.choice(labels, min(3, labels.size), replace=False)]
        checked, skipped = replay_reblock_tree(x, tree, plan.levels, nodes)
        assert checked >= plan.levels
        sel = gpu_rows(plan.idx[0, h].cpu().numpy(), plan.cnt[0, h].cpu().numpy())
        blocks = np.unique(rng.choice(plan.nb, 4, replace=False))
        ref, lref, _ = orc.forward_head(q, k, v, ns, "topk", 0.1, True, reblock=True, perm_override=perm,
                                        qblocks=blocks, sel_override=[sel[i] for i in blocks])
        rows = np.concatenate([perm[i * 64:(i + 1) * 64] for i in blocks])
        check_output(O[0, h].float().cpu().numpy()[rows], ref[rows], f"head {h}")
        check_lse(Lse[0, h].cpu().numpy()[rows], lref[rows], f"head {h}")


# ---------------------------------------------------------------- keys on their own partition
@pytest.mark.parametrize("d,nb,ns,H", [(64, 5, 3, 2), (128, 13, 40, 2), (128, 70, 64, 1)])
def test_reblock_kv_small(spark, d, nb, ns, H):
    """perm_q is the q_reuse_k partition, perm_k the same construction with Q and K swapped
    (node replay against the oracle through the swapped call's tree); Qp follows perm_q,
    Kp and Vp follow perm_k."""
    nv = 64 * nb
    Q, K, V = make_qkv(1, H, nv, ns, d, seed=100 + nb)
    Qd, Kd, Vd = Q.to(DEV), K.to(DEV), V.to(DEV)
    out = spark.reblock_kv(Qd, Kd, Vd, ns)
    ref_q = spark.reblock(Qd, Kd, Vd, ns)
    ref_k = spark.reblock(Kd, Qd, Vd, ns, tree=True)  # keys partitioned, whitened by queries
    torch.cuda.synchronize()
    assert spark.device_error() == 0
    L = orc.n_levels(nb)
    for h in range(H):
        q, k, v = (orc.to_f64(t[0, h]) for t in (Q, K, V))
        pq = out["perm"][0, h].cpu().numpy()
        pk = out["perm_k"][0, h].cpu().numpy()
        assert np.array_equal(pq, ref_q["perm"][0, h].cpu().numpy())
        assert np.array_equal(pk, ref_k["perm"][0, h].cpu().numpy())
        check_partition(pk, nv)
        x = orc.whiten(k[:nv], orc.key_second_moment(q[:nv]))
        replay_reblock_tree(x, ref_k["tree"][0, h].cpu().numpy(), L)
        for name, T, pp in (("Qp", Q, pq), ("Kp", K, pk), ("Vp", V, pk)):
            got = out[name][0, h].cpu()
            exp = torch.cat([T[0, h][torch.from_numpy(pp).long()], T[0, h][nv:]])
            assert torch.equal(got, exp), name


def test_reblock_kv_forward_in_original_order(spark):
    nb, ns, d = 30, 20, 128
    Q, K, V = make_qkv(1, 2, 64 * nb, ns, d, seed=12)
    cfg = spark.ForwardConfig("topk", 0.2, True, reblock=True, reblock_kv=True)
    plan = spark.SparkAttention(1, 2, Q.shape[2], d, ns, cfg, DEV)
    O, Lse = plan.run(Q.to(DEV), K.to(DEV), V.to(DEV))
    torch.cuda.synchronize()
    assert spark.device_error() == 0
    for h in range(2):
        q, k, v = (orc.to_f64(t[0, h]) for t in (Q, K, V))
        pq = plan.rb["perm"][0, h].cpu().numpy()
        pk = plan.rb["perm_k"][0, h].cpu().numpy()
        sel = gpu_rows(plan.idx[0, h].cpu().numpy(), plan.cnt[0, h].cpu().numpy())
        ref, lref, _ = orc.forward_head(q, k, v, ns, "topk", 0.2, True, reblock=True, reblock_kv=True,
                                        perm_override=pq, perm_k_override=pk, sel_override=sel)
        check_output(O[0, h].float().cpu().numpy(), ref, f"head {h}")
        check_lse(Lse[0, h].cpu().numpy(), lref, f"head {h}")
