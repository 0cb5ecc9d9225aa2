"""GPU parity of the 128-query x 64-key route (q_tile = 128: M = 128 tensor-core tiles)
against the fp64 oracle: every element on small cases (odd nb: a one-block last tile;
ragged video tails; several dense 128-row items), sampled tiles at the full size the
benchmark times, the pipeline under many short items, Reblock in front of it, and the
device-side index check."""
import math

import numpy as np
import pytest
import torch

import oracle.spark_oracle as orc
from block_sparse_video_mean_b200.inputs import make_qkv
from tests.parity import check_lse, check_output, check_selection_row, gpu_rows
from tests.test_gpu_parity import DEV, compare_head, full_inputs, run_plan, sample_blocks

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def spark():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_video_mean_b200.spark as spark
    spark.load()
    return spark


SMALL = [
    # d, n_video, n_sink, mode, param, compressed, pool_mode
    (64, 1024, 32, "topk", 0.1, True, "reweight"),           # the tiny 4x16x16 + 32 sink workload
    (128, 64 * 33 + 17, 64, "topk", 0.1, True, "reweight"),  # odd nb, ragged video tail
    (64, 64 * 50, 0, "tau", 1.0, True, "reweight"),          # no sinks
    (128, 64 * 41, 30, "tau", 1.5, False, "reweight"),
    (64, 64 * 24, 16, "topk", 0.3, True, "mean"),
    (128, 64 * 21, 7, "topk", 1.0, False, "reweight"),       # full density: dense attention
    (64, 40, 24, "topk", 0.1, True, "reweight"),             # no full video block at all
    (128, 64 * 151, 300, "topk", 0.05, True, "reweight"),    # three dense items, one ragged
    (128, 64 * 3, 5, "topk", 0.5, True, "reweight"),         # two tiles, the last one block
]


@pytest.mark.parametrize("d,nv,ns,mode,param,compressed,pool_mode", SMALL)
def test_q128_small_every_element(spark, d, nv, ns, mode, param, compressed, pool_mode):
    Q, K, V = make_qkv(1, 2, nv, ns, d, seed=0)
    cfg = spark.ForwardConfig(mode, param, compressed, pool_mode, q_tile=128)
    plan, O, L = run_plan(spark, Q, K, V, ns, cfg)
    assert spark.device_error() == 0
    assert plan.nt == (plan.nb + 1) // 2
    for h in range(2):
        compare_head(plan, O, L, Q, K, V, 0, h, ns, cfg)


def test_q128_batch_and_heads_are_independent(spark):
    Q, K, V = make_qkv(2, 3, 64 * 13, 9, 64, seed=4)
    cfg = spark.ForwardConfig("topk", 0.25, True, q_tile=128)
    plan, O, L = run_plan(spark, Q, K, V, 9, cfg)
    for b in range(2):
        for h in range(3):
            compare_head(plan, O, L, Q, K, V, b, h, 9, cfg)


def test_q128_repeated_block_pairs_match_the_64_query_route(spark):
    """When each tile's second block repeats the first one's queries, both routes select
    the same blocks for every query and give the same outputs (up to the order in which
    the tensor cores add, so compared within the parity tolerance)."""
    nb, ns, d = 40, 24, 128
    Q, K, V = make_qkv(1, 2, nb * 64, ns, d, seed=8)
    Qv = Q[:, :, : nb * 64].reshape(1, 2, nb // 2, 2, 64, d)
    Qv[:, :, :, 1] = Qv[:, :, :, 0]
    Q[:, :, : nb * 64] = Qv.reshape(1, 2, nb * 64, d)
    c64 = spark.ForwardConfig("topk", 0.1, True)
    c128 = spark.ForwardConfig("topk", 0.1, True, q_tile=128)
    p64, O64, L64 = run_plan(spark, Q, K, V, ns, c64)
    O64, L64 = O64.clone(), L64.clone()
    p128, O128, L128 = run_plan(spark, Q, K, V, ns, c128)
    for h in range(2):
        q, k, v = (orc.to_f64(t[0, h]) for t in (Q, K, V))
        P = orc.pool_head(q, k, v, ns, 1 / math.sqrt(d))
        S64 = orc.block_scores(P.qbar, P.kbar, 1 / math.sqrt(d))
        s128 = gpu_rows(p128.idx[0, h].cpu().numpy(), p128.cnt[0, h].cpu().numpy())
        s64 = gpu_rows(p64.idx[0, h].cpu().numpy(), p64.cnt[0, h].cpu().numpy())
        for t in range(nb // 2):
            # the tile's kept set is the one of either of its blocks (up to near-ties)
            assert check_selection_row(s128[t], S64[2 * t], "topk", 0.1)[0], (h, t)
            assert check_selection_row(s64[2 * t + 1], S64[2 * t], "topk", 0.1)[0], (h, t)
        check_output(O128[0, h].float().cpu().numpy(), O64[0, h].float().cpu().numpy().astype(np.float64),
                     f"head {h}")


def test_q128_repeat_calls_are_bitwise_stable(spark):
    Q, K, V = make_qkv(1, 2, 64 * 31, 20, 128, seed=2)
    cfg = spark.ForwardConfig("topk", 0.1, True, q_tile=128)
    plan, O, L = run_plan(spark, Q, K, V, 20, cfg)
    O1, L1, idx1 = O.clone(), L.clone(), plan.idx.clone()
    plan.run(Q.to(DEV), K.to(DEV), V.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(O1, plan.O) and torch.equal(L1, plan.lse) and torch.equal(idx1, plan.idx)


def test_q128_many_items_stay_in_sync(spark):
    """Many short items per CTA, repeated: every pipeline barrier (ring, S/P buffers, the
    warp-pair exchanges, Q and O hand-over) must stay in phase, and the results must be
    bitwise stable."""
    Q, K, V = make_qkv(1, 6, 64 * 701, 40, 128, seed=7, device=DEV)
    cfg = spark.ForwardConfig("tau", 1.8, False, q_tile=128)   # 1-3 tiles per item
    plan = spark.SparkAttention(1, 6, Q.shape[2], 128, 40, cfg, DEV)
    O0, L0 = (t.clone() for t in plan.run(Q, K, V))
    for _ in range(15):
        plan.run(Q, K, V)
        torch.cuda.synchronize()
        assert spark.device_error() == 0
        assert torch.equal(plan.O, O0) and torch.equal(plan.lse, L0)
    Qc, Kc, Vc = Q.cpu(), K.cpu(), V.cpu()
    compare_head(plan, plan.O, plan.lse, Qc, Kc, Vc, 0, 5, 40, cfg, qblocks=sample_blocks(plan.nt, 6, 1))


@pytest.mark.parametrize("mode,param", [("topk", 0.1), ("tau", 1.5)])
def test_q128_full_size_sampled(spark, mode, param):
    (Q, K, V), ns = full_inputs("1152x640x243")
    B, H, N, d = Q.shape
    cfg = spark.ForwardConfig(mode, param, True, q_tile=128)
    plan = spark.SparkAttention(B, H, N, d, ns, cfg, DEV)
    O, L = plan.run(Q, K, V)
    torch.cuda.synchronize()
    assert spark.device_error() == 0
    Qc, Kc, Vc = Q.cpu(), K.cpu(), V.cpu()
    for h in (0, H - 1):
        compare_head(plan, O, L, Qc, Kc, Vc, 0, h, ns, cfg, qblocks=sample_blocks(plan.nt, 6, h),
                     check_pool=(h == 0), dense=(mode == "topk"))


def test_q128_out_of_range_index_is_skipped_and_reported(spark):
    Q, K, V = make_qkv(1, 1, 64 * 8, 8, 64, seed=3)
    Qd, Kd, Vd = Q.to(DEV), K.to(DEV), V.to(DEV)
    pool = spark.pool_kv(Qd, Kd, Vd, 8, q_tile=128)
    idx, cnt = spark.score_select(pool["q_pool"], pool["k_pool"], 8, Qd.shape[2],
                                  spark.SELECT_TOPK_RATIO, 0.25, q_tile=128)
    idx[0, 0, 1, 0] = 1000
    spark.attn_fwd(Qd, Kd, Vd, idx, cnt, 8, pool["pack"], pool["beta"], q_tile=128)
    assert spark.device_error() == -5
    assert spark.device_error() == 0


def test_q128_after_reblock_in_original_order(spark):
    """Reblock, then the 128-query route over the permuted tokens (a tile pairs two
    consecutive leaves); outputs land in the original token order."""
    nb, ns, d = 24, 16, 64
    Q, K, V = make_qkv(1, 2, nb * 64, ns, d, seed=9)
    cfg = spark.ForwardConfig("topk", 0.2, True, reblock=True, q_tile=128)
    plan, O, L = run_plan(spark, Q, K, V, ns, cfg)
    assert spark.device_error() == 0
    for h in range(2):
        q, k, v = (orc.to_f64(t[0, h]) for t in (Q, K, V))
        perm = plan.rb["perm"][0, h].cpu().numpy()
        sel = gpu_rows(plan.idx[0, h].cpu().numpy(), plan.cnt[0, h].cpu().numpy())
        qp, kp, vp = (orc.apply_perm(t, perm, ns) for t in (q, k, v))
        P = orc.pool_head(qp, kp, vp, ns, 1 / math.sqrt(d), 64, "reweight", 128)
        S = orc.block_scores(P.qbar, P.kbar, 1 / math.sqrt(d))
        for t in range(plan.nt):
            assert check_selection_row(sel[t], S[t], "topk", 0.2)[0], (h, t)
        Oo, Lo, _ = orc.forward_head(q, k, v, ns, "topk", 0.2, compressed=True, reblock=True,
                                     perm_override=perm, sel_override=sel, q_tile=128)
        check_output(O[0, h].float().cpu().numpy(), Oo, f"head {h}")
        check_lse(L[0, h].cpu().numpy(), Lo, f"head {h}")
