"""The allocation-free selection entry point, for callers that cannot allocate device
memory themselves (an engine that owns one arena, a plugin inside another framework's
allocator, a loop that must never reach the driver's allocator).

spark_score_select_noalloc keeps its scratch in a fixed device array of the library. Its
selection and that of spark_score_select (caller scratch) are both checked, row by row,
against the fp64 oracle's selection of the same inputs on both query routes; it is called
twice in a row to show that the shared array is cleared between calls. This file runs
last so that a failure here leaves the rest of the suite already run."""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle.spark_oracle as orc
from block_sparse_video_mean_b200.inputs import make_qkv
from tests.parity import check_selection_row, gpu_rows

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def spark():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_video_mean_b200.spark as spark
    spark.load()
    return spark


def _check_against_oracle(sels, Q, K, V, ns, mode, param, q_tile):
    """Every row of every (idx, cnt) selection in ``sels`` against the fp64 oracle's
    selection of the same inputs (pooled by the oracle), up to near-ties."""
    B, H, N, d = Q.shape
    scale = 1.0 / math.sqrt(d)
    host = [(gi.cpu().numpy(), gc.cpu().numpy()) for gi, gc in sels]
    for b in range(B):
        for h in range(H):
            q, k, v = (orc.to_f64(t[b, h]) for t in (Q, K, V))
            P = orc.pool_head(q, k, v, ns, scale, 64, "reweight", q_tile)
            S = orc.block_scores(P.qbar, P.kbar, scale)
            thr = orc.tau_threshold(S, param) if mode == "tau" else None
            for gi, gc in host:
                sel = gpu_rows(gi[b, h], gc[b, h])
                assert len(sel) == S.shape[0]
                for i in range(S.shape[0]):
                    ok, ndiff = check_selection_row(sel[i], S[i], mode, param, thr)
                    assert ok, (b, h, i, ndiff)


@pytest.mark.parametrize("mode,param,q_tile", [("tau", 1.0, 64), ("tau", 2.0, 64), ("topk", 0.1, 64),
                                               ("topk", 0.1, 128), ("tau", 1.5, 128)])
def test_noalloc_matches_scratch_entry_point(spark, mode, param, q_tile):
    B, H, nv, ns, d = 1, 6, 64 * 301, 40, 128
    Q, K, V = make_qkv(B, H, nv, ns, d, seed=9)
    Qd, Kd, Vd = Q.to(DEV), K.to(DEV), V.to(DEV)
    pool = spark.pool_kv(Qd, Kd, Vd, ns, q_tile=q_tile)
    m = spark.SELECT_TAU if mode == "tau" else spark.SELECT_TOPK_RATIO
    ref = spark.score_select(pool["q_pool"], pool["k_pool"], ns, Q.shape[2], m, param, q_tile=q_tile)
    got = []
    for _ in range(2):  # twice in a row: the shared scratch must be cleared by each call
        sel = spark.score_select_noalloc(pool["q_pool"], pool["k_pool"], ns, Q.shape[2], m, param,
                                         q_tile=q_tile)
        torch.cuda.synchronize()
        assert spark.device_error() == 0
        got.append(tuple(t.clone() for t in sel))
    _check_against_oracle([ref] + got, Q, K, V, ns, mode, param, q_tile)


def test_noalloc_rejects_more_heads_than_its_scratch(spark):
    lib = spark.load()
    shape = spark.make_shape(1, spark.NOALLOC_MAX_HEADS + 1, 64 * 4, 64, 0)
    P = ctypes.c_void_p(16)  # never dereferenced: the size check comes first
    assert lib.spark_score_select_noalloc(ctypes.byref(shape), P, P, 1, 1.0, 4, P, P, None) == -7
