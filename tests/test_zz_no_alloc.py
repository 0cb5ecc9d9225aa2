"""The allocation-free selection entry point, for callers that cannot allocate device
memory themselves (an engine that owns one arena, a plugin inside another framework's
allocator, a loop that must never reach the driver's allocator).

spark_score_select_noalloc keeps its scratch in a fixed device array of the library and
must select exactly what spark_score_select selects with caller scratch; it is called
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


def _same_selection(a, b, q_pool, k_pool, mode, param, d):
    """Identical, or different only at near-ties (the suite's selection tolerance)."""
    ia, ca = (t.cpu().numpy() for t in a)
    ib, cb = (t.cpu().numpy() for t in b)
    B, H, nb = ca.shape
    scale = 1.0 / math.sqrt(d)
    for bb in range(B):
        for h in range(H):
            ra, rb = gpu_rows(ia[bb, h], ca[bb, h]), gpu_rows(ib[bb, h], cb[bb, h])
            if all(np.array_equal(x, y) for x, y in zip(ra, rb)):
                continue
            qp = q_pool[bb, h].cpu().double().numpy()
            kp = k_pool[bb, h].cpu().double().numpy()
            S = orc.block_scores(qp, kp, scale)
            thr = orc.tau_threshold(S, param) if mode == "tau" else None
            for i in range(nb):
                assert check_selection_row(rb[i], S[i], mode, param, thr)[0], (bb, h, i)


@pytest.mark.parametrize("mode,param", [("tau", 1.0), ("tau", 2.0), ("topk", 0.1)])
def test_noalloc_matches_scratch_entry_point(spark, mode, param):
    B, H, nv, ns, d = 1, 6, 64 * 300, 40, 128
    Q, K, V = make_qkv(B, H, nv, ns, d, seed=9, device=DEV)
    pool = spark.pool_kv(Q, K, V, ns)
    m = spark.SELECT_TAU if mode == "tau" else spark.SELECT_TOPK_RATIO
    ref = spark.score_select(pool["q_pool"], pool["k_pool"], ns, Q.shape[2], m, param)
    for _ in range(2):  # twice in a row: the shared scratch must be cleared by each call
        got = spark.score_select_noalloc(pool["q_pool"], pool["k_pool"], ns, Q.shape[2], m, param)
        torch.cuda.synchronize()
        assert spark.device_error() == 0
        _same_selection(ref, got, pool["q_pool"], pool["k_pool"], mode, param, d)


def test_noalloc_rejects_more_heads_than_its_scratch(spark):
    lib = spark.load()
    shape = spark.make_shape(1, spark.NOALLOC_MAX_HEADS + 1, 64 * 4, 64, 0)
    P = ctypes.c_void_p(16)  # never dereferenced: the size check comes first
    assert lib.spark_score_select_noalloc(ctypes.byref(shape), P, P, 1, 1.0, 4, P, P, None) == -7
