"""Failure detection without a GPU fault: the attention kernels' pipeline waits are
bounded, and a wait that runs out must end the launch cleanly with SPARK_ETIMEOUT in the
device error word, leaving the device usable.

The test shortens the limit of every pipeline wait to a few hundred clocks (far below
the time one tile's MMAs take), so the first waits of the launch give up; the drains of
copies and MMAs still in flight keep their own full limit. It then restores the default
and checks that a normal forward on the same process and device matches the fp64
oracle."""
import numpy as np
import pytest
import torch

from block_sparse_video_mean_b200.inputs import make_qkv
from tests.test_gpu_parity import DEV, compare_head, run_plan

pytestmark = pytest.mark.gpu

SPARK_ETIMEOUT = -4


@pytest.fixture(scope="module")
def spark():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_video_mean_b200.spark as spark
    spark.load()
    return spark


@pytest.mark.parametrize("q_tile", [64, 128])
def test_short_wait_limit_gives_up_then_device_recovers(spark, q_tile):
    ns = 48
    Q, K, V = make_qkv(1, 2, 64 * 40, ns, 128, seed=13)
    cfg = spark.ForwardConfig("topk", 0.2, True, q_tile=q_tile)
    assert spark.device_error() == 0
    spark.set_wait_limit(300)
    try:
        run_plan(spark, Q, K, V, ns, cfg)
        torch.cuda.synchronize()
        assert spark.device_error() == SPARK_ETIMEOUT
    finally:
        spark.set_wait_limit(0)
    assert spark.device_error() == 0   # the word was cleared by the read
    plan, O, L = run_plan(spark, Q, K, V, ns, cfg)
    assert spark.device_error() == 0
    assert torch.isfinite(O.float()).all()
    for h in range(2):
        compare_head(plan, O, L, Q, K, V, 0, h, ns, cfg)
    # repeated give-ups do not wear anything out
    spark.set_wait_limit(300)
    try:
        for _ in range(3):
            run_plan(spark, Q, K, V, ns, cfg)
            assert spark.device_error() == SPARK_ETIMEOUT
    finally:
        spark.set_wait_limit(0)
    plan2, O2, L2 = run_plan(spark, Q, K, V, ns, cfg)
    assert spark.device_error() == 0
    assert torch.equal(O2, O) and np.array_equal(L2.cpu().numpy(), L.cpu().numpy())
