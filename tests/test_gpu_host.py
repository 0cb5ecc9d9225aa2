"""GPU checks of the forward from host memory (spark_forward_host): the heads are cut into
groups whose copies overlap the neighbouring groups' compute, and since every step of the
method is per (b, h) the result must be bit for bit the device forward's, which the other
GPU tests pin to the fp64 oracle. One case is also compared with the oracle directly."""
import pytest
import torch

from block_sparse_video_mean_b200.inputs import make_qkv
from tests.test_gpu_parity import DEV, compare_head

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def spark():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_sparse_video_mean_b200.spark as spark
    spark.load()
    return spark


def device_and_host(spark, Q, K, V, ns, cfg, heads_per_group):
    B, H, N, d = Q.shape
    plan = spark.SparkAttention(B, H, N, d, ns, cfg, DEV)
    O, L = plan.run(Q.to(DEV), K.to(DEV), V.to(DEV))
    O, L = O.cpu(), L.cpu()
    hQ, hK, hV = (t.contiguous().pin_memory() for t in (Q, K, V))
    hO = torch.full(Q.shape, 7.0, dtype=torch.bfloat16).pin_memory()
    hL = torch.full((B, H, N), 7.0, dtype=torch.float32).pin_memory()
    plan.run_host(hQ, hK, hV, hO, hL, heads_per_group=heads_per_group)
    torch.cuda.synchronize()
    assert spark.device_error() == 0
    return plan, O, L, hO, hL


CASES = [
    # B, H, d, n_video, n_sink, mode, param, compressed, q_tile, heads_per_group
    (2, 3, 64, 64 * 20 + 9, 16, "topk", 0.1, True, 64, 0),     # auto: the 6 small heads in one group
    (2, 3, 128, 64 * 17, 40, "tau", 1.0, True, 64, 4),          # a ragged last group of 2
    (1, 5, 128, 64 * 33 + 17, 64, "topk", 0.2, True, 128, 2),   # 128-query route
    (1, 4, 64, 64 * 12, 0, "topk", 0.3, False, 64, 3),          # no sinks, no compression
    (3, 1, 128, 64 * 9, 8, "tau", 1.5, True, 128, 8),           # one group larger than B*H
    (1, 2, 64, 40, 24, "topk", 0.1, True, 64, 1),               # no full video block
]


@pytest.mark.parametrize("B,H,d,nv,ns,mode,param,compressed,qt,hpg", CASES)
def test_host_forward_equals_device_forward_bitwise(spark, B, H, d, nv, ns, mode, param, compressed,
                                                    qt, hpg):
    Q, K, V = make_qkv(B, H, nv, ns, d, seed=11)
    cfg = spark.ForwardConfig(mode, param, compressed, q_tile=qt)
    _, O, L, hO, hL = device_and_host(spark, Q, K, V, ns, cfg, hpg)
    assert torch.equal(hO.view(torch.int16), O.view(torch.int16))
    assert torch.equal(hL, L) or torch.equal(hL.nan_to_num(), L.nan_to_num())


def test_host_forward_with_reblock_equals_device_forward(spark):
    # nb <= 64 runs the deterministic single-CTA subtree path, so the runs agree bit for bit
    Q, K, V = make_qkv(1, 3, 64 * 24, 12, 128, seed=5)
    for kv in (False, True):
        cfg = spark.ForwardConfig("topk", 0.25, True, reblock=True, reblock_kv=kv)
        _, O, L, hO, hL = device_and_host(spark, Q, K, V, 12, cfg, 2)
        assert torch.equal(hO.view(torch.int16), O.view(torch.int16))
        assert torch.equal(hL, L)


def test_host_forward_matches_the_oracle(spark):
    Q, K, V = make_qkv(1, 3, 64 * 21 + 5, 20, 64, seed=2)
    cfg = spark.ForwardConfig("topk", 0.15, True)
    plan, _, _, hO, hL = device_and_host(spark, Q, K, V, 20, cfg, 2)
    for h in range(3):
        compare_head(plan, hO, hL, Q, K, V, 0, h, 20, cfg, check_pool=False)


def test_host_forward_twice_on_one_workspace(spark):
    # back-to-back calls reuse the staging slots; the second must not overwrite the first's
    # inputs or outputs while they are in flight
    Q, K, V = make_qkv(1, 6, 64 * 30, 10, 64, seed=3)
    Q2, K2, V2 = make_qkv(1, 6, 64 * 30, 10, 64, seed=4)
    cfg = spark.ForwardConfig("topk", 0.1, True)
    plan = spark.SparkAttention(1, 6, Q.shape[2], 64, 10, cfg, DEV)
    O1 = plan.run(Q.to(DEV), K.to(DEV), V.to(DEV))[0].cpu()
    O2 = plan.run(Q2.to(DEV), K2.to(DEV), V2.to(DEV))[0].cpu()
    hs = [tuple(t.pin_memory() for t in x) for x in ((Q, K, V), (Q2, K2, V2))]
    outs = [torch.empty(Q.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    for (a, b, c), o in zip(hs, outs):
        plan.run_host(a, b, c, o, heads_per_group=2)
    torch.cuda.synchronize()
    assert torch.equal(outs[0].view(torch.int16), O1.view(torch.int16))
    assert torch.equal(outs[1].view(torch.int16), O2.view(torch.int16))


@pytest.mark.parametrize("q_tile", [64, 128])
def test_host_forward_full_size_equals_device_forward(spark, q_tile):
    # the configuration the benchmark's end-to-end leg times: 1152x640x243, 24 heads,
    # top-k 10% with the compressed branch, automatic groups (one head at a time)
    from tests.test_gpu_parity import full_inputs
    (Q, K, V), ns = full_inputs("1152x640x243")
    B, H, N, d = Q.shape
    cfg = spark.ForwardConfig("topk", 0.1, True, q_tile=q_tile)
    plan = spark.SparkAttention(B, H, N, d, ns, cfg, DEV)
    O, L = plan.run(Q, K, V)
    O, L = O.cpu(), L.cpu()
    hQ, hK, hV = (t.cpu().pin_memory() for t in (Q, K, V))
    del Q, K, V
    hO = torch.empty(O.shape, dtype=torch.bfloat16).pin_memory()
    hL = torch.empty(L.shape, dtype=torch.float32).pin_memory()
    plan.run_host(hQ, hK, hV, hO, hL)
    torch.cuda.synchronize()
    assert spark.device_error() == 0
    assert torch.equal(hO.view(torch.int16), O.view(torch.int16))
    assert torch.equal(hL, L)
