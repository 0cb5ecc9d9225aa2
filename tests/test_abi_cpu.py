"""Host-side checks of the C ABI (no GPU): the library builds and loads, exports every
entry point that include/spark.h declares, and rejects bad arguments before launching."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spark.h")


@pytest.fixture(scope="module")
def spark():
    from block_sparse_video_mean_b200 import build
    build.build()
    import block_sparse_video_mean_b200.spark as spark
    spark.load()
    return spark


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(spark_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(spark):
    lib = spark.load()
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert set(spark.EXPORTS) <= set(names)


def test_topk_count_matches_fixture(spark):
    path = os.path.join(ROOT, "tests", "golden", "topk_count.txt")
    for ln in open(path):
        if ln.strip() and not ln.startswith("#"):
            r, nb, k = ln.split()
            assert spark.topk_count(float(r), int(nb)) == int(k), ln
    assert spark.topk_count(0.0, 10) == -1
    assert spark.topk_count(1.5, 10) == -1


def test_num_blocks_and_workspace(spark):
    s = spark.make_shape(1, 24, 175680 + 512, 128, 512)
    assert spark.num_blocks(s) == 2745
    # bf16 k_pool and v_summ, then beta*log2(e) padded to 2752 = 43 x 64 entries per head
    assert spark.workspace_bytes(s, spark.CALL_POOL) == 2 * 24 * 2745 * 128 * 2 + 24 * 2752 * 4
    assert spark.workspace_bytes(s, spark.CALL_ATTN) == 256   # the item counter
    ragged = spark.make_shape(1, 1, 64 * 3 + 17 + 5, 64, 5)
    assert spark.num_blocks(ragged) == 3
    assert spark.num_blocks(spark.make_shape(1, 1, 40, 64, 8)) == 0


def test_query_tiles_of_the_128_query_route(spark):
    s64 = spark.make_shape(1, 24, 175680 + 512, 128, 512)
    s128 = spark.make_shape(1, 24, 175680 + 512, 128, 512, q_tile=128)
    assert spark.num_query_tiles(s64) == 2745
    assert spark.num_query_tiles(s128) == 1373          # the last tile holds one block
    assert spark.num_query_tiles(spark.make_shape(1, 1, 64 * 4, 64, 0, q_tile=128)) == 2
    # key-side buffers do not change; the score keys have one row per tile
    assert spark.workspace_bytes(s128, spark.CALL_POOL) == spark.workspace_bytes(s64, spark.CALL_POOL)
    off = (2 * 24 * 8 + 255) // 256 * 256
    assert spark.workspace_bytes(s128, spark.CALL_SELECT) == off + 24 * 1373 * 2748 * 4
    assert spark.workspace_bytes(s64, spark.CALL_SELECT) == off + 24 * 2745 * 2748 * 4
    lib = spark.load()
    bad_tile = spark.make_shape(1, 1, 128, 64, 0, q_tile=96)
    dummy = ctypes.c_void_p(16)
    assert lib.spark_attn_fwd(ctypes.byref(bad_tile), dummy, dummy, dummy, dummy, dummy, 1, None,
                              None, None, None, 0, dummy, None, None, 0, None) == -2
    assert spark.num_query_tiles(bad_tile) == 0


def test_bad_arguments_are_rejected_on_the_host(spark):
    lib = spark.load()
    P = ctypes.c_void_p
    dummy = P(16)  # never dereferenced: validation fails first
    bad_d = spark.make_shape(1, 1, 128, 96, 0)
    assert lib.spark_pool_kv(ctypes.byref(bad_d), dummy, dummy, dummy, 0, dummy, dummy, dummy,
                             dummy, dummy, dummy, 1 << 20, None) == -2
    bad_block = spark.Shape(1, 1, 128, 64, 0, 32, 0.0, 0)
    assert lib.spark_attn_fwd(ctypes.byref(bad_block), dummy, dummy, dummy, dummy, dummy, 1, None,
                              None, None, None, 0, dummy, None, None, 0, None) == -2
    neg = spark.make_shape(1, 1, 128, 64, 200)
    assert lib.spark_attn_fwd(ctypes.byref(neg), dummy, dummy, dummy, dummy, dummy, 1, None, None,
                              None, None, 0, dummy, None, None, 0, None) == -1
    ok = spark.make_shape(1, 1, 128, 64, 0)
    # null inputs, misaligned pointers, bad ratio, kcap below k, unknown mode, bad pool mode
    assert lib.spark_pool_kv(ctypes.byref(ok), None, dummy, dummy, 0, dummy, dummy, dummy, dummy,
                             dummy, dummy, 1 << 20, None) == -1
    assert lib.spark_pool_kv(ctypes.byref(ok), P(18), dummy, dummy, 0, dummy, dummy, dummy, dummy,
                             dummy, dummy, 1 << 20, None) == -1
    assert lib.spark_pool_kv(ctypes.byref(ok), dummy, dummy, dummy, 7, dummy, dummy, dummy, dummy,
                             dummy, dummy, 1 << 20, None) == -1
    assert lib.spark_score_select(ctypes.byref(ok), dummy, dummy, 0, 1.5, 2, dummy, dummy, None, 0,
                                  None) == -1
    assert lib.spark_score_select(ctypes.byref(ok), dummy, dummy, 0, 0.5, 0, dummy, dummy, None, 0,
                                  None) == -1
    assert lib.spark_score_select(ctypes.byref(ok), dummy, dummy, 5, 0.5, 2, dummy, dummy, None, 0,
                                  None) == -1
    assert lib.spark_score_select(ctypes.byref(ok), dummy, dummy, 1, float("nan"), 2, dummy, dummy,
                                  dummy, 1 << 10, None) == -1
    # tau needs its workspace
    assert lib.spark_score_select(ctypes.byref(ok), dummy, dummy, 1, 1.0, 2, dummy, dummy, None, 0,
                                  None) == -1
    assert lib.spark_reblock(ctypes.byref(ok), dummy, dummy, dummy, None, dummy, dummy, dummy, None,
                             dummy, 1 << 30, None) == -1
    # the attention call needs its item-counter workspace
    assert lib.spark_attn_fwd(ctypes.byref(ok), dummy, dummy, dummy, dummy, dummy, 1, None, None,
                              None, None, 0, dummy, None, None, 0, None) == -1
    assert lib.spark_attn_fwd(ctypes.byref(ok), dummy, dummy, dummy, dummy, dummy, 1, None, None,
                              None, None, 0, dummy, None, dummy, 64, None) == -1


def test_extra_token_arguments_are_checked_on_the_host(spark):
    lib = spark.load()
    dummy = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    s = spark.make_shape(1, 2, 64 * 10 + 7, 64, 7)
    # layout: xidx [2, 64] int32, scores [2, 640] fp32, K and V rows [2 * 64, 64] bf16, each
    # part on a 256-byte boundary
    assert spark.extra_pack_bytes(s, 37) == 512 + 5120 + 16384 + 16384
    assert spark.extra_pack_bytes(s, 0) == 0
    assert spark.extra_pack_bytes(s, 10 ** 6) == spark.extra_pack_bytes(s, 640)
    need = spark.extra_pack_bytes(s, 37)
    assert lib.spark_extra_tokens(ctypes.byref(s), dummy, dummy, dummy, -1, 0, None, None, None, 0,
                                  dummy, need, None) == -1
    assert lib.spark_extra_tokens(ctypes.byref(s), dummy, dummy, dummy, 37, 0, None, None, None, 0,
                                  dummy, need - 16, None) == -1
    assert lib.spark_extra_tokens(ctypes.byref(s), dummy, dummy, dummy, 37, 3, None, None, None, 0,
                                  dummy, need, None) == -1
    assert lib.spark_extra_tokens(ctypes.byref(s), dummy, dummy, None, 37, 0, None, None, None, 0,
                                  dummy, need, None) == -1
    assert lib.spark_extra_tokens(ctypes.byref(s), dummy, dummy, dummy, 0, 0, None, None, None, 0,
                                  None, 0, None) == 0          # nothing to do
    assert lib.spark_attn_fwd(ctypes.byref(s), dummy, dummy, dummy, dummy, dummy, 1, None, None,
                              None, None, -3, dummy, None, dummy, 256, None) == -1
    assert lib.spark_attn_fwd(ctypes.byref(s), dummy, dummy, dummy, dummy, dummy, 1, None, None,
                              None, None, 37, dummy, None, dummy, 256, None) == -1   # no pack
    cfg = spark.fwd_config(extra_tokens=-2)
    assert spark.forward_host_workspace_bytes(s, cfg) == 0


def test_empty_inputs_are_a_no_op(spark):
    lib = spark.load()
    empty = spark.make_shape(0, 4, 128, 64, 0)
    assert lib.spark_attn_fwd(ctypes.byref(empty), None, None, None, None, None, 1, None, None,
                              None, None, 0, None, None, None, 0, None) == 0
    zero_n = spark.make_shape(1, 4, 0, 64, 0)
    assert lib.spark_pool_kv(ctypes.byref(zero_n), None, None, None, 0, None, None, None, None,
                             None, None, 0, None) == 0


def test_strerror(spark):
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert spark.strerror(code) and spark.strerror(code) != "unknown status"


def test_host_forward_config_and_workspace(spark):
    assert ctypes.sizeof(spark.FwdConfig) == 40   # double + 7 int32, padded to 8 bytes
    s = spark.make_shape(2, 3, 64 * 10 + 7 + 16, 64, 16)
    nb, N, d = 10, 64 * 10 + 7 + 16, 64
    cfg = spark.fwd_config(heads_per_group=2)
    ws = spark.forward_host_workspace_bytes(s, cfg)

    def up(x):
        return (x + 255) // 256 * 256
    G = 2
    g = spark.make_shape(1, G, N, d, 16)
    slots = 2 * (4 * up(G * N * d * 2) + up(G * N * 4))
    k = spark.topk_count(0.1, nb)
    inter = (up(G * nb * d * 4) + 2 * up(G * nb * d * 4) + up(G * nb * 4) + up(G * d * 4)
             + up(spark.workspace_bytes(g, spark.CALL_POOL)) + up(G * nb * k * 4) + up(G * nb * 4)
             + up(spark.workspace_bytes(g, spark.CALL_SELECT)) + up(256))
    assert ws == slots + inter
    # extra tokens add the extra pack of one group
    ex = spark.forward_host_workspace_bytes(s, spark.fwd_config(heads_per_group=2, extra_tokens=37))
    assert ex == ws + up(spark.extra_pack_bytes(g, 37))
    # reblock adds the permutation, the permuted copies and its own scratch
    rb = spark.forward_host_workspace_bytes(s, spark.fwd_config(heads_per_group=2, reblock=1))
    assert rb == ws + up(G * nb * 64 * 4) + 3 * up(G * N * d * 2) + up(spark.workspace_bytes(g, spark.CALL_REBLOCK))
    # automatic groups hold at least 32 MiB of Q/K/V (capped at B*H): all 6 small heads here,
    # one head at a time at video size; one group never exceeds B*H
    auto = spark.forward_host_workspace_bytes(s, spark.fwd_config())
    assert auto == spark.forward_host_workspace_bytes(s, spark.fwd_config(heads_per_group=6))
    video = spark.make_shape(1, 24, 175680 + 512, 128, 512)
    assert (spark.forward_host_workspace_bytes(video, spark.fwd_config())
            == spark.forward_host_workspace_bytes(video, spark.fwd_config(heads_per_group=1)))
    # with Reblock, automatic groups hold at least 8 heads (its first levels need the CTAs)
    assert (spark.forward_host_workspace_bytes(video, spark.fwd_config(reblock=1))
            == spark.forward_host_workspace_bytes(video, spark.fwd_config(reblock=1, heads_per_group=8)))
    mid = spark.make_shape(1, 24, 4096, 64, 0)   # 1.5 MiB of Q/K/V per head: 22 heads
    assert (spark.forward_host_workspace_bytes(mid, spark.fwd_config())
            == spark.forward_host_workspace_bytes(mid, spark.fwd_config(heads_per_group=22)))
    big = spark.forward_host_workspace_bytes(s, spark.fwd_config(heads_per_group=100))
    assert big == spark.forward_host_workspace_bytes(s, spark.fwd_config(heads_per_group=6))
    # invalid configurations size to 0
    for bad in (spark.fwd_config(mode=7), spark.fwd_config(pool_mode=3), spark.fwd_config(reblock=3),
                spark.fwd_config(param=0.0), spark.fwd_config(param=float("nan"))):
        assert spark.forward_host_workspace_bytes(s, bad) == 0


def test_host_forward_rejects_bad_arguments_before_any_cuda_call(spark):
    lib = spark.load()
    s = spark.make_shape(1, 2, 64 * 4 + 8, 64, 8)
    cfg = spark.fwd_config()
    need = spark.forward_host_workspace_bytes(s, cfg)
    host = (ctypes.c_uint16 * 16)()
    h = ctypes.cast(host, ctypes.c_void_p)
    ws = ctypes.c_void_p(4096)  # never dereferenced: validation fails first
    assert lib.spark_forward_host(ctypes.byref(s), ctypes.byref(cfg), None, h, h, h, None, ws, need, None) == -1
    assert lib.spark_forward_host(ctypes.byref(s), ctypes.byref(cfg), h, h, h, h, None, None, need, None) == -1
    assert lib.spark_forward_host(ctypes.byref(s), ctypes.byref(cfg), h, h, h, h, None, ws, need - 1, None) == -1
    assert lib.spark_forward_host(ctypes.byref(s), ctypes.byref(cfg), h, h, h, h, None,
                                  ctypes.c_void_p(4096 + 16), need, None) == -1   # not 256-aligned
    assert lib.spark_forward_host(ctypes.byref(s), None, h, h, h, h, None, ws, need, None) == -1
    bad_d = spark.make_shape(1, 2, 64 * 4 + 8, 96, 8)
    assert lib.spark_forward_host(ctypes.byref(bad_d), ctypes.byref(cfg), h, h, h, h, None, ws, need, None) == -2
    empty = spark.make_shape(0, 2, 64, 64, 0)
    assert lib.spark_forward_host(ctypes.byref(empty), ctypes.byref(cfg), None, None, None, None, None,
                                  None, 0, None) == 0


def test_host_forward_binding_rejects_bad_host_tensors(spark):
    import torch
    s = spark.make_shape(1, 2, 64 * 4 + 8, 64, 8)
    cfg = spark.fwd_config()
    good = torch.zeros((1, 2, 64 * 4 + 8, 64), dtype=torch.bfloat16)
    for bad in (good.float(), good.transpose(2, 3), good[:, :, ::2]):
        with pytest.raises(ValueError):
            spark.forward_host(bad, good, good, s, cfg)
    with pytest.raises(ValueError):
        spark.forward_host(good, good, good.float(), s, cfg)
