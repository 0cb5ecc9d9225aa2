"""Distance to dense attention of the three compressed-branch choices, on the GPU path.

[Spark-H3] "What Spark-Attn changes": the compressed branch covers the blocks the exact
branch drops; Spark-Reweight (softmax-weighted value summary + log-mass bias) replaces the
plain mean-pooled entry. At the 1152x640x243 shape (2 heads), top-k 10%, the forward
without a compressed branch, with the mean-pooled branch and with the reweighted branch
are compared with the dense forward (density 1.0, which the parity tests tie to dense
softmax attention). Dropping the unselected blocks must be far worse than either
compressed branch.

Two input families: the plain block-correlated one, where the mean query (the anchor) is
short, so beta stays close to log 64 and the two compressed entries nearly coincide (they
differ by about 1e-5 relative, and the reweighted one must not be worse); and queries
with a per-head mean direction (``q_offset = 1``), where the anchor scores inside a block
spread by about one unit, beta departs from log 64 by about 0.5, and the reweighted branch
must be clearly closer to dense attention than the mean-pooled one (the oracle orders them
the same way on smaller heads).
"""
import math

import pytest
import torch

from block_sparse_video_mean_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("q_offset", [0.0, 1.0])
def test_compressed_branch_fidelity_at_full_length(q_offset):
    import block_sparse_video_mean_b200.spark as spark

    spark.load()
    dev = torch.device("cuda", 0)
    B, H, nv, ns, d = 1, 2, 175680, 512, 128
    Q, K, V = make_qkv(B, H, nv, ns, d, seed=4, device=dev, q_offset=q_offset)
    N = nv + ns

    def run(cfg):
        plan = spark.SparkAttention(B, H, N, d, ns, cfg, dev)
        O, _ = plan.run(Q, K, V)
        torch.cuda.synchronize()
        assert spark.device_error(dev) == 0
        return O[:, :, :nv].float().clone(), plan

    dense, _ = run(spark.ForwardConfig("topk", 1.0, False))
    err = {}
    for name, comp, pm in (("none", False, "reweight"), ("mean", True, "mean"),
                           ("reweight", True, "reweight")):
        o, plan = run(spark.ForwardConfig("topk", 0.1, comp, pm))
        err[name] = float(torch.linalg.vector_norm(o - dense) / torch.linalg.vector_norm(dense))
        if name == "reweight":
            excess = float((plan.pool["beta"] - math.log(64)).mean())
    print(f"q_offset {q_offset}: relative distance to dense attention:", err,
          "mean beta - log 64:", excess)
    assert err["none"] > 2.0 * max(err["mean"], err["reweight"]), err
    if q_offset == 0:
        assert err["reweight"] <= err["mean"] * 1.001, err
        assert excess < 0.05
    else:
        assert err["reweight"] < 0.9 * err["mean"], err
        assert excess > 0.2
