"""Benchmark: block-sparse video attention forward.

Default workload (the headline line): the 1152x640, 243-frame clip shape — B=1, H=24,
d=128, 61 x 72 x 40 = 175,680 video tokens + 512 sink rows, 64-token blocks, top-k 10%,
exact + Spark-Reweight compressed branch, bf16 in/out. One step = one whole forward
through the C ABI (pool + score/select + attention), inputs resident in HBM; inputs are
3.2 GB, larger than the 126 MB L2, so no flush is needed between steps.

Other workloads (``--workload``) time the remaining configurations the same way: the 32k
exact-only call, the tau-threshold selection, the full-density run and the 1344x768,
240-frame Spark-Reblock forward (reblock included in the step). ``--heads`` shrinks a
workload for profiling.

Multi-GPU: ``--gpus N`` without a torchrun environment re-launches itself under torchrun
with N ranks (one process per GPU). Every rank runs its own independent problem (weak
scaling, replicas); the only collectives are the timing barrier and the max-over-ranks of
the elapsed time.

Before the timed region, rank 0 checks head 0's block selection against the fp64 oracle
on sampled query tiles (tie window 1e-4) and fails the run on a mismatch.

``--impl reference`` times the fp64 CPU oracle on the host cores instead, on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time
from dataclasses import dataclass

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ms/call & dense-equiv TFLOP/s of sparse attn fwd at 10% density, N=175,680"


def unit_of(w: "Workload") -> str:
    """The unit string of a workload's line (the same on both arms)."""
    return f"TFLOP/s dense-equivalent (4*B*H*N^2*d / time, N={w.nv + w.ns:,})"


def metric_of(w: "Workload") -> str:
    return METRIC if w.name == DEFAULT else f"ms/call & dense-equiv TFLOP/s of sparse attn fwd, workload {w.name}"


@dataclass
class Workload:
    name: str
    desc: str
    H: int
    nv: int
    ns: int
    mode: str = "topk"
    param: float = 0.1
    compressed: bool = True
    reblock: bool = False
    reblock_kv: bool = False
    B: int = 1
    d: int = 128
    q_tile: int = 64
    extra_tokens: int = 0


WORKLOADS = {w.name: w for w in [
    Workload("1152x640x243", "1152x640 243-frame clip: B=1 H=24 d=128, 61x72x40=175680 video tokens "
             "+ 512 sink rows, 64-token blocks, top-k 10%, exact + Spark-Reweight compressed branch, "
             "bf16 in/out", 24, 175680, 512),
    Workload("1152x640x243-top20", "as 1152x640x243 at top-k 20%", 24, 175680, 512, param=0.2),
    Workload("1152x640x243-top30", "as 1152x640x243 at top-k 30%", 24, 175680, 512, param=0.3),
    Workload("1152x640x243-tau1.0", "as 1152x640x243 with the per-head threshold tau=1.0",
             24, 175680, 512, mode="tau", param=1.0),
    Workload("1152x640x243-tau1.5", "as 1152x640x243 with tau=1.5", 24, 175680, 512, mode="tau", param=1.5),
    Workload("1152x640x243-tau2.0", "as 1152x640x243 with tau=2.0", 24, 175680, 512, mode="tau", param=2.0),
    Workload("1152x640x243-dense", "as 1152x640x243 at 100% density, compressed branch off",
             24, 175680, 512, param=1.0, compressed=False),
    Workload("32k-exact", "single call: B=1 H=24 d=128, 32768 video tokens + 512 text sink rows, "
             "top-k 10%, exact branch only", 24, 32768, 512, compressed=False),
    Workload("1344x768x240-reblock", "1344x768 240-frame clip: B=1 H=24 d=128, 61x84x48=245952 video "
             "tokens + 512 sink rows, Spark-Reblock partition, top-k 10%, exact + compressed; "
             "the step includes the reblock", 24, 245952, 512, reblock=True),
    Workload("1344x768x240-reblock-kv", "as 1344x768x240-reblock with the keys on a partition of their "
             "own (whitened by the queries' second moment) instead of reusing the queries'",
             24, 245952, 512, reblock=True, reblock_kv=True),
    Workload("1152x640x243-q128", "as 1152x640x243 on the 128-query x 64-key route: a query tile is two "
             "consecutive blocks pooled together and sharing one selection (M = 128 tensor-core tiles)",
             24, 175680, 512, q_tile=128),
    Workload("1152x640x243-q128-tau1.5", "as 1152x640x243-q128 with tau=1.5", 24, 175680, 512,
             mode="tau", param=1.5, q_tile=128),
    Workload("1152x640x243-q128-dense", "as 1152x640x243-q128 at 100% density, compressed branch off",
             24, 175680, 512, param=1.0, compressed=False, q_tile=128),
    Workload("1344x768x240-reblock-q128", "as 1344x768x240-reblock on the 128-query route (a tile pairs "
             "two consecutive leaves)", 24, 245952, 512, reblock=True, q_tile=128),
    Workload("1152x640x243-extra512", "as 1152x640x243 with 512 extra tokens per head (the highest "
             "anchor scores) added to every video query's exact branch", 24, 175680, 512, extra_tokens=512),
]}
DEFAULT = "1152x640x243"


def flop_counts(w: Workload, nb: int, kept_qrows: int, h=None, extra_qrows: int = 0):
    """Algorithmic FLOPs of one forward (4*d per query-key pair: QK^T and PV).

    kept_qrows = selected (video query row, key block) pairs over all heads: the sum over
    query tiles of (kept blocks x rows of the tile); extra_qrows = (video query row, extra
    token outside the row's selected blocks) pairs."""
    h = w.H if h is None else h
    nv = nb * 64
    n = nv + w.ns
    d, b = w.d, w.B
    exact = kept_qrows * 64 * 4 * d + extra_qrows * 4 * d
    sink_keys = b * h * nv * w.ns * 4 * d          # video queries x dense keys
    sink_queries = b * h * w.ns * n * 4 * d        # dense queries x all keys
    compressed = (b * h * nv * nb - kept_qrows) * 4 * d if w.compressed else 0
    dense_equiv = 4 * b * h * n * n * d
    return dict(exact=exact, sink=sink_keys + sink_queries, compressed=compressed,
                selected=exact + sink_keys + sink_queries,
                attn_total=exact + sink_keys + sink_queries + compressed, dense_equiv=dense_equiv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained"), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# DRAM bytes (read + write) of one attention launch: dram__bytes_read.sum +
# dram__bytes_write.sum of the current kernel from one capture at 4 of the 24 heads (items
# go out head by head, so the traffic grows with the heads), scaled by 24 / 4
# (profiles/attn_tc_1152x640x243_h4_dram.md). A workload without a capture of its current
# kernel reports None.
ATTN_TRAFFIC_BYTES = {"1152x640x243": (4.544962e9 + 0.188276e9) * 6}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for ln in open(self.path):
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def phase_bytes(w: Workload, h: int, nb: int, nt: int, kept_blocks: int, kcap: int):
    """Algorithmic HBM bytes of the bandwidth-bound calls (each input read once, each
    output written once); nt query tiles (nb, or ceil(nb / 2) on the 128-query route)."""
    bh = w.B * h
    nv = nb * 64
    n = nv + w.ns
    row = w.d * 2
    nbp = (nb + 63) // 64 * 64
    pool = (3 * bh * nv * row + (nt + 2 * nb) * bh * w.d * 4 + bh * nb * 4 + 2 * bh * nb * w.d * 2
            + bh * nbp * 4 + bh * w.d * 4)
    select = (nt + nb) * bh * w.d * 4 + kept_blocks * 4 + bh * nt * 4
    gather = 6 * bh * n * row + bh * nv * 4          # permute Q,K,V (read + write) + perm
    return dict(pool=pool, select=select, reblock_gather=gather)


# fp32 FMA peak of the score kernel's bound: 148 SMs x 128 fp32 lanes x 2 flop x 1965 MHz
FP32_PEAK_TFLOPS = round(148 * 128 * 2 * 1965e6 / 1e12, 1)
# bf16 dense tensor rate per SM per clock (kind::f16, M = 128): 2.25 PFLOP/s nominal /
# (148 SMs x 1.855 GHz) = 8,192 flop/clk/SM
TENSOR_FLOP_PER_CLK_SM = 8192


def clock_normalised(achieved_tflops, sm_mhz):
    """The attention kernel's tensor work per SM clock at the median clock it ran at,
    against the nominal rate and against cuBLAS at its own measured clock (the sustained
    peak of MEASURED_PEAKS.json and the median clock under load it was taken at)."""
    if not sm_mhz:
        return None
    per_clk = achieved_tflops * 1e12 / (148 * sm_mhz * 1e6)
    out = {"sm_mhz": sm_mhz, "flop_per_clk_per_sm": round(per_clk, 1),
           "frac_of_nominal_rate": round(per_clk / TENSOR_FLOP_PER_CLK_SM, 4)}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            mp = json.load(f)
        mhz = mp["clocks_under_load"]["sm_mhz_median"]
        cub = mp["bf16_tflops_sustained"] * 1e12 / (148 * mhz * 1e6)
        out.update(cublas_flop_per_clk_per_sm=round(cub, 1), cublas_mhz=mhz,
                   frac_of_cublas_at_same_clock=round(per_clk / cub, 4))
    except Exception:
        pass
    return out


def route_check(w: Workload, plan, Qc, Kc, Vc, n_rows, seed=0):
    """The device's block selection of head (0, 0) against the fp64 oracle on ``n_rows``
    sampled query tiles (plus the first and the last): each device row must equal the
    oracle's, except blocks whose oracle score lies within the tie window (1e-4) of the
    cut (the k-th score for top-k, the threshold for tau). Raises on a mismatch. With
    Reblock, the oracle applies the device's permutation after checking that it is one
    (every leaf 64 ascending tokens), as the parity tests do."""
    import numpy as np

    import oracle.spark_oracle as orc

    TIE = 1e-4
    t0 = time.perf_counter()
    q, k, v = (orc.to_f64(t[0, 0]) for t in (Qc, Kc, Vc))
    nb = plan.nb
    if nb == 0:
        return {"ok": True, "rows": 0, "note": "no video block"}
    if w.reblock:
        nv = nb * 64

        def device_perm(name):
            perm = plan.rb[name][0, 0].cpu().numpy().astype(np.int64)
            leaves = perm.reshape(-1, 64)
            if (sorted(perm.tolist()) != list(range(nv)) or np.any(np.diff(leaves, axis=1) <= 0)):
                raise RuntimeError(f"route check: the device's {name} is not a leaf permutation")
            return perm
        perm = device_perm("perm")
        q = orc.apply_perm(q, perm, w.ns)
        kperm = device_perm("perm_k") if w.reblock_kv else perm
        k = orc.apply_perm(k, kperm, w.ns)
    scale = 1.0 / math.sqrt(w.d)
    P = orc.pool_head(q, k, v, w.ns, scale, 64, "reweight", w.q_tile)
    nt = P.qbar.shape[0]
    rng = np.random.default_rng(seed + 17)
    rows = np.unique(np.concatenate([[0, nt - 1], rng.choice(nt, min(n_rows, nt), replace=False)]))
    S = orc.block_scores(P.qbar, P.kbar, scale, rows)
    thr = orc.tau_threshold(orc.block_scores(P.qbar, P.kbar, scale), w.param) if w.mode == "tau" else None
    idx = plan.idx[0, 0].cpu().numpy()
    cnt = plan.cnt[0, 0].cpu().numpy()
    n_tie = 0
    for t, i in enumerate(rows):
        g = np.sort(idx[i, : cnt[i]].astype(np.int64))
        if w.mode == "topk":
            kk = orc.topk_count(w.param, nb)
            ref = orc.select_topk_row(S[t], kk)
            cut = np.sort(S[t])[::-1][kk - 1]
            if g.shape[0] != kk:
                raise RuntimeError(f"route check: row {i} keeps {g.shape[0]} blocks, not {kk}")
        else:
            ref = orc.select_tau_row(S[t], thr)
            cut = thr
        diff = np.setxor1d(ref, g)
        if diff.size and not np.all(np.abs(S[t][diff] - cut) < TIE):
            raise RuntimeError(f"route check: row {i} of head 0 differs from the oracle beyond the tie window")
        n_tie += int(diff.size)
    return {"ok": True, "head": 0, "rows": int(rows.size), "tie_window": TIE,
            "blocks_differing_at_ties": n_tie, "seconds": round(time.perf_counter() - t0, 2)}


# --------------------------------------------------------------------------- GPU arm

def max_over_ranks(x: float, world: int, device) -> float:
    """The maximum of ``x`` over all ranks of the default process group: every rank must
    call it at the same point (world 1 returns ``x`` without a collective)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_gpu(args, w: Workload, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import block_sparse_video_mean_b200.spark as spark
    from block_sparse_video_mean_b200.inputs import make_qkv

    spark.load()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    h = args.heads or w.H
    N = w.nv + w.ns
    Q, K, V = make_qkv(w.B, h, w.nv, w.ns, w.d, seed=args.seed + rank, device=dev)
    cfg = spark.ForwardConfig(w.mode, w.param, w.compressed, reblock=w.reblock, reblock_kv=w.reblock_kv,
                              q_tile=w.q_tile, extra_tokens=w.extra_tokens)
    plan = spark.SparkAttention(w.B, h, N, w.d, w.ns, cfg, dev)
    nb, nt = plan.nb, plan.nt
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        plan.run(Q, K, V)
    torch.cuda.synchronize(dev)
    err = spark.device_error(dev)
    if err != 0:
        raise RuntimeError(f"device error {err} ({spark.strerror(err)})")
    # the route (block selection) of head 0 against the fp64 oracle before any timing; a
    # mismatch outside the tie window fails the run
    route = None
    if rank == 0 and not args.no_route_check:
        route = route_check(w, plan, Q[:1, :1].cpu(), K[:1, :1].cpu(), V[:1, :1].cpu(),
                            args.route_rows, seed=args.seed)
    kept = int(plan.cnt.to(torch.int64).sum().item()) if nb > 0 else 0
    rows = torch.full((nt,), w.q_tile, dtype=torch.int64, device=dev)
    if nt:
        rows[-1] = nb * 64 - (nt - 1) * w.q_tile   # a one-block last tile on the 128-query route
    kept_qrows = int((plan.cnt.to(torch.int64) * rows).sum().item()) if nb > 0 else 0
    extra_qrows = 0
    if w.extra_tokens and nb > 0:
        # extra tokens outside each tile's selected blocks, times the tile's rows
        sel = torch.zeros((w.B, h, nt, nb), dtype=torch.int32, device=dev)
        slot = torch.arange(plan.kcap, device=dev)[None, None, None, :] < plan.cnt[..., None]
        sel.scatter_add_(3, torch.where(slot, plan.idx, 0).long(), slot.to(torch.int32))
        xb = (plan.extra_rows().long() // 64)[:, :, None, :].expand(-1, -1, nt, -1)
        outside = (torch.gather(sel, 3, xb) == 0).sum(dim=3)
        extra_qrows = int((outside * rows).sum().item())
        del sel, xb
    fl = flop_counts(w, nb, kept_qrows, h, extra_qrows)
    by = phase_bytes(w, h, nb, nt, kept, plan.kcap)

    cpu_line = None
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        cpu_line = cpu_baseline(w, Q[:, :1].cpu(), K[:, :1].cpu(), V[:, :1].cpu(), args.cpu_blocks or 200)

    ev = []
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    launches0 = spark.kernel_launches()
    with ClockSampler(local_rank) as clk:
        t0.record(stream)
        for _ in range(args.steps):
            e = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
            plan.run(Q, K, V, events=e)
            ev.append(e)
        t1.record(stream)
        torch.cuda.synchronize(dev)
    launches = spark.kernel_launches() - launches0
    if world > 1:
        dist.barrier()
    err = spark.device_error(dev)
    if err != 0:
        raise RuntimeError(f"device error {err} ({spark.strerror(err)})")
    ms = t0.elapsed_time(t1)
    phase_ms = {name: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in ev)
                for i, name in enumerate(("reblock", "pool", "select", "attn"))}
    ms = max_over_ranks(ms, world, dev)
    ms_step = ms / args.steps

    # end to end from pinned host buffers through the public host call: each group of heads
    # is copied in, computed and copied out, the copies overlapping the neighbours' compute
    hQ, hK, hV = (t.cpu().pin_memory() for t in (Q, K, V))
    hO = torch.empty(plan.O.shape, dtype=plan.O.dtype).pin_memory()

    def e2e_step():
        plan.run_host(hQ, hK, hV, hO)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_steps = max(2, min(args.steps, 5))
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / e2e_steps

    if rank != 0:
        return None
    hbm, bf16_peak, bf16_sust, peak_src = load_peaks()
    attn_ms = phase_ms["attn"]
    achieved = fl["attn_total"] / (attn_ms * 1e-3) / 1e12
    value = world * fl["dense_equiv"] / (ms_step * 1e-3) / 1e12
    clocks = clk.summary()

    def gbs(nbytes, t_ms):
        return round(nbytes / (t_ms * 1e-3) / 1e9, 1) if t_ms > 0 else None
    score_flops = 2 * w.B * h * nt * nb * w.d
    phases = {
        "pool": {"ms": round(phase_ms["pool"], 3), "bytes": by["pool"],
                 "GB/s": gbs(by["pool"], phase_ms["pool"]),
                 "frac_hbm": round(by["pool"] / (phase_ms["pool"] * 1e-3) / 1e9 / hbm, 3)},
        "select": {"ms": round(phase_ms["select"], 3), "bytes": by["select"],
                   "GB/s": gbs(by["select"], phase_ms["select"]),
                   "frac_hbm": round(by["select"] / (phase_ms["select"] * 1e-3) / 1e9 / hbm, 4),
                   "score_flops": score_flops,
                   "fp32_tflops": round(score_flops / (phase_ms["select"] * 1e-3) / 1e12, 2),
                   "frac_fp32": round(score_flops / (phase_ms["select"] * 1e-3) / 1e12 / FP32_PEAK_TFLOPS, 4),
                   "bound": f"fp32 FMA (scores), peak {FP32_PEAK_TFLOPS} TFLOP/s = 148 SMs x 128 lanes "
                            "x 2 flop x 1965 MHz"},
        "attn": {"ms": round(attn_ms, 3), "selected_flops": fl["selected"],
                 "compressed_flops": fl["compressed"]},
    }
    if w.reblock:
        # the covariance sums of every bisection level, the keys' second moment and the
        # whitening: 2 * N_v * d^2 flops each per head (fp32 products, fp64 sums)
        levels = max(1, math.ceil(math.log2(max(nb, 2))))
        passes = (levels + 2) * (2 if w.reblock_kv else 1)
        cov = 2 * w.B * h * nb * 64 * w.d * w.d * passes
        rb_ms = phase_ms["reblock"]
        phases["reblock"] = {"ms": round(rb_ms, 3), "gather_bytes": by["reblock_gather"],
                             "covariance_flops": cov,
                             "fp32_tflops": round(cov / (rb_ms * 1e-3) / 1e12, 2),
                             "frac_fp32": round(cov / (rb_ms * 1e-3) / 1e12 / FP32_PEAK_TFLOPS, 4),
                             "bound": "fp32 FMA (covariance sums; fp64 eigen-solves beside them), "
                                      "HBM for the gather"}
    line = {
        "metric": metric_of(w),
        "value": round(value, 2),
        "unit": unit_of(w),
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded block-correlated N(0,1) Q/K/V, generated on the device)",
        "config": {"workload": w.name, "desc": w.desc, "global_batch": world * w.B, "heads": h,
                   "seq_len": N, "head_dim": w.d, "select": f"{w.mode} {w.param}",
                   "compressed": w.compressed, "reblock": w.reblock, "video_blocks": nb,
                   "query_tile": w.q_tile,
                   "kept_blocks_mean_per_query_tile": round(kept / max(w.B * h * nt, 1), 2),
                   "parallelism": f"independent problem per GPU x{world}",
                   "l2": f"inputs {3 * Q.numel() * 2 / 1e9:.2f} GB "
                         + ("> 126 MB L2; no flush needed" if 3 * Q.numel() * 2 > 126e6
                            else "(< L2: reduced profiling case)")},
        "selected_tflops": round(fl["selected"] / (ms_step * 1e-3) / 1e12, 2),
        "phases": phases,
        # the attention kernel runs inside back-to-back steps of a seconds-long timed region,
        # under the power cap: the sustained figure is its denominator
        "roofline": {"bound": "tensor",
                     "kernel": f"attn_tc128_kernel<{w.d}>" if w.q_tile == 128 else f"attn_tc_kernel<{w.d}>",
                     "achieved": round(achieved, 2), "peak": bf16_sust or bf16_peak, "unit": "TFLOP/s",
                     "frac": round(achieved / (bf16_sust or bf16_peak), 4),
                     "peak_source": f"{peak_src} bf16 sustained (burst {bf16_peak})",
                     "algorithmic_flops_per_launch": fl["attn_total"],
                     "traffic": ATTN_TRAFFIC_BYTES.get(w.name) if not args.heads else None,
                     "clock_normalised": clock_normalised(achieved, clocks.get("sm_mhz"))},
        "e2e": {"value": round(world * fl["dense_equiv"] / (e2e_ms * 1e-3) / 1e12, 2),
                "unit": "TFLOP/s dense-equivalent, host buffers, copies inside the timed region",
                "ms_per_step": round(e2e_ms, 3),
                "api": "SparkAttention.run_host (spark_forward_host: automatic head groups, "
                       "copies overlapping compute)",
                "h2d_bytes_per_step": 3 * Q.numel() * Q.element_size(),
                "d2h_bytes_per_step": plan.O.numel() * plan.O.element_size()},
        "gpu_launches": launches,
        "clocks": clocks,
        "route_checked": bool(route and route["ok"]),
    }
    if route is not None:
        line["route_check"] = route
    if cpu_line is not None:
        line["cpu_baseline"] = cpu_line
    return line


# --------------------------------------------------------------------------- CPU oracle

def cpu_baseline(w: Workload, Qc, Kc, Vc, n_blocks, seed=0):
    """The fp64 oracle, as it stands, on one head: pooling of all blocks, scores and
    selection of n_blocks sampled query blocks, and their exact (+ compressed) attention.
    Reported as dense-equivalent TFLOP/s of the sampled query rows (their share of
    4*N^2*d). The reblock stage is not part of the sample."""
    import numpy as np

    import oracle.spark_oracle as orc

    t_start = time.perf_counter()
    q, k, v = (orc.to_f64(t[0, 0]) for t in (Qc, Kc, Vc))
    n = q.shape[0]
    scale = 1.0 / math.sqrt(w.d)
    P = orc.pool_head(q, k, v, w.ns, scale, 64, "reweight", w.q_tile)
    nb, nt = P.kbar.shape[0], P.qbar.shape[0]
    rng = np.random.default_rng(seed)
    # the same number of query rows on either route
    blocks = rng.choice(nt, min(max(n_blocks * 64 // w.q_tile, 1), nt), replace=False)
    sel = orc.select_head(P.qbar, P.kbar, scale, w.mode, w.param, blocks)
    rows = 0
    for t, i in enumerate(blocks):
        o, _ = orc.attn_video_block(q, k, v, w.ns, i, sel[t], P if w.compressed else None, scale, 64,
                                    w.q_tile)
        rows += o.shape[0]
    dt = time.perf_counter() - t_start
    flops = 4.0 * rows * n * w.d
    threads = None
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads") or 0) for i in threadpool_info()) or None
    except Exception:
        pass
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s dense-equivalent",
            "cores": threads or os.cpu_count(), "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"1 of {w.H} heads: pooling of all {nb} blocks, {w.mode} {w.param} selection "
                      f"of {len(blocks)} random {w.q_tile}-query tiles and their attention "
                      f"({rows} query rows)"}


def run_reference(args, w: Workload, rank, world):
    if rank != 0:
        return None
    from block_sparse_video_mean_b200.inputs import make_qkv

    # one head of the workload, drawn on the host
    Q, K, V = make_qkv(1, 1, w.nv, w.ns, w.d, seed=args.seed, device="cpu")
    vals = []
    info = None
    for i in range(args.warmup + args.steps):
        info = cpu_baseline(w, Q, K, V, args.cpu_blocks or 64, seed=i)
        if i >= args.warmup:
            vals.append(info)
    value = statistics.mean(v["value"] for v in vals)
    sec = statistics.mean(v["seconds"] for v in vals)
    cb = dict(info)
    cb["value"] = round(value, 6)
    return {
        "impl": "reference", "metric": metric_of(w),
        "value": round(value, 6),
        "unit": unit_of(w), "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded block-correlated N(0,1) Q/K/V, one head drawn on the host)",
        "config": {"workload": w.name, "sample": info["sample"]},
        "cpu_baseline": cb,
        "e2e": {"value": round(value, 6), "unit": unit_of(w),
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def spawn_ranks_command(argv, n, port):
    """torchrun command that runs this benchmark with the same arguments on n local ranks."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(n),
            "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
            *argv]


def spawn_ranks(argv, n, timeout_s=3600):
    """Run the benchmark on n ranks (torchrun, rendezvous on 127.0.0.1) and return its exit
    status; the whole process group is killed if it outlives ``timeout_s``."""
    import signal
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    proc = subprocess.Popen(spawn_ranks_command(argv, n, port), start_new_session=True)
    try:
        return proc.wait(timeout=timeout_s)
    except subprocess.TimeoutExpired:
        os.killpg(proc.pid, signal.SIGKILL)
        proc.wait()
        return 124


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="spark", choices=["spark", "reference"])
    ap.add_argument("--workload", default=DEFAULT, choices=sorted(WORKLOADS))
    ap.add_argument("--heads", type=int, default=0,
                    help="override the head count (smaller profiling cases)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-blocks", type=int, default=0,
                    help="query blocks in the oracle sample (default: 200 for cpu_baseline, 64 per reference step)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-route-check", action="store_true",
                    help="skip the check of head 0's selection against the oracle before timing")
    ap.add_argument("--route-rows", type=int, default=24,
                    help="query tiles of head 0 whose selection is checked against the oracle")
    args = ap.parse_args()
    if args.impl == "spark" and args.warmup < 3:
        args.warmup = 3
    w = WORKLOADS[args.workload]

    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: re-launch this command under torchrun with N ranks
        sys.exit(spawn_ranks(sys.argv[1:], args.gpus))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, w, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    pg = False
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
        pg = True
    try:
        line = run_gpu(args, w, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if pg:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
