"""Thin Python binding of libspark (include/spark.h): argument marshalling only.

Every step of the computation runs in the CUDA library; this module allocates the
caller-owned buffers with torch, passes raw device pointers and the current stream, and
turns negative status codes into exceptions. There is no fallback: without the built
library (``python -m block_sparse_video_mean_b200.build``) and a CUDA device nothing here
computes anything.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libspark.so")

SPARK_OK = 0
SELECT_TOPK_RATIO = 0
SELECT_TAU = 1
POOL_REWEIGHT = 0
POOL_MEAN = 1
CALL_POOL, CALL_SELECT, CALL_ATTN, CALL_REBLOCK = 0, 1, 2, 3
BLOCK = 64

EXPORTS = ("spark_num_blocks", "spark_workspace_bytes", "spark_topk_count", "spark_pool_kv",
           "spark_score_select", "spark_attn_fwd", "spark_reblock", "spark_device_error",
           "spark_strerror", "spark_score_select_noalloc", "spark_kernel_launches", "spark_reblock_kv",
           "spark_num_query_tiles", "spark_forward_host", "spark_forward_host_workspace_bytes",
           "spark_set_wait_limit", "spark_extra_pack_bytes", "spark_extra_tokens")
NOALLOC_MAX_HEADS = 4096


class SparkError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: status {status} ({strerror(status)})")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("n_sink", ctypes.c_int32), ("block", ctypes.c_int32),
                ("scale", ctypes.c_float), ("q_tile", ctypes.c_int32)]


class FwdConfig(ctypes.Structure):
    _fields_ = [("param", ctypes.c_double), ("select_mode", ctypes.c_int32),
                ("kcap", ctypes.c_int32), ("pool_mode", ctypes.c_int32),
                ("compressed", ctypes.c_int32), ("reblock", ctypes.c_int32),
                ("heads_per_group", ctypes.c_int32), ("extra_tokens", ctypes.c_int32)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libspark.so from the package directory (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m block_sparse_video_mean_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_double
    SP = ctypes.POINTER(Shape)
    lib.spark_num_blocks.argtypes = [SP]
    lib.spark_num_blocks.restype = ctypes.c_int32
    lib.spark_num_query_tiles.argtypes = [SP]
    lib.spark_num_query_tiles.restype = ctypes.c_int32
    lib.spark_workspace_bytes.argtypes = [SP, I]
    lib.spark_workspace_bytes.restype = Z
    lib.spark_topk_count.argtypes = [D, ctypes.c_int32]
    lib.spark_topk_count.restype = ctypes.c_int32
    lib.spark_pool_kv.argtypes = [SP, P, P, P, I, P, P, P, P, P, P, Z, P]
    lib.spark_pool_kv.restype = I
    lib.spark_score_select.argtypes = [SP, P, P, I, D, ctypes.c_int32, P, P, P, Z, P]
    lib.spark_score_select.restype = I
    lib.spark_score_select_noalloc.argtypes = [SP, P, P, I, D, ctypes.c_int32, P, P, P]
    lib.spark_score_select_noalloc.restype = I
    lib.spark_attn_fwd.argtypes = [SP, P, P, P, P, P, ctypes.c_int32, P, P, P, P, ctypes.c_int32, P, P, P,
                                   Z, P]
    lib.spark_attn_fwd.restype = I
    lib.spark_extra_pack_bytes.argtypes = [SP, ctypes.c_int32]
    lib.spark_extra_pack_bytes.restype = Z
    lib.spark_extra_tokens.argtypes = [SP, P, P, P, ctypes.c_int32, I, P, P, P, Z, P, Z, P]
    lib.spark_extra_tokens.restype = I
    lib.spark_reblock.argtypes = [SP, P, P, P, P, P, P, P, P, P, Z, P]
    lib.spark_reblock.restype = I
    lib.spark_reblock_kv.argtypes = [SP, P, P, P, P, P, P, P, P, P, Z, P]
    lib.spark_reblock_kv.restype = I
    FP = ctypes.POINTER(FwdConfig)
    lib.spark_forward_host_workspace_bytes.argtypes = [SP, FP]
    lib.spark_forward_host_workspace_bytes.restype = Z
    lib.spark_forward_host.argtypes = [SP, FP, P, P, P, P, P, P, Z, P]
    lib.spark_forward_host.restype = I
    lib.spark_device_error.argtypes = [ctypes.POINTER(ctypes.c_int32), P]
    lib.spark_device_error.restype = I
    lib.spark_strerror.argtypes = [I]
    lib.spark_strerror.restype = ctypes.c_char_p
    lib.spark_kernel_launches.argtypes = []
    lib.spark_kernel_launches.restype = ctypes.c_uint64
    lib.spark_set_wait_limit.argtypes = [ctypes.c_int64]
    lib.spark_set_wait_limit.restype = I
    _lib = lib
    return lib


def strerror(status: int) -> str:
    return load().spark_strerror(int(status)).decode()


def _check(status: int, what: str):
    if status != SPARK_OK:
        raise SparkError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def make_shape(B, H, N, d, n_sink, scale=None, q_tile=BLOCK) -> Shape:
    return Shape(B, H, N, d, n_sink, BLOCK, float(scale) if scale else 0.0, int(q_tile))


def num_blocks(shape: Shape) -> int:
    return int(load().spark_num_blocks(ctypes.byref(shape)))


def num_query_tiles(shape: Shape) -> int:
    """Video query tiles per head: nb, or ceil(nb / 2) on the 128-query route."""
    return int(load().spark_num_query_tiles(ctypes.byref(shape)))


def topk_count(ratio: float, nb: int) -> int:
    return int(load().spark_topk_count(float(ratio), int(nb)))


def workspace_bytes(shape: Shape, call_id: int) -> int:
    return int(load().spark_workspace_bytes(ctypes.byref(shape), int(call_id)))


def kernel_launches() -> int:
    """Kernels launched through the library by this process so far (host-side count)."""
    return int(load().spark_kernel_launches())


def set_wait_limit(clocks: int = 0) -> None:
    """Limit (SM clocks) of the attention kernels' pipeline waits for later launches;
    0 restores the default (about a second)."""
    _check(load().spark_set_wait_limit(int(clocks)), "spark_set_wait_limit")


def device_error(device=None) -> int:
    word = ctypes.c_int32(0)
    _check(load().spark_device_error(ctypes.byref(word), _stream(device)), "spark_device_error")
    return int(word.value)


def _shape_of(Q, n_sink, scale, q_tile=BLOCK):
    B, H, N, d = Q.shape
    return make_shape(B, H, N, d, n_sink, scale, q_tile)


def _need(t, name):
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")


# --------------------------------------------------------------------------- the four calls

def pool_kv(Q, K, V, n_sink, pool_mode=POOL_REWEIGHT, scale=None, out=None, q_tile=BLOCK):
    """spark_pool_kv: returns dict(q_pool [B,H,nt,d], k_pool, v_summ, beta, anchor, pack)."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _need(t, n)
    shape = _shape_of(Q, n_sink, scale, q_tile)
    B, H, N, d = Q.shape
    nb = num_blocks(shape)
    nt = num_query_tiles(shape)
    dev = Q.device
    if out is None:
        out = dict(
            q_pool=torch.empty((B, H, nt, d), dtype=torch.float32, device=dev),
            k_pool=torch.empty((B, H, nb, d), dtype=torch.float32, device=dev),
            v_summ=torch.empty((B, H, nb, d), dtype=torch.float32, device=dev),
            beta=torch.empty((B, H, nb), dtype=torch.float32, device=dev),
            anchor=torch.empty((B, H, d), dtype=torch.float32, device=dev),
            pack=torch.empty(max(workspace_bytes(shape, CALL_POOL), 16), dtype=torch.uint8, device=dev),
        )
    _check(load().spark_pool_kv(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), int(pool_mode),
                                _ptr(out["q_pool"]), _ptr(out["k_pool"]), _ptr(out["v_summ"]),
                                _ptr(out["beta"]), _ptr(out["anchor"]), _ptr(out["pack"]),
                                out["pack"].numel(), _stream(dev)), "spark_pool_kv")
    return out


def score_select(q_pool, k_pool, n_sink, N, mode, param, kcap=None, scale=None, out=None, ws=None,
                 q_tile=BLOCK):
    """spark_score_select: returns (idx [B,H,nt,kcap] int32, cnt [B,H,nt] int32)."""
    B, H, nt, d = q_pool.shape
    nb = k_pool.shape[2]
    shape = make_shape(B, H, N, d, n_sink, scale, q_tile)
    dev = q_pool.device
    if kcap is None:
        kcap = topk_count(param, nb) if mode == SELECT_TOPK_RATIO else max(nb, 1)
    if out is None:
        out = (torch.empty((B, H, nt, max(kcap, 1)), dtype=torch.int32, device=dev),
               torch.empty((B, H, nt), dtype=torch.int32, device=dev))
    if ws is None:
        ws = torch.empty(max(workspace_bytes(shape, CALL_SELECT), 16), dtype=torch.uint8, device=dev)
    idx, cnt = out
    _check(load().spark_score_select(ctypes.byref(shape), _ptr(q_pool), _ptr(k_pool), int(mode),
                                     float(param), int(kcap), _ptr(idx), _ptr(cnt), _ptr(ws),
                                     0 if ws is None else ws.numel(), _stream(dev)),
           "spark_score_select")
    return idx, cnt


def score_select_noalloc(q_pool, k_pool, n_sink, N, mode, param, kcap=None, scale=None, out=None,
                         q_tile=BLOCK):
    """spark_score_select_noalloc: the selection without a scratch argument (the library
    uses its own fixed device array); returns (idx, cnt) like score_select."""
    B, H, nt, d = q_pool.shape
    nb = k_pool.shape[2]
    shape = make_shape(B, H, N, d, n_sink, scale, q_tile)
    dev = q_pool.device
    if kcap is None:
        kcap = topk_count(param, nb) if mode == SELECT_TOPK_RATIO else max(nb, 1)
    if out is None:
        out = (torch.empty((B, H, nt, max(kcap, 1)), dtype=torch.int32, device=dev),
               torch.empty((B, H, nt), dtype=torch.int32, device=dev))
    idx, cnt = out
    _check(load().spark_score_select_noalloc(ctypes.byref(shape), _ptr(q_pool), _ptr(k_pool),
                                             int(mode), float(param), int(kcap), _ptr(idx),
                                             _ptr(cnt), _stream(dev)), "spark_score_select_noalloc")
    return idx, cnt


def extra_pack_bytes(shape: Shape, extra_tokens: int) -> int:
    return int(load().spark_extra_pack_bytes(ctypes.byref(shape), int(extra_tokens)))


def extra_tokens(K, V, pool, n_sink, n_extra, pool_mode=POOL_REWEIGHT, scale=None, out=None, q_tile=BLOCK,
                 compressed=True):
    """spark_extra_tokens after pool_kv (``pool`` = its dict): returns the extra pack (uint8
    device buffer). With ``compressed`` the pooled entries of the blocks that lost tokens
    are rewritten in ``pool`` (pack, v_summ, beta)."""
    for t, n in ((K, "K"), (V, "V")):
        _need(t, n)
    shape = _shape_of(K, n_sink, scale, q_tile)
    dev = K.device
    if out is None:
        out = torch.empty(max(extra_pack_bytes(shape, n_extra), 16), dtype=torch.uint8, device=dev)
    pack = pool["pack"] if compressed else None
    _check(load().spark_extra_tokens(ctypes.byref(shape), _ptr(K), _ptr(V), _ptr(pool["anchor"]),
                                     int(n_extra), int(pool_mode),
                                     _ptr(pool["v_summ"]) if compressed else None,
                                     _ptr(pool["beta"]) if compressed else None, _ptr(pack),
                                     0 if pack is None else pack.numel(), _ptr(out), out.numel(),
                                     _stream(dev)), "spark_extra_tokens")
    return out


def extra_token_rows(xpack, B, H, nb, n_extra):
    """The extra token indices [B, H, E] (ascending) held in an extra pack."""
    ne = min(int(n_extra), nb * BLOCK)
    ep = (ne + BLOCK - 1) // BLOCK * BLOCK
    return xpack[: B * H * ep * 4].view(torch.int32).view(B, H, ep)[:, :, :ne]


def attn_fwd(Q, K, V, idx, cnt, n_sink, pack=None, beta=None, perm=None, scale=None,
             out=None, lse=True, q_tile=BLOCK, ws=None, extra_pack=None, n_extra=0):
    """spark_attn_fwd: returns (O bf16 [B,H,N,d], LSE fp32 [B,H,N] or None)."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _need(t, n)
    shape = _shape_of(Q, n_sink, scale, q_tile)
    B, H, N, d = Q.shape
    dev = Q.device
    if ws is None:
        ws = torch.empty(max(workspace_bytes(shape, CALL_ATTN), 16), dtype=torch.uint8, device=dev)
    if out is None:
        out = (torch.empty_like(Q),
               torch.empty((B, H, N), dtype=torch.float32, device=dev) if lse else None)
    O, L = out
    kcap = idx.shape[-1] if idx is not None else 1
    _check(load().spark_attn_fwd(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx),
                                 _ptr(cnt), int(kcap), _ptr(pack), _ptr(beta), _ptr(perm),
                                 _ptr(extra_pack), int(n_extra), _ptr(O), _ptr(L), _ptr(ws), ws.numel(),
                                 _stream(dev)), "spark_attn_fwd")
    return O, L


def reblock(Q, K, V, n_sink, tree=False, out=None, ws=None):
    """spark_reblock: returns dict(perm, Qp, Kp, Vp, tree or None)."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _need(t, n)
    shape = _shape_of(Q, n_sink, None)
    B, H, N, d = Q.shape
    nb = num_blocks(shape)
    dev = Q.device
    levels = 0 if nb <= 1 else math.ceil(math.log2(nb))
    if out is None:
        out = dict(perm=torch.empty((B, H, nb * BLOCK), dtype=torch.int32, device=dev),
                   Qp=torch.empty_like(Q), Kp=torch.empty_like(K), Vp=torch.empty_like(V),
                   tree=torch.empty((B, H, levels + 1, nb * BLOCK), dtype=torch.int32, device=dev)
                   if tree else None)
    if ws is None:
        ws = torch.empty(max(workspace_bytes(shape, CALL_REBLOCK), 16), dtype=torch.uint8, device=dev)
    _check(load().spark_reblock(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(out["perm"]),
                                _ptr(out["Qp"]), _ptr(out["Kp"]), _ptr(out["Vp"]),
                                _ptr(out.get("tree")), _ptr(ws), ws.numel(), _stream(dev)),
           "spark_reblock")
    return out


def reblock_kv(Q, K, V, n_sink, out=None, ws=None):
    """spark_reblock_kv (keys get their own partition): returns dict(perm, perm_k, Qp, Kp, Vp)."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _need(t, n)
    shape = _shape_of(Q, n_sink, None)
    B, H, N, d = Q.shape
    nb = num_blocks(shape)
    dev = Q.device
    if out is None:
        out = dict(perm=torch.empty((B, H, nb * BLOCK), dtype=torch.int32, device=dev),
                   perm_k=torch.empty((B, H, nb * BLOCK), dtype=torch.int32, device=dev),
                   Qp=torch.empty_like(Q), Kp=torch.empty_like(K), Vp=torch.empty_like(V))
    if ws is None:
        ws = torch.empty(max(workspace_bytes(shape, CALL_REBLOCK), 16), dtype=torch.uint8, device=dev)
    _check(load().spark_reblock_kv(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(out["perm"]),
                                   _ptr(out["perm_k"]), _ptr(out["Qp"]), _ptr(out["Kp"]), _ptr(out["Vp"]),
                                   _ptr(ws), ws.numel(), _stream(dev)),
           "spark_reblock_kv")
    return out


def fwd_config(mode=SELECT_TOPK_RATIO, param=0.1, kcap=0, pool_mode=POOL_REWEIGHT, compressed=True,
               reblock=0, heads_per_group=0, extra_tokens=0) -> FwdConfig:
    """spark_fwd_config of spark_forward_host (reblock: 0 none, 1 shared, 2 own key partition)."""
    return FwdConfig(float(param), int(mode), int(kcap or 0), int(pool_mode), int(bool(compressed)),
                     int(reblock), int(heads_per_group or 0), int(extra_tokens or 0))


def forward_host_workspace_bytes(shape: Shape, cfg: FwdConfig) -> int:
    return int(load().spark_forward_host_workspace_bytes(ctypes.byref(shape), ctypes.byref(cfg)))


def forward_host(hQ, hK, hV, shape: Shape, cfg: FwdConfig, hO=None, hlse=None, ws=None, device=None):
    """The whole forward from host tensors (bf16 [B, H, N, d], pinned for the copies to
    overlap the compute) into host ``hO`` (and ``hlse``), pipelined over groups of heads by
    spark_forward_host. Asynchronous on the current stream of ``device``; synchronise it
    before reading ``hO``."""
    lib = load()
    dev = torch.device(device if device is not None else "cuda")
    for t, name in ((hQ, "Q"), (hK, "K"), (hV, "V")):
        if t.device.type != "cpu" or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 host tensor")
    if hO is None:
        hO = torch.empty(hQ.shape, dtype=torch.bfloat16).pin_memory()
    need = forward_host_workspace_bytes(shape, cfg)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    with torch.cuda.device(ws.device):   # the library's internal streams go on this device
        _check(lib.spark_forward_host(ctypes.byref(shape), ctypes.byref(cfg), _ptr(hQ), _ptr(hK),
                                      _ptr(hV), _ptr(hO), _ptr(hlse), _ptr(ws), ws.numel(),
                                      _stream(ws.device)),
               "spark_forward_host")
    return hO, hlse


# --------------------------------------------------------------------------- whole forward

@dataclass
class ForwardConfig:
    mode: str = "topk"          # "topk" (keep ratio) or "tau" (Sol-Attn threshold)
    param: float = 0.1          # ratio or tau
    compressed: bool = True     # Spark-Reweight compressed branch on/off
    pool_mode: str = "reweight"  # "reweight" or "mean"
    reblock: bool = False       # Spark-Reblock partition first (q_reuse_k)
    reblock_kv: bool = False    # with reblock: keys get their own partition
    scale: float | None = None
    kcap: int | None = None     # slots per selection row (default: k, or nb for tau)
    q_tile: int = BLOCK         # query tile: 64, or 128 (the 128-query x 64-key route)
    extra_tokens: int = 0       # extra tokens per head added to the exact branch (0: none)


class SparkAttention:
    """A planned forward of one shape: every buffer allocated once, then ``run`` issues the
    library calls back to back on the current stream (no host synchronisation)."""

    def __init__(self, B, H, N, d, n_sink, cfg: ForwardConfig, device="cuda"):
        self.cfg = cfg
        self.n_sink = n_sink
        self.shape = make_shape(B, H, N, d, n_sink, cfg.scale, cfg.q_tile)
        self.nb = nb = num_blocks(self.shape)
        self.nt = nt = num_query_tiles(self.shape)
        dev = torch.device(device)
        self.mode = SELECT_TOPK_RATIO if cfg.mode == "topk" else SELECT_TAU
        if cfg.kcap is not None:
            self.kcap = cfg.kcap
        else:
            self.kcap = max(topk_count(cfg.param, nb) if self.mode == SELECT_TOPK_RATIO else nb, 1)
        self.pool_mode = POOL_REWEIGHT if cfg.pool_mode == "reweight" else POOL_MEAN
        f32 = dict(dtype=torch.float32, device=dev)
        self.pool = dict(q_pool=torch.empty((B, H, nt, d), **f32), k_pool=torch.empty((B, H, nb, d), **f32),
                         v_summ=torch.empty((B, H, nb, d), **f32), beta=torch.empty((B, H, nb), **f32),
                         anchor=torch.empty((B, H, d), **f32),
                         pack=torch.empty(max(workspace_bytes(self.shape, CALL_POOL), 16),
                                          dtype=torch.uint8, device=dev))
        self.idx = torch.empty((B, H, nt, self.kcap), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((B, H, nt), dtype=torch.int32, device=dev)
        self.sel_ws = torch.empty(max(workspace_bytes(self.shape, CALL_SELECT), 16), dtype=torch.uint8, device=dev)
        self.attn_ws = torch.empty(max(workspace_bytes(self.shape, CALL_ATTN), 16), dtype=torch.uint8, device=dev)
        self.O = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, H, N), **f32)
        self.xpack = None
        if cfg.extra_tokens > 0 and nb > 0:
            self.xpack = torch.empty(max(extra_pack_bytes(self.shape, cfg.extra_tokens), 16),
                                     dtype=torch.uint8, device=dev)
        self.rb = None
        if cfg.reblock:
            levels = 0 if nb <= 1 else math.ceil(math.log2(nb))
            self.rb = dict(perm=torch.empty((B, H, nb * BLOCK), dtype=torch.int32, device=dev),
                           Qp=torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev),
                           Kp=torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev),
                           Vp=torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev),
                           tree=None)
            if cfg.reblock_kv:
                self.rb["perm_k"] = torch.empty((B, H, nb * BLOCK), dtype=torch.int32, device=dev)
            self.rb_ws = torch.empty(max(workspace_bytes(self.shape, CALL_REBLOCK), 16),
                                     dtype=torch.uint8, device=dev)
            self.levels = levels

    def run(self, Q, K, V, events=None):
        """One forward. ``events`` = optional list of five CUDA events, recorded on the
        current stream before the reblock and after the reblock, the pooling, the
        selection and the attention launch (for per-call timing)."""
        cfg = self.cfg
        stream = torch.cuda.current_stream(Q.device)

        def mark(i):
            if events is not None:
                events[i].record(stream)
        perm = None
        mark(0)
        if self.rb is not None:
            if self.cfg.reblock_kv:
                reblock_kv(Q, K, V, self.n_sink, out=self.rb, ws=self.rb_ws)
            else:
                reblock(Q, K, V, self.n_sink, out=self.rb, ws=self.rb_ws)
            Q, K, V, perm = self.rb["Qp"], self.rb["Kp"], self.rb["Vp"], self.rb["perm"]
        mark(1)
        pool_kv(Q, K, V, self.n_sink, self.pool_mode, cfg.scale, out=self.pool, q_tile=cfg.q_tile)
        if self.xpack is not None:
            extra_tokens(K, V, self.pool, self.n_sink, cfg.extra_tokens, self.pool_mode, cfg.scale,
                         out=self.xpack, q_tile=cfg.q_tile, compressed=cfg.compressed)
        mark(2)
        score_select(self.pool["q_pool"], self.pool["k_pool"], self.n_sink, Q.shape[2], self.mode,
                     cfg.param, self.kcap, cfg.scale, out=(self.idx, self.cnt), ws=self.sel_ws,
                     q_tile=cfg.q_tile)
        mark(3)
        attn_fwd(Q, K, V, self.idx, self.cnt, self.n_sink,
                 pack=self.pool["pack"] if cfg.compressed else None, beta=self.pool["beta"],
                 perm=perm, scale=cfg.scale, out=(self.O, self.lse), q_tile=cfg.q_tile, ws=self.attn_ws,
                 extra_pack=self.xpack, n_extra=cfg.extra_tokens if self.xpack is not None else 0)
        mark(4)
        return self.O, self.lse

    def host_config(self, heads_per_group=0) -> FwdConfig:
        cfg = self.cfg
        rb = 0 if not cfg.reblock else (2 if cfg.reblock_kv else 1)
        return fwd_config(self.mode, cfg.param, self.kcap, self.pool_mode, cfg.compressed, rb,
                          heads_per_group, cfg.extra_tokens)

    def run_host(self, hQ, hK, hV, hO=None, hlse=None, heads_per_group=0):
        """One forward from host tensors into host ``hO`` (and ``hlse``): the copies of
        each group of heads overlap the compute of its neighbours (spark_forward_host).
        The device workspace is allocated on the first call and kept."""
        hcfg = self.host_config(heads_per_group)
        need = forward_host_workspace_bytes(self.shape, hcfg)
        if getattr(self, "host_ws", None) is None or self.host_ws.numel() < need:
            self.host_ws = torch.empty(max(need, 256), dtype=torch.uint8, device=self.O.device)
        return forward_host(hQ, hK, hV, self.shape, hcfg, hO, hlse, self.host_ws, self.O.device)

    def extra_rows(self):
        """The extra tokens of every head, [B, H, E] int32 (rows of the video tokens the
        attention ran on: the reblocked order with Reblock), or None without extra tokens."""
        if self.xpack is None:
            return None
        return extra_token_rows(self.xpack, self.shape.B, self.shape.H, self.nb, self.cfg.extra_tokens)
