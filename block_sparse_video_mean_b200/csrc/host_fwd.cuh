// The whole forward from host memory, pipelined over groups of heads: group g's Q/K/V go
// host-to-device on one stream while group g-1 computes on the caller's stream and group
// g-2's O goes device-to-host on a third. Every step of the method (pooling, anchor,
// selection and its tau moments, Reblock, attention) is per (b, h), so a group of heads is
// a forward of its own shape [1, G, N, d] and the flattened B*H heads are cut into groups
// without changing any result. Included once, at the end of spark_lib.cu.
#pragma once

namespace {

constexpr size_t kHostAlign = 256;

inline size_t align_up(size_t x) { return (x + kHostAlign - 1) / kHostAlign * kHostAlign; }

struct HostPlan {
  int64_t bh = 0;       // flattened heads
  int G = 0;            // heads per group
  int groups = 0;
  int kcap = 0;
  int nb = 0, nt = 0;
  size_t head_x = 0;    // elements of one head's Q (or K, V, O): N * d
  size_t slot_q[2], slot_k[2], slot_v[2], slot_o[2], slot_lse[2];
  size_t q_pool, k_pool, v_summ, beta, anchor, pack, pack_bytes, idx, cnt, sel, sel_bytes, attn,
      attn_bytes, perm, perm_k, qp, kp, vp, rb, rb_bytes, extra, extra_bytes;
  size_t total = 0;
};

inline spark_shape group_shape(const spark_shape* s, int heads) {
  spark_shape g = *s;
  g.B = 1;
  g.H = heads;
  return g;
}

// Resolves the configuration and carves the workspace. Returns SPARK_OK or a status.
int host_plan(const spark_shape* s, const spark_fwd_config* c, HostPlan* p) {
  const int st = check_shape(s);
  if (st != SPARK_OK) return st;
  if (c == nullptr) return SPARK_EINVAL;
  if (c->select_mode != SPARK_SELECT_TOPK_RATIO && c->select_mode != SPARK_SELECT_TAU)
    return SPARK_EINVAL;
  if (c->pool_mode != SPARK_POOL_REWEIGHT && c->pool_mode != SPARK_POOL_MEAN) return SPARK_EINVAL;
  if (c->reblock < 0 || c->reblock > 2) return SPARK_EINVAL;
  if (c->extra_tokens < 0) return SPARK_EINVAL;
  if (!std::isfinite(c->param)) return SPARK_EINVAL;
  p->bh = (int64_t)s->B * s->H;
  p->nb = (int)num_blocks(s);
  p->nt = (int)num_qtiles(s);
  if (c->select_mode == SPARK_SELECT_TOPK_RATIO) {
    const int k = spark_topk_count(c->param, p->nb);
    if (k < 0) return SPARK_EINVAL;
    p->kcap = c->kcap > 0 ? c->kcap : std::max(k, 1);
  } else {
    p->kcap = c->kcap > 0 ? c->kcap : std::max(p->nb, 1);
  }
  // automatic groups carry at least 32 MiB of Q/K/V: large heads go one at a time (a
  // head's K/V then stays in L2 while it is computed), small ones share a copy
  const int64_t head_in = (int64_t)3 * s->N * s->d * 2;
  int64_t G = c->heads_per_group > 0
                  ? c->heads_per_group
                  : (head_in > 0 ? ((int64_t)1 << 25) / head_in + (((int64_t)1 << 25) % head_in != 0) : 1);
  // Reblock's first levels run one CTA per node and head: a group of one head would leave
  // most SMs idle there, so automatic groups hold at least 8 heads when it runs
  if (c->heads_per_group <= 0 && c->reblock != 0) G = std::max<int64_t>(G, 8);
  p->G = (int)std::max<int64_t>(1, std::min<int64_t>(G, std::max<int64_t>(p->bh, 1)));
  p->groups = p->bh == 0 ? 0 : (int)((p->bh + p->G - 1) / p->G);
  const spark_shape g = group_shape(s, p->G);
  const size_t Gs = (size_t)p->G, N = (size_t)s->N, d = (size_t)s->d;
  p->head_x = N * d;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align_up(bytes);
    return at;
  };
  for (int k = 0; k < 2; ++k) {
    p->slot_q[k] = take(Gs * p->head_x * 2);
    p->slot_k[k] = take(Gs * p->head_x * 2);
    p->slot_v[k] = take(Gs * p->head_x * 2);
    p->slot_o[k] = take(Gs * p->head_x * 2);
    p->slot_lse[k] = take(Gs * N * 4);
  }
  // the call sizes grow with the number of heads, so the full group's sizes cover the last
  p->q_pool = take(Gs * p->nt * d * 4);
  p->k_pool = take(Gs * p->nb * d * 4);
  p->v_summ = take(Gs * p->nb * d * 4);
  p->beta = take(Gs * p->nb * 4);
  p->anchor = take(Gs * d * 4);
  p->pack_bytes = spark_workspace_bytes(&g, SPARK_CALL_POOL);
  p->pack = take(p->pack_bytes);
  p->idx = take(Gs * p->nt * (size_t)p->kcap * 4);
  p->cnt = take(Gs * p->nt * 4);
  p->sel_bytes = spark_workspace_bytes(&g, SPARK_CALL_SELECT);
  p->sel = take(p->sel_bytes);
  p->attn_bytes = spark_workspace_bytes(&g, SPARK_CALL_ATTN);
  p->attn = take(p->attn_bytes);
  p->extra_bytes = spark_extra_pack_bytes(&g, c->extra_tokens);
  p->extra = p->extra_bytes ? take(p->extra_bytes) : 0;
  p->perm = p->perm_k = p->qp = p->kp = p->vp = p->rb = p->rb_bytes = 0;
  if (c->reblock != 0) {
    p->perm = take(Gs * p->nb * kBlock * 4);
    if (c->reblock == 2) p->perm_k = take(Gs * p->nb * kBlock * 4);
    p->qp = take(Gs * p->head_x * 2);
    p->kp = take(Gs * p->head_x * 2);
    p->vp = take(Gs * p->head_x * 2);
    p->rb_bytes = spark_workspace_bytes(&g, SPARK_CALL_REBLOCK);
    p->rb = take(p->rb_bytes);
  }
  p->total = off;
  return SPARK_OK;
}

// One group's device calls on `cs`; buffers from the workspace, inputs in slot k.
int host_group(const spark_shape* g, const spark_fwd_config* c, const HostPlan& p, char* ws, int k,
               void* cs) {
  auto at = [&](size_t off) { return static_cast<void*>(ws + off); };
  const uint16_t* Q = static_cast<const uint16_t*>(at(p.slot_q[k]));
  const uint16_t* K = static_cast<const uint16_t*>(at(p.slot_k[k]));
  const uint16_t* V = static_cast<const uint16_t*>(at(p.slot_v[k]));
  const int32_t* perm = nullptr;
  int st = SPARK_OK;
  if (c->reblock != 0) {
    int32_t* pq = static_cast<int32_t*>(at(p.perm));
    uint16_t* Qp = static_cast<uint16_t*>(at(p.qp));
    uint16_t* Kp = static_cast<uint16_t*>(at(p.kp));
    uint16_t* Vp = static_cast<uint16_t*>(at(p.vp));
    st = c->reblock == 1
             ? spark_reblock(g, Q, K, V, pq, Qp, Kp, Vp, nullptr, at(p.rb), p.rb_bytes, cs)
             : spark_reblock_kv(g, Q, K, V, pq, static_cast<int32_t*>(at(p.perm_k)), Qp, Kp, Vp,
                                at(p.rb), p.rb_bytes, cs);
    if (st != SPARK_OK) return st;
    Q = Qp;
    K = Kp;
    V = Vp;
    perm = pq;
  }
  float* q_pool = static_cast<float*>(at(p.q_pool));
  float* k_pool = static_cast<float*>(at(p.k_pool));
  st = spark_pool_kv(g, Q, K, V, c->pool_mode, q_pool, k_pool, static_cast<float*>(at(p.v_summ)),
                     static_cast<float*>(at(p.beta)), static_cast<float*>(at(p.anchor)),
                     at(p.pack), p.pack_bytes, cs);
  if (st != SPARK_OK) return st;
  if (p.extra_bytes > 0) {
    st = spark_extra_tokens(g, K, V, static_cast<const float*>(at(p.anchor)), c->extra_tokens, c->pool_mode,
                            static_cast<float*>(at(p.v_summ)), static_cast<float*>(at(p.beta)), at(p.pack),
                            p.pack_bytes, at(p.extra), p.extra_bytes, cs);
    if (st != SPARK_OK) return st;
  }
  int32_t* idx = static_cast<int32_t*>(at(p.idx));
  int32_t* cnt = static_cast<int32_t*>(at(p.cnt));
  st = spark_score_select(g, q_pool, k_pool, c->select_mode, c->param, p.kcap, idx, cnt, at(p.sel),
                          p.sel_bytes, cs);
  if (st != SPARK_OK) return st;
  return spark_attn_fwd(g, Q, K, V, idx, cnt, p.kcap, c->compressed ? at(p.pack) : nullptr,
                        static_cast<const float*>(at(p.beta)), perm, p.extra_bytes ? at(p.extra) : nullptr,
                        p.extra_bytes ? c->extra_tokens : 0, static_cast<uint16_t*>(at(p.slot_o[k])),
                        static_cast<float*>(at(p.slot_lse[k])), at(p.attn), p.attn_bytes, cs);
}

}  // namespace

extern "C" {

size_t spark_forward_host_workspace_bytes(const spark_shape* s, const spark_fwd_config* cfg) {
  HostPlan p;
  if (host_plan(s, cfg, &p) != SPARK_OK) return 0;
  return p.total;
}

int spark_forward_host(const spark_shape* s, const spark_fwd_config* cfg, const uint16_t* hQ,
                       const uint16_t* hK, const uint16_t* hV, uint16_t* hO, float* hlse,
                       void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("spark_forward_host");
  HostPlan p;
  int st = host_plan(s, cfg, &p);
  if (st != SPARK_OK) return st;
  if (p.bh * s->N == 0) return SPARK_OK;
  if (!hQ || !hK || !hV || !hO || !ws) return SPARK_EINVAL;
  if (ws_bytes < p.total || (reinterpret_cast<uintptr_t>(ws) & (kHostAlign - 1)) != 0)
    return SPARK_EINVAL;
  char* w = static_cast<char*>(ws);
  cudaStream_t cs = as_stream(stream);
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev[7] = {};  // start, in[2], done[2], out[2]
  bool ok = cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking) == cudaSuccess;
  for (int i = 0; ok && i < 7; ++i)
    ok = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) == cudaSuccess;
  cudaEvent_t ev_start = ev[0], *ev_in = ev + 1, *ev_done = ev + 3, *ev_out = ev + 5;
  // the copies into the workspace start after the caller's earlier work on `stream`
  ok = ok && cudaEventRecord(ev_start, cs) == cudaSuccess &&
       cudaStreamWaitEvent(s_in, ev_start, 0) == cudaSuccess;
  const size_t hx = p.head_x, n = (size_t)s->N;
  for (int gi = 0; ok && st == SPARK_OK && gi < p.groups; ++gi) {
    const int k = gi & 1;
    const int64_t h0 = (int64_t)gi * p.G;
    const int heads = (int)std::min<int64_t>(p.G, p.bh - h0);
    const spark_shape g = group_shape(s, heads);
    const size_t xb = (size_t)heads * hx * 2, xo = (size_t)h0 * hx;
    // slot k's inputs were last read by group gi - 2
    if (gi >= 2) ok = cudaStreamWaitEvent(s_in, ev_done[k], 0) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(w + p.slot_q[k], hQ + xo, xb, cudaMemcpyHostToDevice, s_in) == cudaSuccess &&
         cudaMemcpyAsync(w + p.slot_k[k], hK + xo, xb, cudaMemcpyHostToDevice, s_in) == cudaSuccess &&
         cudaMemcpyAsync(w + p.slot_v[k], hV + xo, xb, cudaMemcpyHostToDevice, s_in) == cudaSuccess &&
         cudaEventRecord(ev_in[k], s_in) == cudaSuccess;
    // slot k's outputs were last copied out for group gi - 2
    ok = ok && cudaStreamWaitEvent(cs, ev_in[k], 0) == cudaSuccess;
    if (ok && gi >= 2) ok = cudaStreamWaitEvent(cs, ev_out[k], 0) == cudaSuccess;
    if (!ok) break;
    st = host_group(&g, cfg, p, w, k, stream);
    if (st != SPARK_OK) break;
    ok = cudaEventRecord(ev_done[k], cs) == cudaSuccess &&
         cudaStreamWaitEvent(s_out, ev_done[k], 0) == cudaSuccess &&
         cudaMemcpyAsync(hO + xo, w + p.slot_o[k], xb, cudaMemcpyDeviceToHost, s_out) == cudaSuccess;
    if (ok && hlse)
      ok = cudaMemcpyAsync(hlse + (size_t)h0 * n, w + p.slot_lse[k], (size_t)heads * n * 4,
                           cudaMemcpyDeviceToHost, s_out) == cudaSuccess;
    ok = ok && cudaEventRecord(ev_out[k], s_out) == cudaSuccess;
  }
  // `stream` completes after every copy in and back (also after an error, so that the
  // workspace is not reused while copies are still in flight); the earlier waits have
  // already taken their records, so two of the events can be recorded once more
  if (s_in && s_out && ev[1] && ev[5]) {
    if (cudaEventRecord(ev[1], s_in) != cudaSuccess || cudaEventRecord(ev[5], s_out) != cudaSuccess ||
        cudaStreamWaitEvent(cs, ev[1], 0) != cudaSuccess || cudaStreamWaitEvent(cs, ev[5], 0) != cudaSuccess)
      ok = false;
  }
  for (int i = 0; i < 7; ++i)
    if (ev[i]) cudaEventDestroy(ev[i]);
  if (s_in) cudaStreamDestroy(s_in);
  if (s_out) cudaStreamDestroy(s_out);
  if (st != SPARK_OK) return st;
  return ok ? SPARK_OK : SPARK_ECUDA;
}

}  // extern "C"
