// libspark: the C ABI of include/spark.h. Host-side argument validation and launches;
// every step of the computation runs in the kernels included below. The whole library
// is this one translation unit.
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "spark_common.cuh"
#include "pool.cuh"
#include "extra.cuh"
#include "select.cuh"
#include "attn_tc.cuh"
#include "attn_tc128.cuh"
#include "reblock.cuh"

using namespace spark;

namespace {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// An NVTX range around each entry point of the library (host side: the validation and the
// launches it issues), named after the call; a no-op unless a profiler is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int64_t num_blocks(const spark_shape* s) {
  const int64_t nv = (int64_t)s->N - s->n_sink;
  return nv > 0 ? nv / kBlock : 0;
}

// Query tile of the route (64 or 128 rows) and the number of video query tiles.
inline int q_tile_of(const spark_shape* s) { return s->q_tile == 0 ? kBlock : s->q_tile; }
inline int64_t num_qtiles(const spark_shape* s) {
  const int64_t nb = num_blocks(s);
  return q_tile_of(s) == kBlock ? nb : (nb + 1) / 2;
}

inline float eff_scale(const spark_shape* s) {
  return s->scale > 0.f ? s->scale : 1.0f / std::sqrt((float)s->d);
}

// Shape checks shared by every call. Returns SPARK_OK or a negative status.
int check_shape(const spark_shape* s) {
  if (s == nullptr) return SPARK_EINVAL;
  if (s->B < 0 || s->H < 0 || s->N < 0 || s->n_sink < 0 || s->n_sink > s->N) return SPARK_EINVAL;
  if (!(std::isfinite(s->scale))) return SPARK_EINVAL;
  if (s->block != kBlock) return SPARK_EUNSUPPORTED;
  if (s->q_tile != 0 && s->q_tile != kBlock && s->q_tile != 2 * kBlock) return SPARK_EUNSUPPORTED;
  if (s->d != 64 && s->d != 128) return SPARK_EUNSUPPORTED;
  const int64_t bh = (int64_t)s->B * s->H;
  if (bh > 65535) return SPARK_EUNSUPPORTED;                       // grid.y of the pooling kernels
  if ((int64_t)s->N * s->d * bh > ((int64_t)1 << 40)) return SPARK_EUNSUPPORTED;
  if ((int64_t)s->N > ((int64_t)1 << 30)) return SPARK_EUNSUPPORTED;
  return SPARK_OK;
}

inline bool empty(const spark_shape* s) { return (int64_t)s->B * s->H * s->N == 0; }

// Pool pack layout: bf16 k_pool [bh*nb, d], bf16 v_summ [bh*nb, d], then fp32
// beta*log2(e) [bh, nbp] with nbp = nb rounded up to whole 64-entry tiles.
inline size_t padded_blocks(size_t nb) { return (nb + kBlock - 1) / kBlock * kBlock; }
inline size_t pack_bias_offset(size_t bh, size_t nb, int d) { return 2 * bh * nb * d * sizeof(uint16_t); }

// Select workspace layout: fp64 tau moments [bh] and thresholds [bh], then (256-byte
// aligned) the score keys [bh][nb][nbp] with nbp = nb rounded up to 4.
inline size_t select_row_stride(size_t nb) { return (nb + 3) & ~(size_t)3; }
inline size_t select_scores_offset(size_t bh) { return ((2 * bh * sizeof(double)) + 255) & ~(size_t)255; }

// Score rows a select CTA keeps in shared memory (largest of 8, 4, 2, 1 that fits).
int select_rows_per_cta(int nb, int d, size_t* smem) {
  const size_t nbp = (size_t)((nb + 3) & ~3);
  for (int rt = 8; rt >= 1; rt >>= 1) {
    const size_t bytes = (size_t)rt * nbp * 4 + (size_t)rt * d * 4 + (size_t)d * kSelKT * 4 +
                         (kSelThreads / 32) * 256 * 4;
    if (bytes <= 200 * 1024) {
      *smem = bytes;
      return rt;
    }
  }
  return 0;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2-D bf16 map over `rows` x d, 64 x 64 boxes, 128-byte swizzle (rows of 64 elements).
bool bf16_tile_map(CUtensorMap* m, const void* base, uint64_t rows, int d) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Limit of the attention kernels' pipeline waits, in SM clocks (spark_set_wait_limit).
std::atomic<long long> g_wait_limit{tc::kWaitClocks};

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

template <int D, bool Q128>
int launch_attn_tc(const TcParams& tp, const uint16_t* K, const uint16_t* V, const void* pack,
                   const uint16_t* kx, const uint16_t* vx, cudaStream_t cs) {
  TcMaps maps;
  const uint64_t rows = (uint64_t)tp.BH * tp.N;
  if (!bf16_tile_map(&maps.k, K, rows, D) || !bf16_tile_map(&maps.v, V, rows, D)) return SPARK_ECUDA;
  if (pack != nullptr) {
    const uint16_t* kp = static_cast<const uint16_t*>(pack);
    const uint16_t* vp = kp + (size_t)tp.BH * tp.nb * D;
    const uint64_t prow = (uint64_t)tp.BH * tp.nb;
    if (!bf16_tile_map(&maps.kp, kp, prow, D) || !bf16_tile_map(&maps.vp, vp, prow, D)) return SPARK_ECUDA;
  } else {
    maps.kp = maps.k;
    maps.vp = maps.v;
  }
  if (tp.n_xh > 0) {
    const uint64_t xrow = (uint64_t)tp.BH * tp.ep;
    if (!bf16_tile_map(&maps.kx, kx, xrow, D) || !bf16_tile_map(&maps.vx, vx, xrow, D)) return SPARK_ECUDA;
  } else {
    maps.kx = maps.k;
    maps.vx = maps.v;
  }
  const size_t smem = Q128 ? tc128_smem_bytes<D>(tp.nb) : tc_smem_bytes<D>(tp.nb);
  if (smem > 227 * 1024) return SPARK_EUNSUPPORTED;
  const int sms = num_sms();
  if (sms <= 0) return SPARK_ECUDA;
  // one CTA per SM; the 64-query kernel runs two items at a time per CTA
  const int grid = (int)std::min<int64_t>(sms, Q128 ? (int64_t)tp.n_items : ((int64_t)tp.n_items + 1) / 2);
  auto kern = Q128 ? (tp.n_xh > 0 ? attn_tc128_kernel<D, true> : attn_tc128_kernel<D, false>)
                   : (tp.n_xh > 0 ? attn_tc_kernel<D, true> : attn_tc_kernel<D, false>);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SPARK_ECUDA;
  kern<<<grid, Q128 ? Tc128Cfg<D>::kThreads : TcCfg<D>::kThreads, smem, cs>>>(maps, tp);
  SPARK_LAUNCH_CHECK();
  note_launches(1);
  return SPARK_OK;
}

// Scratch of spark_score_select_noalloc: a file-scope device array (no allocation). In
// host code its name is only a stand-in, so its device address is looked up per device
// (with that device current) and cached together with the unique ID of the context it
// belongs to: a device reset replaces the primary context, the module is loaded again,
// possibly elsewhere, and the next call looks the address up anew.
__device__ __align__(256) double g_noalloc_select_scratch[2 * SPARK_NOALLOC_MAX_HEADS];
std::mutex g_noalloc_mu;
struct NoallocSlot {
  void* ptr = nullptr;
  unsigned long long ctx_id = 0;
};
NoallocSlot g_noalloc[128];

// Unique ID of the context current on this thread (0 if none is current yet).
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur == nullptr || get_id == nullptr || get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPARK_ECUDA;
  if (dev < 0 || dev >= 128) return SPARK_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc[dev];
  const unsigned long long id = current_context_id();
  if (slot.ptr == nullptr || id == 0 || id != slot.ctx_id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_select_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return SPARK_ECUDA;
    }
    slot.ptr = p;
    slot.ctx_id = current_context_id();  // the lookup made the device's context current
  }
  *out = slot.ptr;
  return SPARK_OK;
}

}  // namespace

extern "C" {

int32_t spark_num_blocks(const spark_shape* s) {
  if (check_shape(s) != SPARK_OK) return 0;
  return (int32_t)num_blocks(s);
}

int32_t spark_num_query_tiles(const spark_shape* s) {
  if (check_shape(s) != SPARK_OK) return 0;
  return (int32_t)num_qtiles(s);
}

int32_t spark_topk_count(double ratio, int32_t nb) {
  if (!(ratio > 0.0 && ratio <= 1.0)) return -1;
  if (nb <= 0) return 0;
  double k = std::ceil(ratio * (double)nb - 1e-9);
  if (k < 1.0) k = 1.0;
  if (k > nb) k = nb;
  return (int32_t)k;
}

size_t spark_workspace_bytes(const spark_shape* s, int call_id) {
  if (check_shape(s) != SPARK_OK) return 0;
  const size_t bh = (size_t)s->B * s->H;
  const size_t nb = (size_t)num_blocks(s);
  switch (call_id) {
    case SPARK_CALL_POOL:
      return pack_bias_offset(bh, nb, s->d) + bh * padded_blocks(nb) * sizeof(float);
    case SPARK_CALL_SELECT:
      return select_scores_offset(bh) + bh * (size_t)num_qtiles(s) * select_row_stride(nb) * sizeof(uint32_t);
    case SPARK_CALL_ATTN:
      return 256;  // the per-launch counter of the dynamic item queue
    case SPARK_CALL_REBLOCK:
      return reblock_workspace_bytes(s->B * s->H, (int)nb, s->d);
    default:
      return 0;
  }
}

int spark_pool_kv(const spark_shape* s, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                  int pool_mode, float* q_pool, float* k_pool, float* v_summ, float* beta,
                  float* anchor, void* pool_pack, size_t pool_pack_bytes, void* stream) {
  NvtxRange nvtx_range("spark_pool_kv");
  int st = check_shape(s);
  if (st != SPARK_OK) return st;
  if (pool_mode != SPARK_POOL_REWEIGHT && pool_mode != SPARK_POOL_MEAN) return SPARK_EINVAL;
  if (empty(s)) return SPARK_OK;
  const int nb = (int)num_blocks(s);
  const int bh = s->B * s->H;
  if (!Q || !K || !V || !anchor) return SPARK_EINVAL;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(anchor)) return SPARK_EINVAL;
  cudaStream_t cs = as_stream(stream);
  if (nb == 0) {
    if (cudaMemsetAsync(anchor, 0, (size_t)bh * s->d * sizeof(float), cs) != cudaSuccess) return SPARK_ECUDA;
    return SPARK_OK;
  }
  if (!q_pool || !k_pool || !v_summ || !beta || !pool_pack) return SPARK_EINVAL;
  if (!aligned16(q_pool) || !aligned16(k_pool) || !aligned16(v_summ) || !aligned16(pool_pack))
    return SPARK_EINVAL;
  if (pool_pack_bytes < spark_workspace_bytes(s, SPARK_CALL_POOL)) return SPARK_EINVAL;
  uint16_t* k16 = static_cast<uint16_t*>(pool_pack);
  uint16_t* v16 = k16 + (size_t)bh * nb * s->d;
  float* bl2 = reinterpret_cast<float*>(static_cast<unsigned char*>(pool_pack) +
                                        pack_bias_offset(bh, nb, s->d));
  const int nbp = (int)padded_blocks(nb);
  const float scale = eff_scale(s);
  dim3 grid((nb + kPoolWarps - 1) / kPoolWarps, bh);
  const int nt = (int)num_qtiles(s);
  dim3 gq((nt + kPoolWarps - 1) / kPoolWarps, bh);
  const bool q128 = q_tile_of(s) == 2 * kBlock;
  const float last_w = (q128 && (nb & 1)) ? 0.5f : 1.0f;
  const int nv = nb * kBlock;
  if (s->d == 128) {
    if (q128) pool_q_kernel<128, 128><<<gq, kPoolWarps * 32, 0, cs>>>(Q, q_pool, s->N, nt, nv);
    else pool_q_kernel<128, 64><<<gq, kPoolWarps * 32, 0, cs>>>(Q, q_pool, s->N, nt, nv);
    anchor_kernel<128><<<bh, 256, 0, cs>>>(q_pool, anchor, nt, last_w);
    pool_kv_kernel<128><<<grid, kPoolWarps * 32, 0, cs>>>(K, V, anchor, k_pool, v_summ, beta, k16,
                                                          v16, bl2, nbp, s->N, nb, scale, pool_mode);
  } else {
    if (q128) pool_q_kernel<64, 128><<<gq, kPoolWarps * 32, 0, cs>>>(Q, q_pool, s->N, nt, nv);
    else pool_q_kernel<64, 64><<<gq, kPoolWarps * 32, 0, cs>>>(Q, q_pool, s->N, nt, nv);
    anchor_kernel<64><<<bh, 256, 0, cs>>>(q_pool, anchor, nt, last_w);
    pool_kv_kernel<64><<<grid, kPoolWarps * 32, 0, cs>>>(K, V, anchor, k_pool, v_summ, beta, k16,
                                                         v16, bl2, nbp, s->N, nb, scale, pool_mode);
  }
  SPARK_LAUNCH_CHECK();
  note_launches(3);
  return SPARK_OK;
}

size_t spark_extra_pack_bytes(const spark_shape* s, int32_t extra_tokens) {
  if (check_shape(s) != SPARK_OK || extra_tokens <= 0) return 0;
  const int nb = (int)num_blocks(s);
  if (nb == 0) return 0;
  return extra_layout((size_t)s->B * s->H, nb * kBlock, s->d, extra_tokens).total;
}

int spark_extra_tokens(const spark_shape* s, const uint16_t* K, const uint16_t* V, const float* anchor,
                       int32_t extra_tokens, int pool_mode, float* v_summ, float* beta, void* pool_pack,
                       size_t pool_pack_bytes, void* extra_pack, size_t extra_pack_bytes, void* stream) {
  NvtxRange nvtx_range("spark_extra_tokens");
  int st = check_shape(s);
  if (st != SPARK_OK) return st;
  if (extra_tokens < 0) return SPARK_EINVAL;
  if (pool_mode != SPARK_POOL_REWEIGHT && pool_mode != SPARK_POOL_MEAN) return SPARK_EINVAL;
  const int nb = (int)num_blocks(s);
  if (empty(s) || nb == 0 || extra_tokens == 0) return SPARK_OK;
  const size_t bh = (size_t)s->B * s->H;
  const int nv = nb * kBlock;
  if (!K || !V || !anchor || !extra_pack) return SPARK_EINVAL;
  if (!aligned16(K) || !aligned16(V) || !aligned16(anchor) || !aligned16(extra_pack)) return SPARK_EINVAL;
  const ExtraLayout xl = extra_layout(bh, nv, s->d, extra_tokens);
  if (extra_pack_bytes < xl.total) return SPARK_EINVAL;
  if (pool_pack != nullptr) {
    if (!aligned16(pool_pack) || pool_pack_bytes < spark_workspace_bytes(s, SPARK_CALL_POOL)) return SPARK_EINVAL;
    if ((v_summ && !aligned16(v_summ)) || (beta && !aligned16(beta))) return SPARK_EINVAL;
  }
  unsigned char* xb = static_cast<unsigned char*>(extra_pack);
  int32_t* xidx = reinterpret_cast<int32_t*>(xb + xl.xidx);
  float* scores = reinterpret_cast<float*>(xb + xl.scores);
  uint16_t* kx = reinterpret_cast<uint16_t*>(xb + xl.k);
  uint16_t* vx = reinterpret_cast<uint16_t*>(xb + xl.v);
  const float scale = eff_scale(s);
  cudaStream_t cs = as_stream(stream);
  const dim3 gs((nb + kPoolWarps - 1) / kPoolWarps, (unsigned)bh);
  const dim3 gg(xl.ep / 8, (unsigned)bh);
  const dim3 gf((xl.ne + kPoolWarps - 1) / kPoolWarps, (unsigned)bh);
  uint16_t* k16 = static_cast<uint16_t*>(pool_pack);
  uint16_t* v16 = k16 ? k16 + bh * nb * s->d : nullptr;
  float* bl2 = pool_pack ? reinterpret_cast<float*>(static_cast<unsigned char*>(pool_pack) +
                                                    pack_bias_offset(bh, nb, s->d))
                         : nullptr;
  const int nbp = (int)padded_blocks(nb);
  int launches = 3;
  if (s->d == 128) {
    extra_scores_kernel<128><<<gs, kPoolWarps * 32, 0, cs>>>(K, anchor, scores, s->N, nb, scale);
    extra_select_kernel<<<(unsigned)bh, kExtraThreads, 0, cs>>>(scores, nv, xl.ne, xl.ep, xidx);
    extra_gather_kernel<128><<<gg, 256, 0, cs>>>(K, V, xidx, s->N, nv, xl.ep, kx, vx);
    if (pool_pack) {
      extra_fixup_kernel<128><<<gf, kPoolWarps * 32, 0, cs>>>(K, V, anchor, scores, xidx, s->N, nb, xl.ne, xl.ep,
                                                              scale, pool_mode, v_summ, beta, k16, v16, bl2, nbp);
      ++launches;
    }
  } else {
    extra_scores_kernel<64><<<gs, kPoolWarps * 32, 0, cs>>>(K, anchor, scores, s->N, nb, scale);
    extra_select_kernel<<<(unsigned)bh, kExtraThreads, 0, cs>>>(scores, nv, xl.ne, xl.ep, xidx);
    extra_gather_kernel<64><<<gg, 256, 0, cs>>>(K, V, xidx, s->N, nv, xl.ep, kx, vx);
    if (pool_pack) {
      extra_fixup_kernel<64><<<gf, kPoolWarps * 32, 0, cs>>>(K, V, anchor, scores, xidx, s->N, nb, xl.ne, xl.ep,
                                                             scale, pool_mode, v_summ, beta, k16, v16, bl2, nbp);
      ++launches;
    }
  }
  SPARK_LAUNCH_CHECK();
  note_launches(launches);
  return SPARK_OK;
}

}  // extern "C"

namespace {

// Scores + selection. `fused`: one kernel keeps each CTA's score rows in shared memory
// (scratch: the tau moments only); otherwise the scores are first written to the
// caller's workspace by a tiled kernel and rows are selected from there.
int score_select_impl(const spark_shape* s, const float* q_pool, const float* k_pool, int mode,
                      double param, int32_t kcap, int32_t* idx, int32_t* cnt, void* ws,
                      size_t ws_bytes, void* stream, bool fused) {
  int st = check_shape(s);
  if (st != SPARK_OK) return st;
  const int nb = (int)num_blocks(s);
  const int nq = (int)num_qtiles(s);
  const int bh = s->B * s->H;
  int k = 0;
  if (mode == SPARK_SELECT_TOPK_RATIO) {
    k = spark_topk_count(param, nb);
    if (k < 0) return SPARK_EINVAL;
    if (kcap < k) return SPARK_EINVAL;
  } else if (mode == SPARK_SELECT_TAU) {
    if (!std::isfinite(param)) return SPARK_EINVAL;
  } else {
    return SPARK_EINVAL;
  }
  if (kcap < 0) return SPARK_EINVAL;
  if (empty(s) || nb == 0) return SPARK_OK;
  if (kcap < 1) return SPARK_EINVAL;
  if (!q_pool || !k_pool || !idx || !cnt) return SPARK_EINVAL;
  if (!aligned16(q_pool) || !aligned16(k_pool)) return SPARK_EINVAL;
  size_t smem = 0;
  const int rt = select_rows_per_cta(nb, s->d, &smem);
  if (rt == 0) return SPARK_EUNSUPPORTED;
  cudaStream_t cs = as_stream(stream);
  const float scale = eff_scale(s);
  double* thr = nullptr;
  const size_t need = fused ? select_scores_offset(bh) : spark_workspace_bytes(s, SPARK_CALL_SELECT);
  if ((mode == SPARK_SELECT_TAU || !fused) && (!ws || ws_bytes < need || !aligned16(ws)))
    return SPARK_EINVAL;
  if (mode == SPARK_SELECT_TAU) {
    double* acc = static_cast<double*>(ws);
    thr = acc + bh;
    if (cudaMemsetAsync(acc, 0, (size_t)bh * sizeof(double), cs) != cudaSuccess) return SPARK_ECUDA;
    if (s->d == 128) {
      moments_kernel<128><<<dim3(16, bh), 256, 0, cs>>>(q_pool, k_pool, nq, nb, acc);
      tau_threshold_kernel<128><<<bh, 128, 0, cs>>>(q_pool, k_pool, nq, nb, acc, scale, param, thr);
    } else {
      moments_kernel<64><<<dim3(4, bh), 256, 0, cs>>>(q_pool, k_pool, nq, nb, acc);
      tau_threshold_kernel<64><<<bh, 64, 0, cs>>>(q_pool, k_pool, nq, nb, acc, scale, param, thr);
    }
    SPARK_LAUNCH_CHECK();
    note_launches(2);
  }
  SelectParams sp;
  sp.q_pool = q_pool;
  sp.k_pool = k_pool;
  sp.idx = idx;
  sp.cnt = cnt;
  sp.thr = thr;
  sp.nq = nq;
  sp.nb = nb;
  sp.kcap = kcap;
  sp.k = k;
  sp.mode = mode;
  sp.rt = rt;
  sp.scale = scale;
  // query tiles the attention kernel runs at once: one CTA per SM, two 64-query items
  // per CTA or one 128-query tile
  sp.sweep = num_sms() * (q_tile_of(s) == 2 * kBlock ? 1 : 2);
  if (!fused) {
    const int nbp = (int)select_row_stride(nb);
    uint32_t* skeys = reinterpret_cast<uint32_t*>(static_cast<unsigned char*>(ws) + select_scores_offset(bh));
    dim3 gs((nb + kScJ - 1) / kScJ, (nq + kScI - 1) / kScI, bh);
    if (s->d == 128)
      score_tile_kernel<128><<<gs, 256, 0, cs>>>(q_pool, k_pool, nq, nb, nbp, scale, skeys);
    else
      score_tile_kernel<64><<<gs, 256, 0, cs>>>(q_pool, k_pool, nq, nb, nbp, scale, skeys);
    const size_t smem_sel = (size_t)8 * nbp * 4 + 8 * 256 * 4;
    if (smem_sel > 227 * 1024) return SPARK_EUNSUPPORTED;
    cudaFuncSetAttribute(select_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_sel);
    select_rows_kernel<<<dim3((nq + 7) / 8, bh), 256, smem_sel, cs>>>(sp, skeys, nbp);
    SPARK_LAUNCH_CHECK();
    note_launches(2);
    return SPARK_OK;
  }
  dim3 grid((nq + rt - 1) / rt, bh);
  if (s->d == 128) {
    cudaFuncSetAttribute(score_select_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    score_select_kernel<128><<<grid, kSelThreads, smem, cs>>>(sp);
  } else {
    cudaFuncSetAttribute(score_select_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    score_select_kernel<64><<<grid, kSelThreads, smem, cs>>>(sp);
  }
  SPARK_LAUNCH_CHECK();
  note_launches(1);
  return SPARK_OK;
}

}  // namespace

extern "C" {

int spark_score_select(const spark_shape* s, const float* q_pool, const float* k_pool, int mode,
                       double param, int32_t kcap, int32_t* idx, int32_t* cnt, void* ws,
                       size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("spark_score_select");
  return score_select_impl(s, q_pool, k_pool, mode, param, kcap, idx, cnt, ws, ws_bytes, stream,
                           /*fused=*/false);
}

int spark_score_select_noalloc(const spark_shape* s, const float* q_pool, const float* k_pool,
                               int mode, double param, int32_t kcap, int32_t* idx, int32_t* cnt,
                               void* stream) {
  NvtxRange nvtx_range("spark_score_select_noalloc");
  int st = check_shape(s);
  if (st != SPARK_OK) return st;
  if ((int64_t)s->B * s->H > SPARK_NOALLOC_MAX_HEADS) return SPARK_ESCRATCH;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != SPARK_OK) return st;
  return score_select_impl(s, q_pool, k_pool, mode, param, kcap, idx, cnt, scratch,
                           sizeof(g_noalloc_select_scratch), stream, /*fused=*/true);
}

int spark_attn_fwd(const spark_shape* s, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                   const int32_t* idx, const int32_t* cnt, int32_t kcap, const void* pool_pack,
                   const float* beta, const int32_t* perm, const void* extra_pack, int32_t extra_tokens,
                   uint16_t* O, float* lse, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("spark_attn_fwd");
  int st = check_shape(s);
  if (st != SPARK_OK) return st;
  if (extra_tokens < 0) return SPARK_EINVAL;
  if (empty(s)) return SPARK_OK;
  if (!ws || ws_bytes < spark_workspace_bytes(s, SPARK_CALL_ATTN) || !aligned16(ws)) return SPARK_EINVAL;
  const int nb = (int)num_blocks(s);
  const int bh = s->B * s->H;
  if (!Q || !K || !V || !O) return SPARK_EINVAL;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SPARK_EINVAL;
  if (nb > 0) {
    if (!idx || !cnt || kcap < 1) return SPARK_EINVAL;
    if (pool_pack && !aligned16(pool_pack)) return SPARK_EINVAL;
  }
  const int nv = nb * kBlock;
  const int qt = q_tile_of(s);
  const int nt = (int)num_qtiles(s);
  const int n_dq = (s->N - nv + qt - 1) / qt;
  const int64_t items = (int64_t)bh * (n_dq + nt);
  if (items > 0x7fffffff) return SPARK_EUNSUPPORTED;
  if ((int64_t)bh * s->N >= ((int64_t)1 << 31)) return SPARK_EUNSUPPORTED;  // TMA row coordinates
  TcParams tp;
  tp.Q = Q;
  tp.idx = idx;
  tp.cnt = cnt;
  (void)beta;  // the compressed branch reads the pool pack's padded copy
  tp.bias = nullptr;
  tp.nbp = (int)padded_blocks(nb);
  if (nb > 0 && pool_pack != nullptr)
    tp.bias = reinterpret_cast<const float*>(static_cast<const unsigned char*>(pool_pack) +
                                             pack_bias_offset(bh, nb, s->d));
  tp.perm = perm;
  tp.O = O;
  tp.lse = lse;
  tp.N = s->N;
  tp.nb = nb;
  tp.kcap = kcap;
  tp.BH = bh;
  tp.n_dq = n_dq;
  tp.nt = nt;
  tp.pooled = (nb > 0 && pool_pack != nullptr) ? 1 : 0;
  tp.n_items = (int)items;
  tp.scale_log2 = eff_scale(s) * kLog2e;
  tp.item_ctr = static_cast<int*>(ws);
  tp.wait_clocks = g_wait_limit.load(std::memory_order_relaxed);
  tp.xidx = nullptr;
  tp.n_xh = tp.n_extra = tp.ep = 0;
  const uint16_t* kx = nullptr;
  const uint16_t* vx = nullptr;
  if (extra_tokens > 0 && nb > 0) {
    if (!extra_pack || !aligned16(extra_pack)) return SPARK_EINVAL;
    const ExtraLayout xl = extra_layout((size_t)bh, nv, s->d, extra_tokens);
    const unsigned char* xb = static_cast<const unsigned char*>(extra_pack);
    tp.xidx = reinterpret_cast<const int32_t*>(xb + xl.xidx);
    tp.n_xh = xl.ep / kBlock;
    tp.n_extra = xl.ne;
    tp.ep = xl.ep;
    kx = reinterpret_cast<const uint16_t*>(xb + xl.k);
    vx = reinterpret_cast<const uint16_t*>(xb + xl.v);
    if ((int64_t)bh * xl.ep >= ((int64_t)1 << 31)) return SPARK_EUNSUPPORTED;
  }
  cudaStream_t cs = as_stream(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(int), cs) != cudaSuccess) return SPARK_ECUDA;
  const void* pack = tp.pooled ? pool_pack : nullptr;
  if (qt == 2 * kBlock)
    return s->d == 128 ? launch_attn_tc<128, true>(tp, K, V, pack, kx, vx, cs)
                       : launch_attn_tc<64, true>(tp, K, V, pack, kx, vx, cs);
  return s->d == 128 ? launch_attn_tc<128, false>(tp, K, V, pack, kx, vx, cs)
                     : launch_attn_tc<64, false>(tp, K, V, pack, kx, vx, cs);
}

}  // extern "C"

namespace {

int reblock_impl(const spark_shape* s, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                 int32_t* perm, int32_t* perm_k, bool independent, uint16_t* Qp, uint16_t* Kp,
                 uint16_t* Vp, int32_t* tree, void* ws, size_t ws_bytes, void* stream) {
  int st = check_shape(s);
  if (st != SPARK_OK) return st;
  if (empty(s)) return SPARK_OK;
  if (!Q || !K || !V || !Qp || !Kp || !Vp) return SPARK_EINVAL;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(Qp) || !aligned16(Kp) ||
      !aligned16(Vp))
    return SPARK_EINVAL;
  const int nb = (int)num_blocks(s);
  if (nb > 0 && (!perm || (independent && !perm_k))) return SPARK_EINVAL;
  if (ws_bytes < spark_workspace_bytes(s, SPARK_CALL_REBLOCK)) return SPARK_EINVAL;
  if (spark_workspace_bytes(s, SPARK_CALL_REBLOCK) > 0 && (!ws || !aligned16(ws))) return SPARK_EINVAL;
  return reblock_launch(s->B * s->H, s->N, nb, s->d, Q, K, V, perm, independent ? perm_k : nullptr, Qp, Kp,
                        Vp, tree, ws, as_stream(stream));
}

}  // namespace

extern "C" {

int spark_reblock(const spark_shape* s, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                  int32_t* perm, uint16_t* Qp, uint16_t* Kp, uint16_t* Vp, int32_t* tree, void* ws,
                  size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("spark_reblock");
  return reblock_impl(s, Q, K, V, perm, nullptr, false, Qp, Kp, Vp, tree, ws, ws_bytes, stream);
}

int spark_reblock_kv(const spark_shape* s, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                     int32_t* perm_q, int32_t* perm_k, uint16_t* Qp, uint16_t* Kp, uint16_t* Vp,
                     void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("spark_reblock_kv");
  return reblock_impl(s, Q, K, V, perm_q, perm_k, true, Qp, Kp, Vp, nullptr, ws, ws_bytes, stream);
}

int spark_device_error(int32_t* host_word, void* stream) {
  cudaStream_t cs = as_stream(stream);
  int32_t v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_error_word, sizeof(int32_t), 0, cudaMemcpyDeviceToHost, cs) !=
      cudaSuccess)
    return SPARK_ECUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return SPARK_ECUDA;
  const int32_t zero = 0;
  if (cudaMemcpyToSymbolAsync(g_error_word, &zero, sizeof(int32_t), 0, cudaMemcpyHostToDevice, cs) !=
      cudaSuccess)
    return SPARK_ECUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return SPARK_ECUDA;
  if (host_word) *host_word = v;
  return SPARK_OK;
}

uint64_t spark_kernel_launches(void) { return g_kernel_launches.load(std::memory_order_relaxed); }

int spark_set_wait_limit(int64_t clocks) {
  g_wait_limit.store(clocks > 0 ? (long long)clocks : tc::kWaitClocks, std::memory_order_relaxed);
  return SPARK_OK;
}

const char* spark_strerror(int status) {
  switch (status) {
    case SPARK_OK: return "ok";
    case SPARK_EINVAL: return "invalid argument (shape, pointer, alignment, ratio/tau or kcap)";
    case SPARK_EUNSUPPORTED: return "unsupported (d must be 64 or 128, block 64, sizes within limits)";
    case SPARK_ECUDA: return "CUDA launch or copy failed";
    case SPARK_ETIMEOUT: return "device: a bounded wait gave up";
    case SPARK_EDEVICE_INDEX: return "device: block index or count out of range (skipped)";
    case SPARK_ECAPACITY: return "device: more blocks kept than kcap (row truncated)";
    case SPARK_ESCRATCH: return "B*H exceeds the static scratch of spark_score_select_noalloc";
    default: return "unknown status";
  }
}

}  // extern "C"
#include "host_fwd.cuh"
