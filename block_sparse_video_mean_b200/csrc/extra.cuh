// Extra tokens: a per-head budget of individual keys added to every video query's exact
// branch, beyond its selected blocks.
//
// Method: "ComfyUI adds a core sparse-attention node and the Comfy Compiler", section
// "Block-sparse attention: one node, three backends": the extra_tokens option adds the
// highest-scoring tokens beyond the selected blocks to stay close to dense attention.
// Reading (the pages give neither the score nor the unit of the count): E tokens per
// head, ranked by the anchor score s_j = a . k_j * scale that the compressed branch
// already uses ("Spark-H3...", Spark-Reweight bullet), ties to the lower token index;
// each compressed entry then summarises only the remaining tokens of its block, and a
// block whose 64 tokens are all extra keeps no entry.
//
// Kernels (all HBM- or L2-bound and small next to the attention):
//   extra_scores_kernel   s_j for every video key (one pass over K, the pooling layout)
//   extra_select_kernel   per head: radix select of the E-th largest score key, then the
//                         tokens above it plus the lowest-index ties, in ascending order
//   extra_gather_kernel   K and V rows of the extra tokens into the extra pack (TMA rows
//                         for the attention kernel)
//   extra_fixup_kernel    the entries of the blocks that lost tokens, over their
//                         remaining tokens (a warp per such block)
#pragma once
#include "spark_common.cuh"
#include "pool.cuh"

namespace spark {

// Extra pack layout (caller-owned): xidx int32 [bh, ep] (extra token rows, ascending, -1
// past the head's count), scores fp32 [bh, nv], then bf16 K and V rows [bh * ep, d]; each
// part starts on a 256-byte boundary. ep = 64 * ceil(min(E, nv) / 64).
struct ExtraLayout {
  size_t xidx, scores, k, v, total;
  int ep, ne;  // padded rows per head, extra tokens per head
};
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
inline ExtraLayout extra_layout(size_t bh, int nv, int d, int extra) {
  ExtraLayout L;
  L.ne = extra < nv ? extra : nv;
  if (L.ne < 0) L.ne = 0;
  L.ep = (L.ne + kBlock - 1) / kBlock * kBlock;
  L.xidx = 0;
  L.scores = align256(bh * L.ep * sizeof(int32_t));
  L.k = L.scores + align256(bh * (size_t)nv * sizeof(float));
  L.v = L.k + align256(bh * L.ep * (size_t)d * sizeof(uint16_t));
  L.total = L.v + align256(bh * L.ep * (size_t)d * sizeof(uint16_t));
  return L;
}

// s_j = a . k_j * scale for the video keys of every block, with the pooling kernel's
// arithmetic (same lane layout and summation order, so the values match its own).
template <int D>
__global__ void __launch_bounds__(kPoolWarps * 32)
    extra_scores_kernel(const uint16_t* __restrict__ K, const float* __restrict__ anchor,
                        float* __restrict__ scores, int N, int nb, float scale) {
  using L = RowLayout<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bi = blockIdx.x * kPoolWarps + warp;
  if (bi >= nb) return;
  const size_t bh = blockIdx.y;
  const int c = lane % L::CPR, r0 = lane / L::CPR;
  const uint16_t* kb = K + (bh * N + (size_t)bi * kBlock) * D + c * 8;
  float a[8];
  {
    const float4* ap = reinterpret_cast<const float4*>(anchor + bh * D + c * 8);
    const float4 a0 = ap[0], a1 = ap[1];
    a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
    a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
  }
  constexpr int NBATCH = L::NR < 8 ? L::NR : 8;
  float s[L::NR];
#pragma unroll
  for (int i0 = 0; i0 < L::NR; i0 += NBATCH) {
    uint4 uk[NBATCH];
#pragma unroll
    for (int i = 0; i < NBATCH; ++i) uk[i] = ldg_nc_v4(kb + (size_t)(r0 + L::RPP * (i0 + i)) * D);
#pragma unroll
    for (int i = 0; i < NBATCH; ++i) {
      float f[8];
      bf16x8_to_f32(uk[i], f);
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(a[e], f[e], dot);
      s[i0 + i] = dot;
    }
  }
#pragma unroll
  for (int off = 1; off < L::CPR; off <<= 1)
#pragma unroll
    for (int i = 0; i < L::NR; ++i) s[i] += __shfl_xor_sync(0xffffffffu, s[i], off);
  if (c == 0) {
    float* dst = scores + bh * (size_t)nb * kBlock + (size_t)bi * kBlock;
#pragma unroll
    for (int i = 0; i < L::NR; ++i) dst[r0 + L::RPP * i] = s[i] * scale;
  }
}

constexpr int kExtraThreads = 1024;

// Block-wide exclusive prefix sums of two counters (1024 threads).
__device__ __forceinline__ void block_scan2(int a, int b, int* ea, int* eb, int* tot_a, int* tot_b, int* sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int ia = a, ib = b;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int ya = __shfl_up_sync(0xffffffffu, ia, off), yb = __shfl_up_sync(0xffffffffu, ib, off);
    if (lane >= off) {
      ia += ya;
      ib += yb;
    }
  }
  if (lane == 31) {
    sm[warp] = ia;
    sm[32 + warp] = ib;
  }
  __syncthreads();
  if (warp == 0) {
    int wa = sm[lane], wb = sm[32 + lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int ya = __shfl_up_sync(0xffffffffu, wa, off), yb = __shfl_up_sync(0xffffffffu, wb, off);
      if (lane >= off) {
        wa += ya;
        wb += yb;
      }
    }
    sm[64 + lane] = wa;  // inclusive warp totals
    sm[96 + lane] = wb;
  }
  __syncthreads();
  *ea = ia - a + (warp > 0 ? sm[64 + warp - 1] : 0);
  *eb = ib - b + (warp > 0 ? sm[96 + warp - 1] : 0);
  *tot_a = sm[64 + 31];
  *tot_b = sm[96 + 31];
  __syncthreads();
}

// One CTA per head: the ne highest scores (ties to the lower index), ascending, into xidx.
__global__ void __launch_bounds__(kExtraThreads)
    extra_select_kernel(const float* __restrict__ scores, int nv, int ne, int ep, int32_t* __restrict__ xidx) {
  __shared__ int hist[256];
  __shared__ int sm[128];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_want;
  const size_t bh = blockIdx.x;
  const float* sc = scores + bh * (size_t)nv;
  int32_t* out = xidx + bh * (size_t)ep;
  const int tid = threadIdx.x, lane = tid & 31;
  if (tid == 0) {
    s_prefix = 0u;
    s_mask = 0u;
    s_want = ne;  // rank (from the top, 1-based) of the threshold key among the candidates
  }
  for (int i = tid; i < ep; i += kExtraThreads) out[i] = -1;
  __syncthreads();
  if (ne <= 0) return;
  // ---- radix select (MSB first, 8 bits per pass) of the ne-th largest key
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += kExtraThreads) hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int j0 = 0; j0 < nv; j0 += kExtraThreads) {
      const int j = j0 + tid;
      const bool in = j < nv;
      const uint32_t key = in ? float_to_key(sc[j]) : 0u;
      const bool cand = in && (key & mask) == prefix;
      const uint32_t bin = (key >> shift) & 255u;
      // one shared atomic per group of lanes with the same bin
      const uint32_t act = __ballot_sync(0xffffffffu, cand);
      if (cand) {
        const uint32_t peers = __match_any_sync(act, bin);
        if ((peers & lanemask_lt()) == 0) atomicAdd(&hist[bin], __popc(peers));
      }
    }
    __syncthreads();
    if (tid == 0) {
      int want = s_want, b = 255;
      for (; b > 0; --b) {
        if (hist[b] >= want) break;
        want -= hist[b];
      }
      s_want = want;
      s_prefix = prefix | ((uint32_t)b << shift);
      s_mask = mask | (255u << shift);
    }
    __syncthreads();
  }
  const uint32_t T = s_prefix;
  const int budget_eq = s_want;  // keys equal to T that are taken (the lowest indices)
  // ---- compaction in token order: thread t owns tokens [t * chunk, (t + 1) * chunk)
  const int chunk = (nv + kExtraThreads - 1) / kExtraThreads;
  const int j_lo = min(nv, tid * chunk), j_hi = min(nv, j_lo + chunk);
  int gt = 0, eq = 0;
  for (int j = j_lo; j < j_hi; ++j) {
    const uint32_t key = float_to_key(sc[j]);
    gt += key > T;
    eq += key == T;
  }
  int gt_before, eq_before, gt_tot, eq_tot;
  block_scan2(gt, eq, &gt_before, &eq_before, &gt_tot, &eq_tot, sm);
  int pos = gt_before + min(eq_before, budget_eq);
  int eq_seen = eq_before;
  for (int j = j_lo; j < j_hi; ++j) {
    const uint32_t key = float_to_key(sc[j]);
    if (key > T) {
      if (pos < ne) out[pos] = j;
      ++pos;
    } else if (key == T) {
      if (eq_seen < budget_eq) {
        if (pos < ne) out[pos] = j;
        ++pos;
      }
      ++eq_seen;
    }
  }
  (void)lane;
}

// K and V rows of the extra tokens into the pack (zero rows past the count); a warp per row.
template <int D>
__global__ void __launch_bounds__(256)
    extra_gather_kernel(const uint16_t* __restrict__ K, const uint16_t* __restrict__ V,
                        const int32_t* __restrict__ xidx, int N, int nv, int ep,
                        uint16_t* __restrict__ kx, uint16_t* __restrict__ vx) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * 8 + warp;
  if (j >= ep) return;
  const size_t bh = blockIdx.y;
  const int row = xidx[bh * ep + j];
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  const bool is_v = lane >= 16;
  const int c = lane & 15;
  if (c >= CPR) return;
  uint16_t* dst = (is_v ? vx : kx) + (bh * ep + j) * D + c * 8;
  uint4 val = make_uint4(0, 0, 0, 0);
  if (row >= 0 && row < nv) val = ldg_nc_v4((is_v ? V : K) + (bh * N + row) * D + c * 8);
  *reinterpret_cast<uint4*>(dst) = val;
}

// The compressed entry of every block that lost tokens, over its remaining tokens: key mean,
// value summary and log-mass bias (Spark-Reweight), or mean value and log |R_b| (mean-pool
// branch); no entry (beta = -inf) when all 64 tokens are extra. A warp per extra token; the
// warp holding the first extra token of a block does the block.
template <int D>
__global__ void __launch_bounds__(kPoolWarps * 32)
    extra_fixup_kernel(const uint16_t* __restrict__ K, const uint16_t* __restrict__ V,
                       const float* __restrict__ anchor, const float* __restrict__ scores,
                       const int32_t* __restrict__ xidx, int N, int nb, int ne, int ep, float scale,
                       int mode, float* __restrict__ v_summ, float* __restrict__ beta,
                       uint16_t* __restrict__ k_pool16, uint16_t* __restrict__ v_summ16,
                       float* __restrict__ beta_l2, int nbp) {
  using L = RowLayout<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * kPoolWarps + warp;
  if (j >= ne) return;
  const size_t bh = blockIdx.y;
  const int32_t* xs = xidx + bh * ep;
  const int t0 = xs[j];
  const int bi = t0 / kBlock;
  if (t0 < 0 || bi >= nb || (j > 0 && xs[j - 1] / kBlock == bi)) return;
  uint64_t gone = 0;  // tokens of block bi that are extra
  for (int jj = j; jj < ne && jj < j + kBlock; ++jj) {
    const int t = xs[jj];
    if (t / kBlock != bi) break;
    gone |= 1ull << (t % kBlock);
  }
  const int nkeep = kBlock - __popcll(gone);
  const int c = lane % L::CPR, r0 = lane / L::CPR;
  const size_t row0 = bh * N + (size_t)bi * kBlock;
  const float* sb = scores + bh * (size_t)nb * kBlock + (size_t)bi * kBlock;
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < L::NR; ++i) {
    const int r = r0 + L::RPP * i;
    if (!((gone >> r) & 1ull)) mx = fmaxf(mx, sb[r]);
  }
#pragma unroll
  for (int off = L::CPR; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float se = 0.f;
#pragma unroll
  for (int i = 0; i < L::NR; ++i) {
    const int r = r0 + L::RPP * i;
    if (!((gone >> r) & 1ull)) se += expf(sb[r] - mx);
  }
#pragma unroll
  for (int off = L::CPR; off < 32; off <<= 1) se += __shfl_xor_sync(0xffffffffu, se, off);
  const float lse = nkeep > 0 ? mx + logf(se) : -INFINITY;
  float ksum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float vacc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < L::NR; ++i) {
    const int r = r0 + L::RPP * i;
    if ((gone >> r) & 1ull) continue;
    const float w = (mode == SPARK_POOL_REWEIGHT) ? expf(sb[r] - lse) : 1.0f / (float)nkeep;
    float fk[8], fv[8];
    bf16x8_to_f32(ldg_nc_v4(K + (row0 + r) * D + c * 8), fk);
    bf16x8_to_f32(ldg_nc_v4(V + (row0 + r) * D + c * 8), fv);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      ksum[e] += fk[e];
      vacc[e] = fmaf(w, fv[e], vacc[e]);
    }
  }
#pragma unroll
  for (int off = L::CPR; off < 32; off <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      vacc[e] += __shfl_xor_sync(0xffffffffu, vacc[e], off);
      ksum[e] += __shfl_xor_sync(0xffffffffu, ksum[e], off);
    }
  float a[8];
  {
    const float4* ap = reinterpret_cast<const float4*>(anchor + bh * D + c * 8);
    const float4 a0 = ap[0], a1 = ap[1];
    a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
    a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
  }
  float kc[8];
  float dot = 0.f;
  const float inv = nkeep > 0 ? 1.0f / (float)nkeep : 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    kc[e] = ksum[e] * inv;
    dot = fmaf(a[e], kc[e], dot);
  }
#pragma unroll
  for (int off = 1; off < L::CPR; off <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
  if (r0 == 0) {
    const size_t o = (bh * nb + bi) * D + c * 8;
    if (v_summ != nullptr) {
      float4* vd = reinterpret_cast<float4*>(v_summ + o);
      vd[0] = make_float4(vacc[0], vacc[1], vacc[2], vacc[3]);
      vd[1] = make_float4(vacc[4], vacc[5], vacc[6], vacc[7]);
    }
    uint4 k16, v16;
    k16.x = pack_bf16x2(kc[0], kc[1]); k16.y = pack_bf16x2(kc[2], kc[3]);
    k16.z = pack_bf16x2(kc[4], kc[5]); k16.w = pack_bf16x2(kc[6], kc[7]);
    v16.x = pack_bf16x2(vacc[0], vacc[1]); v16.y = pack_bf16x2(vacc[2], vacc[3]);
    v16.z = pack_bf16x2(vacc[4], vacc[5]); v16.w = pack_bf16x2(vacc[6], vacc[7]);
    *reinterpret_cast<uint4*>(k_pool16 + o) = k16;
    *reinterpret_cast<uint4*>(v_summ16 + o) = v16;
    if (lane == 0) {
      float b = -INFINITY;
      if (nkeep > 0) b = (mode == SPARK_POOL_REWEIGHT) ? lse - dot * scale : logf((float)nkeep);
      if (beta != nullptr) beta[bh * nb + bi] = b;
      beta_l2[bh * nbp + bi] = nkeep > 0 ? b * kLog2e : -INFINITY;
    }
  }
}

}  // namespace spark
