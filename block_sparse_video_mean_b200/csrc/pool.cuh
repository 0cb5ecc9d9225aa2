// Pooling, anchor and Spark-Reweight summaries (HBM-bound; one pass over Q, one over K/V).
//
// Method: "Spark-H3: speeding up MiniMax-H3 in ComfyUI with block-sparse attention",
// section "What Spark-Attn changes", Spark-Reweight bullet and the figure caption after
// it: the compressed branch replaces a mean-pooled key/value summary by a weighted
// summary plus a log-mass bias; one anchor per head (the mean video query) scores the
// keys, so the extra cost stays linear.
//
// Layout: one warp per 64-row block. With d = 8*CPR columns, lane l reads the 16-byte
// chunk (l % CPR) of rows (l / CPR) + RPP*i, RPP = 32 / CPR: every warp load is 512
// contiguous bytes (fully coalesced 128-bit loads, read-only non-allocating path).
#pragma once
#include "spark_common.cuh"

namespace spark {

constexpr int kPoolWarps = 8;

template <int D>
struct RowLayout {
  static constexpr int CPR = D / 8;        // 16-byte chunks per row
  static constexpr int RPP = 32 / CPR;     // rows per warp pass
  static constexpr int NR = kBlock / RPP;  // rows per lane
};

// q_pool[bh, i, :] = mean of the queries of query tile i: QT = 64 rows (a block) or 128
// (two blocks; the last tile holds one block when nb is odd).
template <int D, int QT>
__global__ void __launch_bounds__(kPoolWarps * 32) pool_q_kernel(const uint16_t* __restrict__ Q,
                                                                 float* __restrict__ q_pool, int N,
                                                                 int nt, int nv) {
  using L = RowLayout<D>;
  constexpr int NR = QT / L::RPP;  // rows per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bi = blockIdx.x * kPoolWarps + warp;
  if (bi >= nt) return;
  const size_t bh = blockIdx.y;
  const int c = lane % L::CPR, r0 = lane / L::CPR;
  const int nrows = min(QT, nv - bi * QT);  // a multiple of 64, so of RPP
  const int nr = nrows / L::RPP;             // rows this lane reads (warp-uniform)
  const uint16_t* base = Q + (bh * N + (size_t)bi * QT) * D + c * 8;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  constexpr int NBATCH = NR < 8 ? NR : 8;  // 8 loads in flight per lane
#pragma unroll
  for (int i0 = 0; i0 < NR; i0 += NBATCH) {
    if (i0 < nr) {
      uint4 u[NBATCH];
#pragma unroll
      for (int i = 0; i < NBATCH; ++i) u[i] = ldg_nc_v4(base + (size_t)(r0 + L::RPP * (i0 + i)) * D);
#pragma unroll
      for (int i = 0; i < NBATCH; ++i) {
        float f[8];
        bf16x8_to_f32(u[i], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += f[e];
      }
    }
  }
#pragma unroll
  for (int off = L::CPR; off < 32; off <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  if (r0 == 0) {
    float4* dst = reinterpret_cast<float4*>(q_pool + (bh * nt + bi) * D + c * 8);
    const float inv = 1.0f / nrows;
    dst[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    dst[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
  }
}

// anchor[bh, :] = the mean video query: the mean of the nt rows of q_pool, the last one
// weighted by last_w (1, or 0.5 for a one-block last tile of the 128-query route).
// Fixed-order reduction (deterministic): thread group g sums tiles g, g+G, ... then the
// groups are added in order.
template <int D>
__global__ void __launch_bounds__(256) anchor_kernel(const float* __restrict__ q_pool,
                                                     float* __restrict__ anchor, int nt, float last_w) {
  constexpr int G = 256 / D;
  __shared__ float part[G][D];
  const int c = threadIdx.x % D, g = threadIdx.x / D;
  const size_t bh = blockIdx.x;
  const float* src = q_pool + bh * (size_t)nt * D;
  float acc = 0.f;
  for (int b = g; b < nt; b += G) acc += src[(size_t)b * D + c] * (b == nt - 1 ? last_w : 1.0f);
  part[g][c] = acc;
  __syncthreads();
  if (g == 0) {
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < G; ++i) t += part[i][c];
    anchor[bh * D + c] = nt > 0 ? t / ((float)(nt - 1) + last_w) : 0.f;
  }
}

// k_pool, v_summ, beta of every video block of a head (see spark.h for the formulas).
template <int D>
__global__ void __launch_bounds__(kPoolWarps * 32)
    pool_kv_kernel(const uint16_t* __restrict__ K, const uint16_t* __restrict__ V,
                   const float* __restrict__ anchor, float* __restrict__ k_pool,
                   float* __restrict__ v_summ, float* __restrict__ beta,
                   uint16_t* __restrict__ k_pool16, uint16_t* __restrict__ v_summ16,
                   float* __restrict__ beta_l2, int nbp, int N, int nb, float scale, int mode) {
  using L = RowLayout<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bi = blockIdx.x * kPoolWarps + warp;
  if (bi >= nb) return;
  const size_t bh = blockIdx.y;
  const int c = lane % L::CPR, r0 = lane / L::CPR;
  const size_t row0 = bh * N + (size_t)bi * kBlock;
  const uint16_t* kb = K + row0 * D + c * 8;
  const uint16_t* vb = V + row0 * D + c * 8;

  float a[8];
  {
    const float4* ap = reinterpret_cast<const float4*>(anchor + bh * D + c * 8);
    float4 a0 = ap[0], a1 = ap[1];
    a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
    a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
  }
  constexpr int NBATCH = L::NR < 8 ? L::NR : 8;  // 8 loads in flight per lane
  float ksum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
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
      for (int e = 0; e < 8; ++e) {
        ksum[e] += f[e];
        dot = fmaf(a[e], f[e], dot);
      }
      s[i0 + i] = dot;
    }
  }
  // complete the row dot products across the CPR lanes of a row
#pragma unroll
  for (int off = 1; off < L::CPR; off <<= 1)
#pragma unroll
    for (int i = 0; i < L::NR; ++i) s[i] += __shfl_xor_sync(0xffffffffu, s[i], off);
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < L::NR; ++i) {
    s[i] *= scale;
    mx = fmaxf(mx, s[i]);
  }
#pragma unroll
  for (int off = L::CPR; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float se = 0.f;
#pragma unroll
  for (int i = 0; i < L::NR; ++i) se += expf(s[i] - mx);
#pragma unroll
  for (int off = L::CPR; off < 32; off <<= 1) se += __shfl_xor_sync(0xffffffffu, se, off);
  const float lse = mx + logf(se);

  float vacc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i0 = 0; i0 < L::NR; i0 += NBATCH) {
    uint4 uv[NBATCH];
#pragma unroll
    for (int i = 0; i < NBATCH; ++i) uv[i] = ldg_nc_v4(vb + (size_t)(r0 + L::RPP * (i0 + i)) * D);
#pragma unroll
    for (int i = 0; i < NBATCH; ++i) {
      const float w = (mode == SPARK_POOL_REWEIGHT) ? expf(s[i0 + i] - lse) : (1.0f / kBlock);
      float f[8];
      bf16x8_to_f32(uv[i], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) vacc[e] = fmaf(w, f[e], vacc[e]);
    }
  }
#pragma unroll
  for (int off = L::CPR; off < 32; off <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      vacc[e] += __shfl_xor_sync(0xffffffffu, vacc[e], off);
      ksum[e] += __shfl_xor_sync(0xffffffffu, ksum[e], off);
    }
  float kbar[8];
  float dot = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    kbar[e] = ksum[e] * (1.0f / kBlock);
    dot = fmaf(a[e], kbar[e], dot);
  }
#pragma unroll
  for (int off = 1; off < L::CPR; off <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);

  if (r0 == 0) {
    const size_t o = (bh * nb + bi) * D + c * 8;
    float4* kd = reinterpret_cast<float4*>(k_pool + o);
    float4* vd = reinterpret_cast<float4*>(v_summ + o);
    kd[0] = make_float4(kbar[0], kbar[1], kbar[2], kbar[3]);
    kd[1] = make_float4(kbar[4], kbar[5], kbar[6], kbar[7]);
    vd[0] = make_float4(vacc[0], vacc[1], vacc[2], vacc[3]);
    vd[1] = make_float4(vacc[4], vacc[5], vacc[6], vacc[7]);
    uint4 k16, v16;
    k16.x = pack_bf16x2(kbar[0], kbar[1]); k16.y = pack_bf16x2(kbar[2], kbar[3]);
    k16.z = pack_bf16x2(kbar[4], kbar[5]); k16.w = pack_bf16x2(kbar[6], kbar[7]);
    v16.x = pack_bf16x2(vacc[0], vacc[1]); v16.y = pack_bf16x2(vacc[2], vacc[3]);
    v16.z = pack_bf16x2(vacc[4], vacc[5]); v16.w = pack_bf16x2(vacc[6], vacc[7]);
    *reinterpret_cast<uint4*>(k_pool16 + o) = k16;
    *reinterpret_cast<uint4*>(v_summ16 + o) = v16;
    if (lane == 0) {
      const float b = (mode == SPARK_POOL_REWEIGHT) ? lse - dot * scale : logf((float)kBlock);
      beta[bh * nb + bi] = b;
      // padded log2-scaled copy for the attention kernel; entries past nb are -inf
      beta_l2[bh * nbp + bi] = b * kLog2e;
      for (int j = nb + bi; j < nbp; j += nb) beta_l2[bh * nbp + j] = -INFINITY;
    }
  }
}

}  // namespace spark
