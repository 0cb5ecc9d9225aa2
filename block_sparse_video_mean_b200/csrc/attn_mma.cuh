// Exact + compressed block-sparse attention forward, warp-level mma.sync version.
//
// Method: "Spark-H3: speeding up MiniMax-H3 in ComfyUI with block-sparse attention",
// section "What Spark-Attn changes": the exact branch computes the top-ranked key/value
// blocks in full and the compressed branch covers every other block; here both feed one
// online softmax (one log-sum-exp merge). Sink/text keys are always attended exactly
// ("ComfyUI adds a core sparse-attention node...", sink_conditioning) and dense rows
// (sinks, ragged tail) attend to every key ("H3 Optimizations" README, "Nodes").
//
// One CTA (4 warps) owns one 64-query block; each warp owns 16 query rows. Key/value
// tiles of 64 rows stream through a two-stage cp.async ring in XOR-swizzled shared
// memory (conflict-free ldmatrix). For a video query block the tile sequence is: the
// selected blocks, the dense key rows, then (compressed branch on) the pooled entries
// of all video blocks with the selected ones masked out and beta added to the logits.
// Dense query blocks walk every key. The softmax runs in base 2 with the scale folded
// into the exponent.
#pragma once
#include "spark_common.cuh"

namespace spark {

struct AttnParams {
  const uint16_t* Q;
  const uint16_t* K;
  const uint16_t* V;
  const int32_t* idx;
  const int32_t* cnt;
  const uint16_t* kp16;  // pooled keys, bf16 [BH, nb, D] (nullable: compressed branch off)
  const uint16_t* vp16;  // pooled values, bf16 [BH, nb, D]
  const float* beta;     // [BH, nb]
  const int32_t* perm;   // [BH, nb*64] (nullable)
  uint16_t* O;
  float* lse;  // nullable
  int N, nb, kcap, BH;
  int n_dq;  // dense query blocks per head
  float scale_log2;
};

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte chunk `ch` of row `row` in a [64][D] bf16 tile.
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int ch) {
  return (uint32_t)(row * D * 2 + ((ch ^ (row & 7)) << 4));
}

template <int D>
struct MmaAttn {
  static constexpr int kThreads = 128;
  static constexpr int kChunks = D / 8;
  static constexpr int kTile = 64 * D * 2;  // bytes of one K or V tile
  static constexpr int kSmemFixed = kTile /*Q*/ + 4 * kTile /*K,V x 2 stages*/;
};

// Tile t of a work item: which rows feed K/V, how many are valid, and how to mask.
struct TileSrc {
  const uint16_t* k;
  const uint16_t* v;
  int valid;  // rows 0..valid-1 of the tile are real
  int kind;   // 0 exact rows, 1 pooled entries (bias + selection mask)
  int j0;     // first pooled entry of the tile (kind 1)
};

template <int D>
__global__ void __launch_bounds__(128) attn_mma_kernel(AttnParams p) {
  using C = MmaAttn<D>;
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned char* sQ = smem;
  unsigned char* sKV = smem + C::kTile;  // stage s: K at 2s*kTile, V at (2s+1)*kTile
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + C::kSmemFixed);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- work item
  const int item = blockIdx.x;
  const int n_dense_items = p.BH * p.n_dq;
  const bool dense_q = item < n_dense_items;
  int bh, qb;
  if (dense_q) {
    bh = item / p.n_dq;
    qb = item % p.n_dq;
  } else {
    bh = (item - n_dense_items) / p.nb;
    qb = (item - n_dense_items) % p.nb;
  }
  const int nv = p.nb * kBlock;
  const int q0 = dense_q ? nv + qb * kBlock : qb * kBlock;
  const int nq = min(kBlock, p.N - q0);
  const size_t head = (size_t)bh * p.N;
  const uint16_t* Kh = p.K + head * D;
  const uint16_t* Vh = p.V + head * D;

  int cnt = 0;
  const int32_t* idx = nullptr;
  const int n_dk = (p.N - nv + kBlock - 1) / kBlock;  // dense key tiles
  const bool pooled = !dense_q && p.kp16 != nullptr;
  const int n_pk = pooled ? (p.nb + kBlock - 1) / kBlock : 0;
  int ntiles;
  if (dense_q) {
    ntiles = (p.N + kBlock - 1) / kBlock;
  } else {
    const size_t row = (size_t)bh * p.nb + qb;
    cnt = p.cnt[row];
    if (cnt < 0 || cnt > p.kcap) {
      set_error(SPARK_EDEVICE_INDEX);
      cnt = cnt < 0 ? 0 : p.kcap;
    }
    idx = p.idx + row * p.kcap;
    ntiles = cnt + n_dk + n_pk;
  }
  if (pooled) {
    const int nw = (p.nb + 31) / 32;
    for (int w = tid; w < nw; w += C::kThreads) bitmap[w] = 0u;
    __syncthreads();
    for (int t = tid; t < cnt; t += C::kThreads) {
      const int b = idx[t];
      if (b >= 0 && b < p.nb) atomicOr(&bitmap[b >> 5], 1u << (b & 31));
    }
    // (visibility to all threads is ensured by the __syncthreads in the main loop)
  }

  auto tile_src = [&](int t) -> TileSrc {
    TileSrc s;
    s.kind = 0;
    s.j0 = 0;
    if (dense_q) {
      const int r0 = t * kBlock;
      s.k = Kh + (size_t)r0 * D;
      s.v = Vh + (size_t)r0 * D;
      s.valid = min(kBlock, p.N - r0);
    } else if (t < cnt) {
      const int b = idx[t];
      const bool ok = b >= 0 && b < p.nb;
      if (!ok) set_error(SPARK_EDEVICE_INDEX);
      const int r0 = ok ? b * kBlock : 0;
      s.k = Kh + (size_t)r0 * D;
      s.v = Vh + (size_t)r0 * D;
      s.valid = ok ? kBlock : 0;
    } else if (t < cnt + n_dk) {
      const int r0 = nv + (t - cnt) * kBlock;
      s.k = Kh + (size_t)r0 * D;
      s.v = Vh + (size_t)r0 * D;
      s.valid = min(kBlock, p.N - r0);
    } else {
      const int j0 = (t - cnt - n_dk) * kBlock;
      const size_t o = ((size_t)bh * p.nb + j0) * D;
      s.k = p.kp16 + o;
      s.v = p.vp16 + o;
      s.valid = min(kBlock, p.nb - j0);
      s.kind = 1;
      s.j0 = j0;
    }
    return s;
  };

  auto load_tile = [&](int t, int stage) {
    const TileSrc s = tile_src(t);
    const uint32_t kb = smem_u32(sKV + (2 * stage) * C::kTile);
    const uint32_t vb = smem_u32(sKV + (2 * stage + 1) * C::kTile);
#pragma unroll
    for (int e = tid; e < kBlock * C::kChunks; e += C::kThreads) {
      const int r = e / C::kChunks, ch = e % C::kChunks;
      const bool ok = r < s.valid;
      const size_t o = ok ? (size_t)r * D + ch * 8 : 0;
      cp_async16(kb + swz<D>(r, ch), s.k + o, ok);
      cp_async16(vb + swz<D>(r, ch), s.v + o, ok);
    }
  };

  // ---- prologue: Q block and tile 0
  {
    const uint16_t* Qb = p.Q + (head + q0) * D;
    const uint32_t qbase = smem_u32(sQ);
#pragma unroll
    for (int e = tid; e < kBlock * C::kChunks; e += C::kThreads) {
      const int r = e / C::kChunks, ch = e % C::kChunks;
      const bool ok = r < nq;
      cp_async16(qbase + swz<D>(r, ch), Qb + (ok ? (size_t)r * D + ch * 8 : 0), ok);
    }
  }
  if (ntiles > 0) load_tile(0, 0);
  cp_async_commit();

  uint32_t qf[D / 16][4];
  float o_acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o_acc[n][0] = o_acc[n][1] = o_acc[n][2] = o_acc[n][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  const int wr = warp * 16;  // first query row of this warp

  for (int t = 0; t < ntiles || t == 0; ++t) {
    if (t + 1 < ntiles) {
      load_tile(t + 1, (t + 1) & 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (t == 0) {
      const uint32_t qbase = smem_u32(sQ);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int mi = lane >> 3;
        const int row = wr + (mi & 1) * 8 + (lane & 7);
        ldsm_x4(qbase + swz<D>(row, 2 * kk + (mi >> 1)), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
    }
    if (ntiles == 0) break;
    const TileSrc src = tile_src(t);
    const uint32_t kb = smem_u32(sKV + (2 * (t & 1)) * C::kTile);
    const uint32_t vb = smem_u32(sKV + (2 * (t & 1) + 1) * C::kTile);

    // ---- S = Q K^T (16 x 64 per warp)
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int mi = lane >> 3;
        const int key = 16 * np + (mi >> 1) * 8 + (lane & 7);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + swz<D>(key, 2 * kk + (mi & 1)), b0, b1, b2, b3);
        mma_bf16_16816(s[2 * np], qf[kk], b0, b1);
        mma_bf16_16816(s[2 * np + 1], qf[kk], b2, b3);
      }
    }
    // ---- logits in base 2, masks and bias
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kj = 8 * n + 2 * (lane & 3) + (e & 1);
        float x = s[n][e] * p.scale_log2;
        if (kj >= src.valid) {
          x = -INFINITY;
        } else if (src.kind == 1) {
          const int j = src.j0 + kj;
          if ((bitmap[j >> 5] >> (j & 31)) & 1u) x = -INFINITY;
          else x += p.beta[(size_t)bh * p.nb + j] * kLog2e;
        }
        s[n][e] = x;
        mx[e >> 1] = fmaxf(mx[e >> 1], x);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
    }
    float m_use[2], alpha[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float m_new = fmaxf(m_run[h], mx[h]);
      m_use[h] = (m_new == -INFINITY) ? 0.f : m_new;
      alpha[h] = exp2f(m_run[h] - m_use[h]);
      m_run[h] = m_new;
      l_run[h] *= alpha[h];
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      o_acc[n][0] *= alpha[0];
      o_acc[n][1] *= alpha[0];
      o_acc[n][2] *= alpha[1];
      o_acc[n][3] *= alpha[1];
    }
    uint32_t pf[4][4];  // P as A fragments, one per 16-key step
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const float p0 = exp2f(s[n][0] - m_use[0]);
      const float p1 = exp2f(s[n][1] - m_use[0]);
      const float p2 = exp2f(s[n][2] - m_use[1]);
      const float p3 = exp2f(s[n][3] - m_use[1]);
      l_run[0] += p0 + p1;
      l_run[1] += p2 + p3;
      pf[n >> 1][(n & 1) * 2 + 0] = pack_bf16x2(p0, p1);
      pf[n >> 1][(n & 1) * 2 + 1] = pack_bf16x2(p2, p3);
    }
    // ---- O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {
        const int mi = lane >> 3;
        const int key = 16 * kk + (mi & 1) * 8 + (lane & 7);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + swz<D>(key, 2 * np + (mi >> 1)), b0, b1, b2, b3);
        mma_bf16_16816(o_acc[2 * np], pf[kk], b0, b1);
        mma_bf16_16816(o_acc[2 * np + 1], pf[kk], b2, b3);
      }
    }
    __syncthreads();  // stage (t & 1) is reloaded by the next-but-one iteration
  }

  // ---- epilogue
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = wr + (lane >> 2) + 8 * h;
    if (r >= nq) continue;
    const float inv = l_run[h] > 0.f ? 1.0f / l_run[h] : 0.f;
    int orow = q0 + r;
    if (!dense_q && p.perm != nullptr) {
      orow = p.perm[(size_t)bh * nv + q0 + r];
      if (orow < 0 || orow >= nv) {
        set_error(SPARK_EDEVICE_INDEX);
        continue;
      }
    }
    uint16_t* dst = p.O + (head + orow) * D + 2 * (lane & 3);
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
      *reinterpret_cast<uint32_t*>(dst + 8 * n) =
          pack_bf16x2(o_acc[n][2 * h] * inv, o_acc[n][2 * h + 1] * inv);
    if (p.lse != nullptr && (lane & 3) == 0)
      p.lse[head + orow] = l_run[h] > 0.f ? (m_run[h] + log2f(l_run[h])) * kLn2 : -INFINITY;
  }
}

}  // namespace spark
