// Exact + compressed block-sparse attention forward on the 5th-generation tensor cores.
//
// Method: "Spark-H3: speeding up MiniMax-H3 in ComfyUI with block-sparse attention",
// section "What Spark-Attn changes": top-ranked key/value blocks are computed exactly, the
// rest through the compressed branch; both feed one online softmax (one log-sum-exp
// merge). Sink/text keys are attended exactly ("ComfyUI adds a core sparse-attention
// node...", sink_conditioning); dense rows attend to every key ("H3 Optimizations"
// README, "Nodes").
//
// Design (sm_100a):
// * The unit of work is one 64-query block: video blocks select their own key blocks,
//   so two query blocks cannot share an MMA B operand. tcgen05.mma with M = 64 runs at
//   half the M = 128 rate, and every key of a 64-query block costs >= 1 KB of shared
//   memory traffic (TMA writes K and V, the tensor core reads them) against a 128 B/clk
//   port, so the kernel keeps everything else out of shared memory: Q and P live in
//   tensor memory (A operand of "TS" MMAs), shared memory only carries the K/V ring.
// * Each persistent CTA runs two independent query blocks ("slots") whose M = 64
//   accumulators share TMEM columns in the two lane halves of every sub-partition
//   (slot 0: lanes 0-15, slot 1: lanes 16-31 of each 32-lane group), so the tensor core
//   works on one slot while the other slot's softmax runs.
// * Warp roles: warps 0-3 softmax of slot 0, warps 4-7 softmax of slot 1 (warp w reads
//   TMEM sub-partition w % 4), warp 8 issues TMA loads, warp 9 issues MMAs and owns TMEM.
// * Per 64-key tile: S = Q K^T (8 MMAs 64x64x16 from TMEM Q and a 128B-swizzled K tile),
//   softmax in base 2 with a lazy running max (O is rescaled only when the row max grows
//   by more than 2^8), P written back over S as bf16, then O += P V (4 MMAs 64xDx16 with
//   V as an MN-major operand). Tile order per video query block: selected blocks, dense
//   key rows, then pooled entries (beta added, selected blocks masked).
// * Every mbarrier wait is bounded; a timeout records SPARK_ETIMEOUT, raises the CTA abort
//   flag, the TMA role drains its copies in flight and TMEM is released.
#pragma once
#include "spark_common.cuh"
#include "tc_util.cuh"

namespace spark {

struct TcMaps {
  CUtensorMap k, v, kp, vp;  // K, V over [B*H*N, D]; pooled pack over [B*H*nb, D]
};

struct TcParams {
  const uint16_t* Q;
  const int32_t* idx;
  const int32_t* cnt;
  const float* beta;
  const int32_t* perm;
  uint16_t* O;
  float* lse;
  int N, nb, kcap, BH, n_dq, pooled, n_items;
  float scale_log2;
};

template <int D>
struct TcCfg {
  static constexpr int kStages = 6;
  static constexpr int kPanels = D / 64;         // 128-byte swizzle panels per row
  static constexpr int kPanelBytes = 64 * 128;   // 64 rows x 128 B
  static constexpr int kTileBytes = 64 * D * 2;  // one K or V tile (64 keys)
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kColS = 0;                // S/P buffers at 0 and 64
  static constexpr int kColO = 128;
  static constexpr int kColQ = 128 + D;
  static constexpr int kTmemCols = (kColQ + D / 2 <= 256) ? 256 : 512;
  static constexpr int kThreads = 320;
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kBarBytes = 1024;
};

struct TcItem {
  int bh, q0, nq, dense, cnt, ntiles;
  size_t row;  // selection row (video items)
};

__device__ __forceinline__ TcItem tc_item(const TcParams& p, int it) {
  TcItem r;
  const int nd = p.BH * p.n_dq;
  const int nv = p.nb * kBlock;
  const int n_dk = (p.N - nv + kBlock - 1) / kBlock;
  if (it < nd) {
    r.bh = it / p.n_dq;
    r.dense = 1;
    r.q0 = nv + (it % p.n_dq) * kBlock;
    r.cnt = 0;
    r.row = 0;
    r.ntiles = (p.N + kBlock - 1) / kBlock;
  } else {
    const int v = it - nd;
    r.bh = v / p.nb;
    r.dense = 0;
    r.q0 = (v % p.nb) * kBlock;
    r.row = (size_t)r.bh * p.nb + (v % p.nb);
    int c = p.cnt[r.row];
    c = c < 0 ? 0 : (c > p.kcap ? p.kcap : c);
    r.cnt = c;
    r.ntiles = c + n_dk + (p.pooled ? (p.nb + kBlock - 1) / kBlock : 0);
  }
  r.nq = min(kBlock, p.N - r.q0);
  return r;
}

// Row coordinate of tile t in the K/V (or pooled pack) tensor map.
__device__ __forceinline__ int tc_tile_row(const TcParams& p, const TcItem& I, int t, int* pooled) {
  const int nv = p.nb * kBlock;
  const int n_dk = (p.N - nv + kBlock - 1) / kBlock;
  *pooled = 0;
  if (I.dense) return I.bh * p.N + t * kBlock;
  if (t < I.cnt) {
    int b = p.idx[I.row * (size_t)p.kcap + t];
    if (b < 0 || b >= p.nb) b = 0;  // masked by the softmax, reported there
    return I.bh * p.N + b * kBlock;
  }
  if (t < I.cnt + n_dk) return I.bh * p.N + nv + (t - I.cnt) * kBlock;
  *pooled = 1;
  return I.bh * p.nb + (t - I.cnt - n_dk) * kBlock;
}

// Slot s of CTA c walks items 2c + s, 2c + s + 2G, ... and skips items without tiles.
struct TcSlotWalk {
  int it, stride, n;
  __device__ __forceinline__ bool next_nonempty(const TcParams& p, TcItem* I) {
    while (it < n) {
      *I = tc_item(p, it);
      it += stride;
      if (I->ntiles > 0) return true;
    }
    return false;
  }
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Bounded wait that ignores the abort flag (used to drain copies in flight on abort).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!tc::mbar_try_wait(bar, parity))
    if (clock64() - t0 > tc::kWaitClocks) return;
}

template <int D>
__device__ __forceinline__ uint64_t tc_kdesc(uint32_t stage_addr, int kk) {
  // K tile: K-major, 128B swizzle; k-step kk covers d = 16kk .. 16kk+15
  return tc::make_sdesc(stage_addr + (kk >> 2) * TcCfg<D>::kPanelBytes + (kk & 3) * 32, 16, 1024,
                        tc::kSwizzle128);
}
template <int D>
__device__ __forceinline__ uint64_t tc_vdesc(uint32_t stage_addr, int kk) {
  // V tile as an MN-major operand (N = d): k-step kk covers keys 16kk .. 16kk+15 (two 8-row
  // atoms of 1 KB); the d panels are kPanelBytes apart.
  return tc::make_sdesc(stage_addr + TcCfg<D>::kTileBytes + kk * 2048, TcCfg<D>::kPanelBytes, 1024,
                        tc::kSwizzle128);
}

template <int D>
__global__ void __launch_bounds__(320, 1)
    attn_tc_kernel(const __grid_constant__ TcMaps maps, const TcParams p) {
  using C = TcCfg<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ring = smem;
  uint64_t* kfull = reinterpret_cast<uint64_t*>(ring + C::kRingBytes);
  uint64_t* vfull = kfull + C::kStages;
  uint64_t* kvempty = vfull + C::kStages;
  uint64_t* sfull = kvempty + C::kStages;  // [slot][buf]
  uint64_t* pfull = sfull + 4;             // [slot][buf]
  uint64_t* oready = pfull + 4;            // [slot]
  uint64_t* qfull = oready + 2;            // [slot]
  uint64_t* ofree = qfull + 2;             // [slot]
  uint64_t* finbar = ofree + 2;            // all MMAs of the CTA done
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(finbar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(ring + C::kRingBytes + C::kBarBytes);
  const int nbw = (p.nb + 31) / 32;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      tc::mbar_init(&kfull[i], 1);
      tc::mbar_init(&vfull[i], 1);
      tc::mbar_init(&kvempty[i], 1);
    }
    for (int i = 0; i < 4; ++i) {
      tc::mbar_init(&sfull[i], 1);
      tc::mbar_init(&pfull[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&oready[i], 1);
      tc::mbar_init(&qfull[i], 4);
      tc::mbar_init(&ofree[i], 4);
    }
    tc::mbar_init(finbar, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 9) {
    tc::tmem_alloc(tmem_holder, C::kTmemCols);
    tc::tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tc::tma_prefetch_desc(&maps.k);
    tc::tma_prefetch_desc(&maps.v);
    tc::tma_prefetch_desc(&maps.kp);
    tc::tma_prefetch_desc(&maps.vp);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  const int stride = 2 * gridDim.x;

  if (warp == 8) {
    // ================================================================ TMA producer
    if (lane == 0) {
      TcSlotWalk walk[2] = {{2 * (int)blockIdx.x, stride, p.n_items},
                            {2 * (int)blockIdx.x + 1, stride, p.n_items}};
      TcItem cur[2];
      bool have[2];
      int t[2] = {0, 0};
      for (int s = 0; s < 2; ++s) have[s] = walk[s].next_nonempty(p, &cur[s]);
      uint32_t q = 0;
      bool ok = true;
      while (ok && (have[0] || have[1])) {
        for (int s = 0; s < 2 && ok; ++s) {
          if (!have[s]) continue;
          const int stage = q % C::kStages;
          if (q >= (uint32_t)C::kStages &&
              !tc::mbar_wait(&kvempty[stage], ((q / C::kStages) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          int pooled;
          const int y = tc_tile_row(p, cur[s], t[s], &pooled);
          const CUtensorMap* mk = pooled ? &maps.kp : &maps.k;
          const CUtensorMap* mv = pooled ? &maps.vp : &maps.v;
          unsigned char* st = ring + stage * C::kStageBytes;
          tc::mbar_expect_tx(&kfull[stage], C::kTileBytes);
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn)
            tc::tma_load_2d(st + pn * C::kPanelBytes, mk, pn * 64, y, &kfull[stage]);
          tc::mbar_expect_tx(&vfull[stage], C::kTileBytes);
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn)
            tc::tma_load_2d(st + C::kTileBytes + pn * C::kPanelBytes, mv, pn * 64, y, &vfull[stage]);
          ++q;
          if (++t[s] == cur[s].ntiles) {
            t[s] = 0;
            have[s] = walk[s].next_nonempty(p, &cur[s]);
          }
        }
      }
      if (!ok || *abort_flag) {
        // drain every copy that may still be in flight before the CTA leaves
        const uint32_t first = q > (uint32_t)C::kStages ? q - C::kStages : 0;
        for (uint32_t j = first; j < q; ++j) {
          mbar_drain(&kfull[j % C::kStages], (j / C::kStages) & 1);
          mbar_drain(&vfull[j % C::kStages], (j / C::kStages) & 1);
        }
      }
    }
  } else if (warp == 9) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = tc::make_idesc_bf16(64, 64, 0, 0);
      constexpr uint32_t idPV = tc::make_idesc_bf16(64, D, 0, 1);
      TcSlotWalk walk[2] = {{2 * (int)blockIdx.x, stride, p.n_items},
                            {2 * (int)blockIdx.x + 1, stride, p.n_items}};
      TcItem cur[2];
      bool have[2];
      int t[2] = {0, 0};
      uint32_t g[2] = {0, 0};       // tiles issued per slot (all items)
      uint32_t nitem[2] = {0, 0};   // non-empty items started per slot
      struct Pend {
        int valid;
        uint32_t q, g, item;
        int first;
      } pend[2] = {{0, 0, 0, 0, 0}, {0, 0, 0, 0, 0}};
      for (int s = 0; s < 2; ++s) have[s] = walk[s].next_nonempty(p, &cur[s]);
      const uint32_t ring_addr = tc::smem_addr(ring);
      bool ok = true;
      auto issue_pv = [&](int s, const Pend& pe) -> bool {
        const uint32_t b = pe.g & 1;
        if (!tc::mbar_wait(&pfull[2 * s + b], (pe.g >> 1) & 1, abort_flag)) return false;
        const int stage = pe.q % C::kStages;
        if (!tc::mbar_wait(&vfull[stage], (pe.q / C::kStages) & 1, abort_flag)) return false;
        if (pe.first && pe.item > 0 && !tc::mbar_wait(&ofree[s], (pe.item - 1) & 1, abort_flag))
          return false;
        tc::tc_fence_after();
        const uint32_t lanes = (uint32_t)(16 * s) << 16;
        const uint32_t st = ring_addr + stage * C::kStageBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc::mma_ts(tbase + lanes + C::kColO, tbase + lanes + C::kColS + 64 * b + kk * 8,
                     tc_vdesc<D>(st, kk), idPV, (pe.first && kk == 0) ? 0u : 1u);
        tc::mma_commit(&kvempty[stage]);
        tc::mma_commit(&oready[s]);
        return true;
      };
      uint32_t q = 0;
      while (ok && (have[0] || have[1])) {
        for (int s = 0; s < 2 && ok; ++s) {
          if (!have[s]) continue;
          if (t[s] == 0 && !tc::mbar_wait(&qfull[s], nitem[s] & 1, abort_flag)) {
            ok = false;
            break;
          }
          const int stage = q % C::kStages;
          if (!tc::mbar_wait(&kfull[stage], (q / C::kStages) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t b = g[s] & 1;
          const uint32_t lanes = (uint32_t)(16 * s) << 16;
          const uint32_t st = ring_addr + stage * C::kStageBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            tc::mma_ts(tbase + lanes + C::kColS + 64 * b, tbase + lanes + C::kColQ + kk * 8,
                       tc_kdesc<D>(st, kk), idS, kk > 0 ? 1u : 0u);
          tc::mma_commit(&sfull[2 * s + b]);
          if (pend[s].valid && !issue_pv(s, pend[s])) {
            ok = false;
            break;
          }
          pend[s].valid = 1;
          pend[s].q = q;
          pend[s].g = g[s];
          pend[s].item = nitem[s];
          pend[s].first = (t[s] == 0);
          ++q;
          ++g[s];
          if (++t[s] == cur[s].ntiles) {
            t[s] = 0;
            ++nitem[s];
            have[s] = walk[s].next_nonempty(p, &cur[s]);
            if (!have[s]) {  // this slot is done: release its last tile now
              if (!issue_pv(s, pend[s])) {
                ok = false;
                break;
              }
              pend[s].valid = 0;
            }
          }
        }
      }
      for (int s = 0; s < 2 && ok; ++s)
        if (pend[s].valid && !issue_pv(s, pend[s])) ok = false;
      // every MMA of this CTA must be complete before TMEM is released
      tc::mma_commit(finbar);
      mbar_drain(finbar, 0);
    }
  } else {
    // ================================================================ softmax (slot s)
    const int s = warp >> 2;
    const int w = warp & 3;
    const int r = 16 * w + (lane & 15);  // query row within the block
    const int h = lane >> 4;             // key half (scores) / d half (O, Q)
    const uint32_t lanes = (uint32_t)(32 * w + 16 * s) << 16;
    uint32_t* bm = bitmap + warp * nbw;  // this warp's selection bitmap
    const int nv = p.nb * kBlock;
    const int n_dk = (p.N - nv + kBlock - 1) / kBlock;

    TcSlotWalk walk = {2 * (int)blockIdx.x + s, stride, p.n_items};
    uint32_t g = 0;
    int have_prev = 0;
    TcItem prev;
    prev.ntiles = 0;
    float m_prev = -INFINITY, l_prev = 0.f;
    uint32_t g_prev_last = 0;
    uint32_t nitem = 0;
    int cur_bad = 0;

    auto epilogue = [&](const TcItem& I, float m_run, float l_run, uint32_t g_last) -> bool {
      // oready completes once per PV. Two PVs may still be outstanding here, and a parity
      // wait only tells phases apart within one phase of the barrier, so step through
      // PV(g_last - 1) before PV(g_last).
      if (g_last > 0 && !tc::mbar_wait(&oready[s], (g_last - 1) & 1, abort_flag)) return false;
      if (!tc::mbar_wait(&oready[s], g_last & 1, abort_flag)) return false;
      tc::tc_fence_after();
      const float l_tot = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
      const float inv = l_tot > 0.f ? 1.0f / l_tot : 0.f;
      int orow = I.q0 + r;
      bool write = r < I.nq;
      if (write && !I.dense && p.perm != nullptr) {
        orow = p.perm[(size_t)I.bh * nv + I.q0 + r];
        if (orow < 0 || orow >= nv) {
          set_error(SPARK_EDEVICE_INDEX);
          write = false;
        }
      }
      uint16_t* dst = p.O + ((size_t)I.bh * p.N + orow) * D + h * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[16];
        tc::tmem_ld_16x32bx2_x16<D / 2>(tbase + lanes + C::kColO + 16 * c, v);
        tc::tmem_wait_ld();
        if (write) {
          uint4 o0, o1;
          o0.x = pack_bf16x2(__uint_as_float(v[0]) * inv, __uint_as_float(v[1]) * inv);
          o0.y = pack_bf16x2(__uint_as_float(v[2]) * inv, __uint_as_float(v[3]) * inv);
          o0.z = pack_bf16x2(__uint_as_float(v[4]) * inv, __uint_as_float(v[5]) * inv);
          o0.w = pack_bf16x2(__uint_as_float(v[6]) * inv, __uint_as_float(v[7]) * inv);
          o1.x = pack_bf16x2(__uint_as_float(v[8]) * inv, __uint_as_float(v[9]) * inv);
          o1.y = pack_bf16x2(__uint_as_float(v[10]) * inv, __uint_as_float(v[11]) * inv);
          o1.z = pack_bf16x2(__uint_as_float(v[12]) * inv, __uint_as_float(v[13]) * inv);
          o1.w = pack_bf16x2(__uint_as_float(v[14]) * inv, __uint_as_float(v[15]) * inv);
          *reinterpret_cast<uint4*>(dst + 16 * c) = o0;
          *reinterpret_cast<uint4*>(dst + 16 * c + 8) = o1;
        }
      }
      if (write && h == 0 && p.lse != nullptr)
        p.lse[(size_t)I.bh * p.N + orow] = l_tot > 0.f ? (m_run + __log2f(l_tot)) * kLn2 : -INFINITY;
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&ofree[s]);
      return true;
    };

    bool ok = true;
    while (ok) {
      // ---- next item of this slot (possibly empty)
      TcItem I;
      bool more = false;
      while (walk.it < walk.n) {
        I = tc_item(p, walk.it);
        walk.it += walk.stride;
        if (I.ntiles > 0) {
          more = true;
          break;
        }
        // an item with nothing to attend to: O = 0, LSE = -inf
        if (r < I.nq) {
          int orow = I.q0 + r;
          bool write = true;
          if (!I.dense && p.perm != nullptr) {
            orow = p.perm[(size_t)I.bh * nv + I.q0 + r];
            write = orow >= 0 && orow < nv;
          }
          if (write) {
            uint4 z = make_uint4(0, 0, 0, 0);
            uint16_t* dst = p.O + ((size_t)I.bh * p.N + orow) * D + h * (D / 2);
#pragma unroll
            for (int c = 0; c < D / 16; ++c) *reinterpret_cast<uint4*>(dst + 8 * c) = z;
            if (h == 0 && p.lse != nullptr) p.lse[(size_t)I.bh * p.N + orow] = -INFINITY;
          }
        }
      }
      if (more) {
        // ---- selection bitmap (pooled masking) and index validity, one copy per warp so
        //      that no barrier wider than a warp is needed
        int bad_idx = 0;
        if (!I.dense && (p.pooled || I.cnt > 0)) {
          for (int i = lane; i < nbw; i += 32) bm[i] = 0u;
          __syncwarp();
          const int32_t* ip = p.idx + I.row * (size_t)p.kcap;
          int bad = 0;
          for (int i = lane; i < I.cnt; i += 32) {
            const int b = ip[i];
            if (b >= 0 && b < p.nb) atomicOr(&bm[b >> 5], 1u << (b & 31));
            else bad = 1;
          }
          bad_idx = __any_sync(0xffffffffu, bad);
          if (bad_idx && lane == 0) set_error(SPARK_EDEVICE_INDEX);
          if (lane == 0 && w == 0 && p.cnt[I.row] != I.cnt) set_error(SPARK_EDEVICE_INDEX);
          __syncwarp();
        }
        cur_bad = bad_idx;
        // ---- Q block into TMEM (bf16 pairs, A-operand layout of the M = 64 MMA)
        {
          const bool rv = r < I.nq;
          const uint16_t* qrow = p.Q + ((size_t)I.bh * p.N + I.q0 + (rv ? r : 0)) * D + h * (D / 2);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t v[16];
            uint4 a = rv ? ldg_nc_v4(qrow + 32 * c) : make_uint4(0, 0, 0, 0);
            uint4 b2 = rv ? ldg_nc_v4(qrow + 32 * c + 8) : make_uint4(0, 0, 0, 0);
            uint4 c2 = rv ? ldg_nc_v4(qrow + 32 * c + 16) : make_uint4(0, 0, 0, 0);
            uint4 d2 = rv ? ldg_nc_v4(qrow + 32 * c + 24) : make_uint4(0, 0, 0, 0);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b2.x; v[5] = b2.y; v[6] = b2.z; v[7] = b2.w;
            v[8] = c2.x; v[9] = c2.y; v[10] = c2.z; v[11] = c2.w;
            v[12] = d2.x; v[13] = d2.y; v[14] = d2.z; v[15] = d2.w;
            tc::tmem_st_16x32bx2_x16<D / 4>(tbase + lanes + C::kColQ + 16 * c, v);
          }
          tc::tmem_wait_st();
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&qfull[s]);
        }
      }
      // ---- finish the previous item (its last PV was issued after this item's first S)
      if (have_prev) {
        if (!epilogue(prev, m_prev, l_prev, g_prev_last)) {
          ok = false;
          break;
        }
        have_prev = 0;
      }
      if (!more) break;

      // ---- tiles of this item
      const int bad_idx = cur_bad;
      float m_run = -INFINITY, l_run = 0.f;
      for (int t = 0; t < I.ntiles; ++t, ++g) {
        const uint32_t b = g & 1;
        if (!tc::mbar_wait(&sfull[2 * s + b], (g >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        uint32_t sv[32];
        tc::tmem_ld_16x32bx2_x16<32>(tbase + lanes + C::kColS + 64 * b, sv);
        tc::tmem_ld_16x32bx2_x16<32>(tbase + lanes + C::kColS + 64 * b + 16, sv + 16);
        tc::tmem_wait_ld();
        // ---- logits (base 2) and masks
        float x[32];
        int kind = 0, valid = kBlock, j0 = 0;
        if (I.dense) {
          valid = min(kBlock, p.N - t * kBlock);
        } else if (t < I.cnt) {
          if (bad_idx) {
            const int bb = p.idx[I.row * (size_t)p.kcap + t];
            if (bb < 0 || bb >= p.nb) valid = 0;
          }
        } else if (t < I.cnt + n_dk) {
          valid = min(kBlock, p.N - (nv + (t - I.cnt) * kBlock));
        } else {
          kind = 1;
          j0 = (t - I.cnt - n_dk) * kBlock;
          valid = min(kBlock, p.nb - j0);
        }
        const int kb0 = 32 * h;  // first key of this thread's half
        if (kind == 0) {
          if (valid >= kBlock) {
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(sv[j]) * p.scale_log2;
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              x[j] = (kb0 + j < valid) ? __uint_as_float(sv[j]) * p.scale_log2 : -INFINITY;
          }
        } else {
          const float* bp = p.beta + (size_t)I.bh * p.nb;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int jj = min(j0 + kb0 + j, p.nb - 1);
            const bool m = (kb0 + j >= valid) || ((bm[jj >> 5] >> (jj & 31)) & 1u);
            x[j] = m ? -INFINITY : fmaf(__uint_as_float(sv[j]), p.scale_log2, bp[jj] * kLog2e);
          }
        }
        float mx = x[0];
#pragma unroll
        for (int j = 1; j < 32; ++j) mx = fmaxf(mx, x[j]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_run, mx);
        const bool need = m_new > m_run + 8.0f;  // also true when m_run = -inf and m_new finite
        const float alpha = need ? ex2f(m_run - m_new) : 1.0f;
        if (__any_sync(0xffffffffu, need && t > 0)) {
          // rescale the O rows of this warp once the previous PV has landed
          if (!tc::mbar_wait(&oready[s], (g - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t v[16];
            tc::tmem_ld_16x32bx2_x16<D / 2>(tbase + lanes + C::kColO + 16 * c, v);
            tc::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha);
            tc::tmem_st_16x32bx2_x16<D / 2>(tbase + lanes + C::kColO + 16 * c, v);
          }
        }
        if (need) {
          l_run *= alpha;
          m_run = m_new;
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        uint32_t pk[16];
        float ls = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float p0 = ex2f(x[2 * j] - m_use);
          const float p1 = ex2f(x[2 * j + 1] - m_use);
          ls += p0 + p1;
          pk[j] = pack_bf16x2(p0, p1);
        }
        l_run += ls;
        tc::tmem_st_16x32bx2_x16<16>(tbase + lanes + C::kColS + 64 * b, pk);
        tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&pfull[2 * s + b]);
      }
      if (!ok) break;
      have_prev = 1;
      prev = I;
      m_prev = m_run;
      l_prev = l_run;
      g_prev_last = g - 1;
      ++nitem;
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 9) tc::tmem_dealloc(tbase, C::kTmemCols);
}

}  // namespace spark
