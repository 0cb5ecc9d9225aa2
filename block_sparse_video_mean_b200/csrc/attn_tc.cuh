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
//   TMEM sub-partition w % 4), warp 8 fills the K ring and warp 10 the V ring with TMA,
//   warp 9 issues MMAs and owns TMEM. K stages are released when their S MMAs complete and
//   V stages when their PV MMAs complete, so neither producer waits on an MMA that the
//   issuer can only start later.
// * A tile is 128 keys made of two 64-key halves (a selected block, 64 dense rows or 64
//   pooled entries each; per video query block the halves run selected blocks, dense key
//   rows, then pooled entries). Per tile: S = Q K^T (8 MMAs 64x128x16 from TMEM Q and a
//   128B-swizzled K tile), softmax in base 2 (each thread owns one half of one row) with a
//   lazy running max (O is rescaled only when the row max grows by more than 2^8), P
//   written back over S as bf16, then O += P V (8 MMAs 64xDx16, V as an MN-major operand).
// * Every mbarrier wait is bounded; a timeout records SPARK_ETIMEOUT, raises the CTA abort
//   flag, the TMA role drains its copies in flight and TMEM is released.
#pragma once
#include "spark_common.cuh"
#include "tc_util.cuh"

// Timing hooks for out-of-tree instrumented builds; no-ops here.
#ifndef SPARK_TC_T0
#define SPARK_TC_T0(v)
#define SPARK_TC_ACC(slot, v)
#define SPARK_TC_EV(who, what)
#define SPARK_TC_DECL
#define SPARK_TC_FLUSH
#endif

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
  // A tile is 128 keys: two 64-key halves (each a selected block, 64 dense rows or 64
  // pooled entries), so S = Q K^T is one N = 128 MMA per K step.
  static constexpr int kStages = D == 128 ? 3 : 6;
  static constexpr int kPanels = D / 64;           // 128-byte swizzle panels per row
  static constexpr int kHalfBytes = 64 * 128;      // 64 rows x 128 B (one TMA box)
  static constexpr int kPanelBytes = 128 * 128;    // 128 rows x 128 B
  static constexpr int kTileBytes = 128 * D * 2;   // K (or V) of one 128-key tile
  static constexpr int kColS = 0;                  // S/P buffers at 0 and 128
  static constexpr int kColO = 256;
  static constexpr int kColQ = 256 + D;
  static constexpr int kTmemCols = 512;
  static constexpr int kThreads = 352;
  static constexpr int kRingBytes = 2 * kStages * kTileBytes;  // K ring, then V ring
  static constexpr int kBarBytes = 1024;
};

struct TcItem {
  int bh, q0, nq, dense, cnt, nhalf, ntiles;  // nhalf 64-key halves, ntiles = ceil(nhalf / 2)
  size_t row;                                  // selection row (video items)
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
    r.nhalf = (p.N + kBlock - 1) / kBlock;
  } else {
    const int v = it - nd;
    r.bh = v / p.nb;
    r.dense = 0;
    r.q0 = (v % p.nb) * kBlock;
    r.row = (size_t)r.bh * p.nb + (v % p.nb);
    int c = p.cnt[r.row];
    c = c < 0 ? 0 : (c > p.kcap ? p.kcap : c);
    r.cnt = c;
    r.nhalf = c + n_dk + (p.pooled ? (p.nb + kBlock - 1) / kBlock : 0);
  }
  r.ntiles = (r.nhalf + 1) / 2;
  r.nq = min(kBlock, p.N - r.q0);
  return r;
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

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

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
  // K tile (128 rows): K-major, 128B swizzle; k-step kk covers d = 16kk .. 16kk+15
  return tc::make_sdesc(stage_addr + (kk >> 2) * TcCfg<D>::kPanelBytes + (kk & 3) * 32, 16, 1024,
                        tc::kSwizzle128);
}
template <int D>
__device__ __forceinline__ uint64_t tc_vdesc(uint32_t stage_addr, int kk) {
  // V tile as an MN-major operand (N = d): k-step kk covers keys 16kk .. 16kk+15 (two 8-row
  // atoms of 1 KB); the d panels are kPanelBytes apart.
  return tc::make_sdesc(stage_addr + kk * 2048, TcCfg<D>::kPanelBytes, 1024, tc::kSwizzle128);
}

template <int D>
__global__ void __launch_bounds__(352, 1)
    attn_tc_kernel(const __grid_constant__ TcMaps maps, const TcParams p) {
  using C = TcCfg<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ring = smem;
  unsigned char* vring = ring + C::kStages * C::kTileBytes;
  uint64_t* kfull = reinterpret_cast<uint64_t*>(ring + C::kRingBytes);
  uint64_t* vfull = kfull + C::kStages;
  uint64_t* kempty = vfull + C::kStages;   // K stage free: its S MMAs completed
  uint64_t* vempty = kempty + C::kStages;  // V stage free: its PV MMAs completed
  uint64_t* sfull = vempty + C::kStages;   // [slot][buf]
  uint64_t* pfull = sfull + 4;             // [slot][buf]
  uint64_t* oready = pfull + 4;            // [slot]
  uint64_t* qfull = oready + 2;            // [slot]
  uint64_t* ofree = qfull + 2;             // [slot]
  uint64_t* odone = ofree + 2;             // [slot]: last PV of an item completed
  uint64_t* finbar = odone + 2;            // all MMAs of the CTA done
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(finbar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(ring + C::kRingBytes + C::kBarBytes);
  const int nbw = (p.nb + 31) / 32;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  SPARK_TC_DECL
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      tc::mbar_init(&kfull[i], 1);
      tc::mbar_init(&vfull[i], 1);
      tc::mbar_init(&kempty[i], 1);
      tc::mbar_init(&vempty[i], 1);
    }
    for (int i = 0; i < 4; ++i) {
      tc::mbar_init(&sfull[i], 1);
      tc::mbar_init(&pfull[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&oready[i], 1);
      tc::mbar_init(&qfull[i], 4);
      tc::mbar_init(&ofree[i], 4);
      tc::mbar_init(&odone[i], 1);
    }
    tc::mbar_init(finbar, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 9) {
    tc::tmem_alloc(tmem_holder, C::kTmemCols);
    tc::tmem_relinquish();
  }
  if ((warp == 8 || warp == 10) && lane == 0) {
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

  if (warp == 8 || warp == 10) {
    // ================================================================ TMA producers
    // warp 8 fills the K ring, warp 10 the V ring, both in the same tile order.
    const bool is_v = warp == 10;
    uint64_t* full = is_v ? vfull : kfull;
    uint64_t* empty = is_v ? vempty : kempty;
    unsigned char* rbase = is_v ? vring : ring;
    const CUtensorMap* map_x = is_v ? &maps.v : &maps.k;
    const CUtensorMap* map_p = is_v ? &maps.vp : &maps.kp;
    // The whole warp walks the tile sequence; the selected block indices are fetched 32
    // halves at a time, one chunk ahead, so no global load sits on the issue path.
    TcSlotWalk walk[2] = {{2 * (int)blockIdx.x, stride, p.n_items},
                          {2 * (int)blockIdx.x + 1, stride, p.n_items}};
    TcItem cur[2];
    bool have[2];
    int t[2] = {0, 0};
    int ic[2] = {0, 0}, in[2] = {0, 0};  // idx of halves 32c + lane (current / next chunk)
    auto chunk = [&](int s, int c) -> int {
      const int hh = 32 * c + lane;
      return hh < cur[s].cnt ? p.idx[cur[s].row * (size_t)p.kcap + hh] : 0;
    };
    for (int s = 0; s < 2; ++s) {
      have[s] = walk[s].next_nonempty(p, &cur[s]);
      if (have[s] && !cur[s].dense) {
        ic[s] = chunk(s, 0);
        in[s] = chunk(s, 1);
      }
    }
    const int nv = p.nb * kBlock;
    const int n_dk = (p.N - nv + kBlock - 1) / kBlock;
    uint32_t q = 0;
    bool ok = true;
    while (ok && (have[0] || have[1])) {
      for (int s = 0; s < 2 && ok; ++s) {
        if (!have[s]) continue;
        const int stage = q % C::kStages;
        SPARK_TC_T0(t_ew);
        if (q >= (uint32_t)C::kStages &&
            !tc::mbar_wait(&empty[stage], ((q / C::kStages) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        SPARK_TC_ACC(4, t_ew);
        const TcItem& I = cur[s];
        int y[2], pooled[2];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          int hi = 2 * t[s] + hf;
          if (hi >= I.nhalf) hi = 2 * t[s];  // a missing second half repeats the first (masked)
          const int bsel = __shfl_sync(0xffffffffu, ic[s], hi & 31);
          pooled[hf] = 0;
          if (I.dense) {
            y[hf] = I.bh * p.N + hi * kBlock;
          } else if (hi < I.cnt) {
            y[hf] = I.bh * p.N + ((bsel >= 0 && bsel < p.nb) ? bsel : 0) * kBlock;
          } else if (hi < I.cnt + n_dk) {
            y[hf] = I.bh * p.N + nv + (hi - I.cnt) * kBlock;
          } else {
            pooled[hf] = 1;
            y[hf] = I.bh * p.nb + (hi - I.cnt - n_dk) * kBlock;
          }
        }
        if (lane == 0) {
          unsigned char* st = rbase + stage * C::kTileBytes;
          tc::mbar_expect_tx(&full[stage], C::kTileBytes);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int pn = 0; pn < C::kPanels; ++pn)
              tc::tma_load_2d(st + pn * C::kPanelBytes + hf * C::kHalfBytes,
                              pooled[hf] ? map_p : map_x, pn * 64, y[hf], &full[stage]);
        }
        __syncwarp();
        ++q;
        if (++t[s] == cur[s].ntiles) {
          t[s] = 0;
          have[s] = walk[s].next_nonempty(p, &cur[s]);
          if (have[s] && !cur[s].dense) {
            ic[s] = chunk(s, 0);
            in[s] = chunk(s, 1);
          }
        } else if ((t[s] & 15) == 0 && !cur[s].dense && 2 * t[s] < cur[s].cnt) {
          ic[s] = in[s];
          in[s] = chunk(s, (t[s] >> 4) + 1);
        }
      }
    }
    if ((!ok || *abort_flag) && lane == 0) {
      // drain every copy that may still be in flight before the CTA leaves
      const uint32_t first = q > (uint32_t)C::kStages ? q - C::kStages : 0;
      for (uint32_t j = first; j < q; ++j) mbar_drain(&full[j % C::kStages], (j / C::kStages) & 1);
    }
  } else if (warp == 9) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = tc::make_idesc_bf16(64, 128, 0, 0);
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
        int first, last;
      } pend[2] = {{0, 0, 0, 0, 0, 0}, {0, 0, 0, 0, 0, 0}};
      for (int s = 0; s < 2; ++s) have[s] = walk[s].next_nonempty(p, &cur[s]);
      const uint32_t ring_addr = tc::smem_addr(ring);
      const uint32_t vring_addr = tc::smem_addr(vring);
      bool ok = true;
      auto issue_pv = [&](int s, const Pend& pe) -> bool {
        const uint32_t b = pe.g & 1;
        SPARK_TC_T0(t_pw);
        if (!tc::mbar_wait(&pfull[2 * s + b], (pe.g >> 1) & 1, abort_flag)) return false;
        SPARK_TC_ACC(0, t_pw);
        SPARK_TC_EV(0, 30 + s);
        const int stage = pe.q % C::kStages;
        SPARK_TC_T0(t_vw);
        if (!tc::mbar_wait(&vfull[stage], (pe.q / C::kStages) & 1, abort_flag)) return false;
        SPARK_TC_ACC(1, t_vw);
        SPARK_TC_T0(t_ow);
        if (pe.first && pe.item > 0 && !tc::mbar_wait(&ofree[s], (pe.item - 1) & 1, abort_flag))
          return false;
        SPARK_TC_ACC(9, t_ow);
        SPARK_TC_T0(t_pv);
        tc::tc_fence_after();
        const uint32_t lanes = (uint32_t)(16 * s) << 16;
        const uint32_t st = vring_addr + stage * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_ts(tbase + lanes + C::kColO, tbase + lanes + C::kColS + 128 * b + kk * 8,
                     tc_vdesc<D>(st, kk), idPV, (pe.first && kk == 0) ? 0u : 1u);
        tc::mma_commit(&vempty[stage]);
        tc::mma_commit(&oready[s]);
        if (pe.last) tc::mma_commit(&odone[s]);
        SPARK_TC_EV(0, 20 + s);
        SPARK_TC_ACC(10, t_pv);
        return true;
      };
      uint32_t q = 0;
      SPARK_TC_T0(t_all);
      while (ok && (have[0] || have[1])) {
        // S of both slots first, so the tensor core has work while a softmax finishes
        Pend nxt[2] = {{0, 0, 0, 0, 0, 0}, {0, 0, 0, 0, 0, 0}};
        for (int s = 0; s < 2 && ok; ++s) {
          if (!have[s]) continue;
          SPARK_TC_T0(t_qw);
          if (t[s] == 0 && !tc::mbar_wait(&qfull[s], nitem[s] & 1, abort_flag)) {
            ok = false;
            break;
          }
          SPARK_TC_ACC(3, t_qw);
          const int stage = q % C::kStages;
          SPARK_TC_T0(t_kw);
          if (!tc::mbar_wait(&kfull[stage], (q / C::kStages) & 1, abort_flag)) {
            ok = false;
            break;
          }
          SPARK_TC_ACC(2, t_kw);
          SPARK_TC_T0(t_si);
          tc::tc_fence_after();
          const uint32_t b = g[s] & 1;
          const uint32_t lanes = (uint32_t)(16 * s) << 16;
          const uint32_t st = ring_addr + stage * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            tc::mma_ts(tbase + lanes + C::kColS + 128 * b, tbase + lanes + C::kColQ + kk * 8,
                       tc_kdesc<D>(st, kk), idS, kk > 0 ? 1u : 0u);
          tc::mma_commit(&sfull[2 * s + b]);
          tc::mma_commit(&kempty[stage]);
          SPARK_TC_EV(0, 10 + s);
          SPARK_TC_ACC(11, t_si);
          nxt[s].valid = 1;
          nxt[s].q = q;
          nxt[s].g = g[s];
          nxt[s].item = nitem[s];
          nxt[s].first = (t[s] == 0);
          nxt[s].last = (t[s] + 1 == cur[s].ntiles);
          ++q;
          ++g[s];
          if (++t[s] == cur[s].ntiles) {
            t[s] = 0;
            ++nitem[s];
            SPARK_TC_T0(t_nx);
            have[s] = walk[s].next_nonempty(p, &cur[s]);
            SPARK_TC_ACC(12, t_nx);
          }
        }
        // then the PV of each slot's previous tile; a slot that just ran out also
        // releases its last tile
        for (int s = 0; s < 2 && ok; ++s) {
          if (pend[s].valid && !issue_pv(s, pend[s])) {
            ok = false;
            break;
          }
          pend[s] = nxt[s];
          if (pend[s].valid && !have[s]) {
            if (!issue_pv(s, pend[s])) {
              ok = false;
              break;
            }
            pend[s].valid = 0;
          }
        }
      }
      for (int s = 0; s < 2 && ok; ++s)
        if (pend[s].valid && !issue_pv(s, pend[s])) ok = false;
      SPARK_TC_ACC(13, t_all);
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
    uint32_t nitem = 0;
    int cur_bad = 0;

    uint32_t ndone = 0;  // non-empty items whose epilogue ran
    auto epilogue = [&](const TcItem& I, float m_run, float l_run) -> bool {
      // odone completes once per item, after its last PV; it cannot run an item ahead
      // because the next item's PVs need this slot's P tiles.
      if (!tc::mbar_wait(&odone[s], ndone & 1, abort_flag)) return false;
      ++ndone;
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
        if (!epilogue(prev, m_prev, l_prev)) {
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
        SPARK_TC_T0(t_sw);
        if (!tc::mbar_wait(&sfull[2 * s + b], (g >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        SPARK_TC_ACC(5, t_sw);
        SPARK_TC_EV(1 + s, 40);
        tc::tc_fence_after();
        // this thread's 64 keys: half h of the tile (columns 64h .. 64h+63 of the S buffer)
        float x[64];
        SPARK_TC_T0(t_ld);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tc::tmem_ld_16x32bx2_x16<64>(tbase + lanes + C::kColS + 128 * b + 16 * c,
                                       reinterpret_cast<uint32_t*>(x) + 16 * c);
        tc::tmem_wait_ld();
        SPARK_TC_ACC(6, t_ld);
        SPARK_TC_T0(t_cp);
        // ---- logits (base 2) and masks of this half
        const int hi = 2 * t + h;
        int kind = 0, valid = kBlock, j0 = 0;
        if (hi >= I.nhalf) {
          valid = 0;
        } else if (I.dense) {
          valid = min(kBlock, p.N - hi * kBlock);
        } else if (hi < I.cnt) {
          if (bad_idx) {
            const int bb = p.idx[I.row * (size_t)p.kcap + hi];
            if (bb < 0 || bb >= p.nb) valid = 0;
          }
        } else if (hi < I.cnt + n_dk) {
          valid = min(kBlock, p.N - (nv + (hi - I.cnt) * kBlock));
        } else {
          kind = 1;
          j0 = (hi - I.cnt - n_dk) * kBlock;
          valid = min(kBlock, p.nb - j0);
        }
        // Exact halves keep raw scores (the scale is folded into the exponent's FFMA);
        // pooled halves become scale*logit + beta (base 2), with the selected blocks and
        // entries past nb masked. The half's bias values are loaded up front, unconditionally
        // (clamped index), so their latencies overlap.
        if (kind == 0) {
          if (valid < kBlock) {
#pragma unroll
            for (int j = 0; j < 64; ++j)
              if (j >= valid) x[j] = -INFINITY;
          }
        } else {
          const float* bp = p.beta + (size_t)I.bh * p.nb;
          const int wb = j0 >> 5;  // j0 is a multiple of 64
          const uint32_t w0 = bm[wb];
          const uint32_t w1 = (j0 + 32 < p.nb) ? bm[wb + 1] : 0u;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float bv[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) bv[j] = __ldg(bp + min(j0 + 16 * q + j, p.nb - 1));
            const uint32_t wm = (q < 2 ? w0 : w1) >> (16 * (q & 1));
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const bool m = (16 * q + j >= valid) || ((wm >> j) & 1u);
              x[16 * q + j] = m ? -INFINITY : fmaf(x[16 * q + j], p.scale_log2, bv[j] * kLog2e);
            }
          }
        }
        const float xs = kind == 0 ? p.scale_log2 : 1.0f;  // factor still to apply to x
        SPARK_TC_ACC(14 + kind, t_cp);
        SPARK_TC_T0(t_mx);
        // row max: 3-input max tree over this thread's 64 keys, then the partner half
        float mx;
        {
          float a0 = x[0], a1 = x[1], a2 = x[2], a3 = x[3];  // four independent chains
#pragma unroll
          for (int i = 4; i < 64; i += 8) {
            a0 = max3f(a0, x[i], x[i + 1]);
            a1 = max3f(a1, x[i + 2], x[i + 3]);
            a2 = max3f(a2, x[i + 4], x[i + 5]);
            a3 = max3f(a3, x[i + 6], x[i + 7]);
          }
          mx = max3f(max3f(a0, a1, a2), a3, a3) * xs;
        }
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
        SPARK_TC_ACC(16, t_mx);
        SPARK_TC_T0(t_ex);
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        uint32_t pk[32];
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float p0 = ex2f(fmaf(x[2 * j], xs, -m_use));
          const float p1 = ex2f(fmaf(x[2 * j + 1], xs, -m_use));
          ls[j & 3] += p0 + p1;
          pk[j] = pack_bf16x2(p0, p1);
        }
        l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        SPARK_TC_ACC(17, t_ex);
        SPARK_TC_ACC(7, t_cp);
        SPARK_TC_T0(t_st);
        // P over S: packed columns 32h .. 32h+31 of the buffer
        tc::tmem_st_16x32bx2_x16<32>(tbase + lanes + C::kColS + 128 * b, pk);
        tc::tmem_st_16x32bx2_x16<32>(tbase + lanes + C::kColS + 128 * b + 16, pk + 16);
        tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&pfull[2 * s + b]);
        SPARK_TC_ACC(8, t_st);
        SPARK_TC_EV(1 + s, 41);
      }
      if (!ok) break;
      have_prev = 1;
      prev = I;
      m_prev = m_run;
      l_prev = l_run;
      ++nitem;
    }
  }

  SPARK_TC_FLUSH
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 9) tc::tmem_dealloc(tbase, C::kTmemCols);
}

}  // namespace spark
