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
// * The unit of work is one 64-query block (an item): video blocks select their own key
//   blocks, so two query blocks cannot share an MMA B operand. tcgen05.mma with M = 64
//   runs at half the M = 128 rate, and every key of a 64-query block costs >= 1 KB of
//   shared-memory traffic (TMA writes K and V, the tensor core reads them), so the kernel
//   keeps everything else out of that path: Q and P live in tensor memory (A operand of
//   "TS" MMAs), shared memory carries the K/V rings.
// * Each persistent CTA runs two independent query blocks ("slots") whose M = 64
//   accumulators share TMEM columns in the two lane halves of every sub-partition
//   (slot 0: lanes 0-15, slot 1: lanes 16-31 of each 32-lane group), so the tensor core
//   works on one slot while the other slot's softmax runs.
// * Warp roles: warps 0-3 softmax of slot 0, warps 4-7 softmax of slot 1 (warp w reads
//   TMEM sub-partition w % 4), warp 8 fills the K ring and warp 10 the V ring with TMA,
//   warps 9 and 11 issue the MMAs of slot 0 and slot 1 (warp 9 owns TMEM). The tensor
//   pipe queues little more than one MMA, so an issuer's barrier checks between MMA
//   blocks leave it idle; with one issuer per slot the other slot's MMAs fill that gap.
//   K stages are released when their S MMAs complete and V stages when their PV MMAs
//   complete.
// * A tile is 128 keys made of two 64-key halves (a selected block, 64 dense rows or 64
//   pooled entries each; per video query block the halves run selected blocks, dense key
//   rows, then pooled entries). Per tile: S = Q K^T (8 MMAs 64x128x16 from TMEM Q and a
//   128B-swizzled K tile), softmax in base 2 (each thread owns one half of one row) with a
//   lazy running max (O is rescaled only when the row max grows by more than 2^8), P
//   written back over S as bf16, then O += P V (8 MMAs 64xDx16, V as an MN-major operand).
// * Item transitions: Q is double-buffered in TMEM, so a slot's softmax warps store the
//   next item's Q (and build its selection bitmap) right after the current item's last
//   tile, while the other slot keeps the tensor pipe busy; the epilogue releases O as soon
//   as it has read it. A pooled half's biases are warmed into L1 before its S wait.
// * Every mbarrier wait is bounded; a timeout records SPARK_ETIMEOUT, raises the CTA abort
//   flag, the TMA roles drain their copies in flight and TMEM is released.
#pragma once
#include "spark_common.cuh"
#include "tc_util.cuh"

namespace spark {

struct TcMaps {
  CUtensorMap k, v, kp, vp;  // K, V over [B*H*N, D]; pooled pack over [B*H*nb, D]
  CUtensorMap kx, vx;        // extra-token rows over [B*H*ep, D] (the extra pack)
};

struct TcParams {
  const uint16_t* Q;
  const int32_t* idx;
  const int32_t* cnt;
  const float* bias;  // pooled bias * log2(e), [B*H, nbp] (-inf past nb); pooled only
  const int32_t* perm;
  uint16_t* O;
  float* lse;
  int N, nb, nbp, kcap, BH, n_dq, pooled, n_items;
  int nt;  // video query tiles per head (the 128-query route; nb for 64-query tiles)
  float scale_log2;
  int* item_ctr;  // per-launch counter of items handed out (zeroed before the launch)
  long long wait_clocks;  // limit of every pipeline wait (the drains keep the default)
  const int32_t* xidx;    // extra tokens [B*H, ep] (video rows, -1 past n_extra); extra only
  int n_xh, n_extra, ep;  // extra halves per video item, extra tokens per head, padded rows
};

// Items handed out at run time: the claiming warp takes the next item index from the
// launch's counter and publishes it in a ring of shared-memory entries; every other role
// of the CTA reads the same entries in the same order. Longer items (the dense ones come
// first) and rows of varying length (tau) then spread over the CTAs as they free up.
constexpr int kQueueLen = 16;
struct TcQueue {
  int* ids;         // [kQueueLen] item index, -1 after the last item
  uint64_t* full;   // [kQueueLen] arrival: the claimer wrote the entry
  uint64_t* empty;  // [kQueueLen] arrivals: every reader took the entry
  // The claiming warp (all lanes): entry j gets the next item index (or -1).
  __device__ __forceinline__ bool claim(uint32_t j, const TcParams& p, volatile int* abort_flag, int* id) {
    const int e = j % kQueueLen;
    const bool ok = j < (uint32_t)kQueueLen || tc::mbar_wait(&empty[e], ((j / kQueueLen) - 1) & 1, abort_flag, p.wait_clocks);
    if (!__all_sync(0xffffffffu, ok)) return false;
    int v = 0;
    if ((threadIdx.x & 31) == 0) {
      v = atomicAdd(p.item_ctr, 1);
      if (v >= p.n_items) v = -1;
      ids[e] = v;
      tc::mbar_arrive(&full[e]);
    }
    *id = __shfl_sync(0xffffffffu, v, 0);
    return true;
  }
  // A reading warp (all lanes) or a single reading thread (one_thread): entry j.
  __device__ __forceinline__ bool read(uint32_t j, volatile int* abort_flag, int* id, bool one_thread,
                                       long long limit) {
    const int e = j % kQueueLen;
    bool ok = tc::mbar_wait(&full[e], (j / kQueueLen) & 1, abort_flag, limit);
    if (!one_thread) ok = __all_sync(0xffffffffu, ok);
    if (!ok) return false;
    *id = ids[e];
    if (one_thread) {
      tc::mbar_arrive(&empty[e]);
    } else {
      __syncwarp();
      if ((threadIdx.x & 31) == 0) tc::mbar_arrive(&empty[e]);
    }
    return true;
  }
};

template <int D>
struct TcCfg {
  // A tile is 128 keys: two 64-key halves (each a selected block, 64 dense rows or 64
  // pooled entries), so S = Q K^T is one N = 128 MMA per K step.
  // Three 32 KB stages per ring (202 KB of shared memory with the bitmaps): each K/V tile
  // takes about 1.7 us from L2 under load, so the copies in flight set the delivery rate.
  static constexpr int kStages = D == 128 ? 3 : 4;
  static constexpr int kPanels = D / 64;           // 128-byte swizzle panels per row
  static constexpr int kHalfBytes = 64 * 128;      // 64 rows x 128 B (one TMA box)
  static constexpr int kPanelBytes = 128 * 128;    // 128 rows x 128 B
  static constexpr int kTileBytes = 128 * D * 2;   // K (or V) of one 128-key tile
  static constexpr int kColS = 0;                  // S/P buffers at 0 and 128
  static constexpr int kColO = 256;
  static constexpr int kColQ = 256 + D;            // Q buffers at kColQ and kColQ + D/2
  static constexpr int kTmemCols = 512;
  static constexpr int kThreads = 384;
  static constexpr int kRingBytes = 2 * kStages * kTileBytes;  // K ring, then V ring
  static constexpr int kBarBytes = 1024;
  static constexpr int kQPieces = D / 64;          // 16-word pieces of a thread's half Q row
};

// Words of one selection bitmap (even, so a 64-entry pooled half never reads past it).
__host__ __device__ inline int tc_bitmap_words(int nb) { return ((nb + 31) / 32 + 1) & ~1; }

template <int D>
__host__ __device__ inline size_t tc_smem_bytes(int nb) {
  using C = TcCfg<D>;
  return 1024 /*alignment slack*/ + C::kRingBytes + C::kBarBytes +
         (size_t)8 * 2 * tc_bitmap_words(nb) * 4;  // two bitmaps per softmax warp
}

struct TcItem {
  int bh, q0, nq, dense, cnt, nhalf, ntiles;  // nhalf 64-key halves, ntiles = ceil(nhalf / 2)
  size_t row;                                  // selection row (video items)
};

// Item `it`, head-major: each head's dense items (64 dense query rows each, the longest
// items) and then its video query blocks (nb), so that the CTAs at work at any moment share
// one or two heads' K/V in L2.
__device__ __forceinline__ TcItem tc_item(const TcParams& p, int it) {
  TcItem r;
  const int nv = p.nb * kBlock;
  const int n_dk = (p.N - nv + kBlock - 1) / kBlock;
  const int per_h = p.n_dq + p.nb;
  const int hb = it / per_h, jj = it - hb * per_h;
  if (jj < p.n_dq) {
    r.bh = hb;
    r.dense = 1;
    r.q0 = nv + jj * kBlock;
    r.cnt = 0;
    r.row = 0;
    r.nhalf = (p.N + kBlock - 1) / kBlock;
  } else {
    const int v = jj - p.n_dq;
    r.bh = hb;
    r.dense = 0;
    r.q0 = v * kBlock;
    r.row = (size_t)r.bh * p.nb + v;
    int c = p.cnt[r.row];
    c = c < 0 ? 0 : (c > p.kcap ? p.kcap : c);
    r.cnt = c;
    r.nhalf = c + n_dk + p.n_xh + (p.pooled ? p.nbp / kBlock : 0);
  }
  r.ntiles = (r.nhalf + 1) / 2;
  r.nq = min(kBlock, p.N - r.q0);
  return r;
}

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

__device__ __forceinline__ void prefetch_l1(const void* ptr) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(ptr));
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

// The 64-key half kinds of a tile. A video item runs its halves in the order: selected
// blocks, dense key rows, extra tokens, pooled entries.
enum : int { kHalfExact = 0, kHalfDense = 1, kHalfPooled = 2, kHalfMissing = 3, kHalfExtra = 4 };

// Kind of half `hi` of item I (video or dense).
__device__ __forceinline__ int tc_half_kind(const TcItem& I, int hi, int n_dk, int n_xh) {
  if (hi >= I.nhalf) return kHalfMissing;
  if (I.dense) return kHalfDense;
  if (hi < I.cnt) return kHalfExact;
  if (hi < I.cnt + n_dk) return kHalfDense;
  if (hi < I.cnt + n_dk + n_xh) return kHalfExtra;
  return kHalfPooled;
}

// Keep-mask (bit e set: entry e attended) of the extra-token half starting at entry e0:
// entries past the head's count and tokens whose block the item selected (attended there)
// are dropped. One 16-byte load at a time, so that the few registers it needs do not
// compete with the thread's 64 scores.
__device__ __forceinline__ uint64_t tc_extra_keep(const int32_t* xs, int e0, int n_extra, const uint32_t* bm) {
  uint64_t keep = 0;
#pragma unroll 1
  for (int q4 = 0; q4 < 16; ++q4) {
    const int4 t4 = __ldg(reinterpret_cast<const int4*>(xs + e0) + q4);
    const int tt[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = 4 * q4 + i;
      const int tok = tt[i];
      bool on = e0 + e < n_extra && tok >= 0;
      if (on) {
        const int blk = tok >> 6;
        on = !((bm[blk >> 5] >> (blk & 31)) & 1u);
      }
      keep |= (uint64_t)(on ? 1u : 0u) << e;
    }
  }
  return keep;
}

// kExtra: the extra-token half kind is compiled in only when a launch has extra tokens
// (launches without them run code without it: it changes how the rest is compiled, and
// the 128-query kernel's results then varied from run to run within the tolerance).
template <int D, bool kExtra>
__global__ void __launch_bounds__(384, 1)
    attn_tc_kernel(const __grid_constant__ TcMaps maps, const TcParams p) {
  const int n_xh = kExtra ? p.n_xh : 0;
  using C = TcCfg<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ring = smem;
  unsigned char* vring = ring + C::kStages * C::kTileBytes;
  // [slot][stage]: the stage holds this slot's tile. The two slots' tiles alternate over the
  // shared stages and an issuer waits only for its own tiles, so with one barrier per stage
  // its parity wait could be satisfied by the phase of its own previous tile while the other
  // slot's tile in between is still in flight (copies need not land in issue order); with a
  // barrier per slot every phase of a barrier is waited for by its one consumer.
  uint64_t* kfull = reinterpret_cast<uint64_t*>(ring + C::kRingBytes);
  uint64_t* vfull = kfull + 2 * C::kStages;
  uint64_t* kempty = vfull + 2 * C::kStages;  // K stage free: its S MMAs completed
  uint64_t* vempty = kempty + C::kStages;  // V stage free: its PV MMAs completed
  uint64_t* sfull = vempty + C::kStages;   // [slot][S buffer]
  uint64_t* pfull = sfull + 4;             // [slot][S buffer]
  uint64_t* oready = pfull + 4;            // [slot]: a PV completed
  uint64_t* qfull = oready + 2;            // [slot][Q buffer]
  uint64_t* ofree = qfull + 4;             // [slot]: the epilogue has read O
  uint64_t* odone = ofree + 2;             // [slot]: last PV of an item completed
  uint64_t* finbar = odone + 2;            // [slot]: all MMAs of that slot's issuer done
  TcQueue queue[2];                        // [slot]: items handed out at run time (warp 8 claims)
  queue[0].full = finbar + 2;
  queue[0].empty = queue[0].full + kQueueLen;
  queue[1].full = queue[0].empty + kQueueLen;
  queue[1].empty = queue[1].full + kQueueLen;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(queue[1].empty + kQueueLen);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  queue[0].ids = const_cast<int*>(abort_flag) + 1;
  queue[1].ids = queue[0].ids + kQueueLen;
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(ring + C::kRingBytes + C::kBarBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  static_assert((6 * C::kStages + 20 + 4 * kQueueLen) * 8 + 8 + 2 * kQueueLen * 4 <= C::kBarBytes,
                "barriers, queues and flags exceed their shared-memory region");
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * C::kStages; ++i) {
      tc::mbar_init(&kfull[i], 1);
      tc::mbar_init(&vfull[i], 1);
    }
    for (int i = 0; i < C::kStages; ++i) {
      tc::mbar_init(&kempty[i], 1);
      tc::mbar_init(&vempty[i], 1);
    }
    for (int i = 0; i < 4; ++i) {
      tc::mbar_init(&sfull[i], 1);
      tc::mbar_init(&pfull[i], 4);
      tc::mbar_init(&qfull[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&oready[i], 1);
      tc::mbar_init(&ofree[i], 4);
      tc::mbar_init(&odone[i], 1);
    }
    tc::mbar_init(&finbar[0], 1);
    tc::mbar_init(&finbar[1], 1);
    for (int q = 0; q < 2; ++q)
      for (int i = 0; i < kQueueLen; ++i) {
        tc::mbar_init(&queue[q].full[i], 1);
        tc::mbar_init(&queue[q].empty[i], 7);  // V producer, two issuers, the slot's 4 softmax warps
      }
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
    tc::tma_prefetch_desc(&maps.kx);
    tc::tma_prefetch_desc(&maps.vx);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  const int nv = p.nb * kBlock;
  const int n_dk = (p.N - nv + kBlock - 1) / kBlock;

  // Registers: launched at 168 per thread (384 threads). The producer / issuer warpgroup
  // (warps 8-11) gives back down to 104 so the two softmax warpgroups (about 186 needed)
  // can grow to 200: 128 x 104 + 256 x 200 = 64,512 = 384 x 168.
  if (warp >= 8) {
  tc::regs_dec<104>();
  if (warp == 8 || warp == 10) {
    // ================================================================ TMA producers
    // warp 8 fills the K ring, warp 10 the V ring, both in the same tile order: per round,
    // one tile of slot 0 then one of slot 1 (a slot without items is skipped).
    const bool is_v = warp == 10;
    uint64_t* full = is_v ? vfull : kfull;
    uint64_t* empty = is_v ? vempty : kempty;
    unsigned char* rbase = is_v ? vring : ring;
    const CUtensorMap* map_x = is_v ? &maps.v : &maps.k;
    const CUtensorMap* map_p = is_v ? &maps.vp : &maps.kp;
    const CUtensorMap* map_e = is_v ? &maps.vx : &maps.kx;
    // The whole warp walks the tile sequence (warp 8 claims each slot's items, warp 10
    // reads them from the slot's queue); the selected block indices are fetched 32 halves
    // at a time, one chunk ahead, so no global load sits on the issue path.
    uint32_t qj[2] = {0, 0};
    bool ok = true;
    auto take_nonempty = [&](int s, TcItem* I) -> bool {
      while (true) {
        int id;
        if (!(is_v ? queue[s].read(qj[s], abort_flag, &id, false, p.wait_clocks) : queue[s].claim(qj[s], p, abort_flag, &id))) {
          ok = false;
          return false;
        }
        ++qj[s];
        if (id < 0) return false;
        *I = tc_item(p, id);
        if (I->ntiles > 0) return true;
      }
    };
    // warp 8 keeps one non-empty item per slot claimed ahead of the one it loads, so that
    // every reader finds a slot's next item published when it starts an item
    TcItem ahead_item[2] = {};
    bool have_ahead[2] = {false, false};
    auto next_nonempty = [&](int s, TcItem* I) -> bool {
      if (is_v) return take_nonempty(s, I);
      bool have_now;
      if (qj[s] == 0) {
        have_now = take_nonempty(s, I);
      } else {
        have_now = have_ahead[s];
        *I = ahead_item[s];
      }
      have_ahead[s] = have_now && take_nonempty(s, &ahead_item[s]);
      return have_now && ok;
    };
    TcItem cur[2];
    bool have[2];
    int t[2] = {0, 0};
    int ic[2] = {0, 0}, in[2] = {0, 0};  // idx of halves 32c + lane (current / next chunk)
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      have[s] = next_nonempty(s, &cur[s]);
      if (have[s] && !cur[s].dense) {
        const int h0 = lane, h1 = 32 + lane;
        ic[s] = h0 < cur[s].cnt ? p.idx[cur[s].row * (size_t)p.kcap + h0] : 0;
        in[s] = h1 < cur[s].cnt ? p.idx[cur[s].row * (size_t)p.kcap + h1] : 0;
      }
    }
    uint32_t q = 0;
    // per (slot, stage) barrier, bit slot * kStages + stage: a copy was issued on it; the
    // parity of the number of copies issued on it
    uint32_t fused = 0, fpar = 0;
    while (ok && (have[0] || have[1])) {
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        if (ok && have[s]) {
          const int stage = q % C::kStages;
          if (q >= (uint32_t)C::kStages &&
              !tc::mbar_wait(&empty[stage], ((q / C::kStages) - 1) & 1, abort_flag, p.wait_clocks)) {
            ok = false;
          } else {
            const TcItem& I = cur[s];
            int y[2], src[2];  // src: 0 K/V, 1 pooled pack, 2 extra pack
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              int hi = 2 * t[s] + hf;
              if (hi >= I.nhalf) hi = 2 * t[s];  // a missing second half repeats the first (masked)
              const int bsel = __shfl_sync(0xffffffffu, ic[s], hi & 31);
              src[hf] = 0;
              if (I.dense) {
                y[hf] = I.bh * p.N + hi * kBlock;
              } else if (hi < I.cnt) {
                y[hf] = I.bh * p.N + ((bsel >= 0 && bsel < p.nb) ? bsel : 0) * kBlock;
              } else if (hi < I.cnt + n_dk) {
                y[hf] = I.bh * p.N + nv + (hi - I.cnt) * kBlock;
              } else if (hi < I.cnt + n_dk + n_xh) {
                src[hf] = 2;
                y[hf] = I.bh * p.ep + (hi - I.cnt - n_dk) * kBlock;
              } else {
                // pooled entries past nb read rows of the next head (or TMA zero fill);
                // their bias is -inf, so they carry no weight
                src[hf] = 1;
                y[hf] = I.bh * p.nb + (hi - I.cnt - n_dk - n_xh) * kBlock;
              }
            }
            // one box per lane (lanes 0 .. 2 kPanels - 1): TMA issue throughput is per
            // issuing lane and warp, so spreading a tile's boxes over lanes raises the
            // delivery rate (measured on this SM: 22 B/clk with one lane, 31 with four)
            unsigned char* st = rbase + stage * C::kTileBytes;
            uint64_t* fb = &full[s * C::kStages + stage];
            if (lane == 0) tc::mbar_expect_tx(fb, C::kTileBytes);
            __syncwarp();
            if (lane < 2 * C::kPanels) {
              const int hf = lane / C::kPanels, pn = lane % C::kPanels;
              const int sk = hf ? src[1] : src[0];
              tc::tma_load_2d(st + pn * C::kPanelBytes + hf * C::kHalfBytes,
                              sk == 1 ? map_p : (sk == 2 ? map_e : map_x), pn * 64, hf ? y[1] : y[0], fb);
            }
            __syncwarp();
            fused |= 1u << (s * C::kStages + stage);
            fpar ^= 1u << (s * C::kStages + stage);
            ++q;
            if (++t[s] == cur[s].ntiles) {
              t[s] = 0;
              have[s] = next_nonempty(s, &cur[s]);
              if (have[s] && !cur[s].dense) {
                const int h0 = lane, h1 = 32 + lane;
                ic[s] = h0 < cur[s].cnt ? p.idx[cur[s].row * (size_t)p.kcap + h0] : 0;
                in[s] = h1 < cur[s].cnt ? p.idx[cur[s].row * (size_t)p.kcap + h1] : 0;
              }
            } else if ((t[s] & 15) == 0 && !cur[s].dense && 2 * t[s] < cur[s].cnt) {
              const int hn = 32 * ((t[s] >> 4) + 1) + lane;
              ic[s] = in[s];
              in[s] = hn < cur[s].cnt ? p.idx[cur[s].row * (size_t)p.kcap + hn] : 0;
            }
          }
        }
      }
    }
    if ((!ok || *abort_flag) && lane == 0) {
      // drain every copy that may still be in flight before the CTA leaves: the latest
      // phase of each (slot, stage) barrier (a stage is reused only after its earlier copy
      // was consumed)
      for (int i = 0; i < 2 * C::kStages; ++i)
        if ((fused >> i) & 1u) mbar_drain(&full[i], ((fpar >> i) & 1u) ^ 1u);
    }
  } else if (warp == 9 || warp == 11) {
    // ================================================================ MMA issuers
    // One issuing thread per slot (warp 9: slot 0, warp 11: slot 1): per tile, S of the
    // slot's next tile then PV of its previous one. Two issuers keep the tensor pipe fed
    // while either waits on a barrier. Both replay the producers' round-robin tile order
    // to find the ring stage of each of their tiles.
    if (lane == 0) {
      const int s = warp == 9 ? 0 : 1;
      constexpr uint32_t idS = tc::make_idesc_bf16(64, 128, 0, 0);
      constexpr uint32_t idPV = tc::make_idesc_bf16(64, D, 0, 1);
      const uint32_t lanes = (uint32_t)(16 * s) << 16;
      uint32_t qj[2] = {0, 0};
      bool ok = true;
      auto next_nonempty = [&](int o, TcItem* I) -> bool {
        while (true) {
          int id;
          if (!queue[o].read(qj[o], abort_flag, &id, true, p.wait_clocks)) {
            ok = false;
            return false;
          }
          ++qj[o];
          if (id < 0) return false;
          *I = tc_item(p, id);
          if (I->ntiles > 0) return true;
        }
      };
      TcItem cur[2];
      bool have[2];
      int t[2] = {0, 0};
#pragma unroll
      for (int o = 0; o < 2; ++o) have[o] = next_nonempty(o, &cur[o]);
      uint32_t g = 0;      // tiles of this slot issued (all items)
      uint32_t nitem = 0;  // non-empty items of this slot started
      bool pend = false;   // PV of the previous tile still to issue
      uint32_t pq = 0, pg = 0, pitem = 0;
      bool pfirst = false, plast = false;
      const uint32_t ring_addr = tc::smem_addr(ring);
      const uint32_t vring_addr = tc::smem_addr(vring);
      // parity of this slot's tiles on each stage so far (bit = stage), K and V rings
      uint32_t kpar = 0, vpar = 0;
      auto issue_pv = [&]() -> bool {
        const uint32_t b = pg & 1;
        if (!tc::mbar_wait(&pfull[2 * s + b], (pg >> 1) & 1, abort_flag, p.wait_clocks)) return false;
        const int stage = pq % C::kStages;
        const uint32_t vp = (vpar >> stage) & 1u;
        vpar ^= 1u << stage;
        if (!tc::mbar_wait(&vfull[s * C::kStages + stage], vp, abort_flag, p.wait_clocks)) return false;
        if (pfirst && pitem > 0 && !tc::mbar_wait(&ofree[s], (pitem - 1) & 1, abort_flag, p.wait_clocks)) return false;
        tc::tc_fence_after();
        const uint32_t st = vring_addr + stage * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_ts(tbase + lanes + C::kColO, tbase + lanes + C::kColS + 128 * b + kk * 8,
                     tc_vdesc<D>(st, kk), idPV, (pfirst && kk == 0) ? 0u : 1u);
        tc::mma_commit(&vempty[stage]);
        tc::mma_commit(&oready[s]);
        if (plast) tc::mma_commit(&odone[s]);
        return true;
      };
      uint32_t q = 0;  // ring position of the producers' next tile
      while (ok && (have[0] || have[1])) {
#pragma unroll
        for (int o = 0; o < 2; ++o) {
          if (ok && have[o]) {
            if (o == s) {
              const uint32_t qb = nitem & 1;
              bool good = t[o] != 0 || tc::mbar_wait(&qfull[2 * s + qb], (nitem >> 1) & 1, abort_flag, p.wait_clocks);
              const int stage = q % C::kStages;
              const uint32_t kp = (kpar >> stage) & 1u;
              kpar ^= 1u << stage;
              good = good && tc::mbar_wait(&kfull[s * C::kStages + stage], kp, abort_flag, p.wait_clocks);
              if (!good) {
                ok = false;
              } else {
                tc::tc_fence_after();
                const uint32_t b = g & 1;
                const uint32_t st = ring_addr + stage * C::kTileBytes;
                const uint32_t qcol = C::kColQ + qb * (D / 2);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                  tc::mma_ts(tbase + lanes + C::kColS + 128 * b, tbase + lanes + qcol + kk * 8,
                             tc_kdesc<D>(st, kk), idS, kk > 0 ? 1u : 0u);
                tc::mma_commit(&sfull[2 * s + b]);
                tc::mma_commit(&kempty[stage]);
                // then the PV of the previous tile of this slot
                if (pend) ok = issue_pv();
                pend = true;
                pq = q;
                pg = g;
                pitem = nitem;
                pfirst = (t[o] == 0);
                plast = (t[o] + 1 == cur[o].ntiles);
                ++g;
                if (t[o] + 1 == cur[o].ntiles) ++nitem;
              }
            }
            if (ok) {
              ++q;
              if (++t[o] == cur[o].ntiles) {
                t[o] = 0;
                have[o] = next_nonempty(o, &cur[o]);
                // this slot is done: its last PV goes out now, since the V stage it holds is
                // needed by the other slot's tiles (this issuer keeps reading the other
                // slot's items only to stay in step with the queue)
                if (o == s && !have[o] && ok && pend) {
                  ok = issue_pv();
                  pend = false;
                }
              }
            }
          }
        }
      }
      if (ok && pend) ok = issue_pv();
      // every MMA of this issuer must be complete before TMEM is released
      tc::mma_commit(&finbar[s]);
      mbar_drain(&finbar[s], 0);
    }
  }
  } else {
    tc::regs_inc<200>();
    // ================================================================ softmax (slot s)
    const int s = warp >> 2;
    const int w = warp & 3;
    const int r = 16 * w + (lane & 15);  // query row within the block
    const int h = lane >> 4;             // key half (scores) / d half (O, Q)
    const int lh = lane & 15;
    const uint32_t lanes = (uint32_t)(32 * w + 16 * s) << 16;
    const int nbwp = tc_bitmap_words(p.nb);
    uint32_t* bm2 = bitmap + warp * 2 * nbwp;  // this warp's two selection bitmaps
    bool ok = true;

    // ---- preparation of an item: the thread's Q half row into a TMEM Q buffer (then
    //      qfull), and the warp's selection bitmap from the item's index row. Runs at the
    //      end of the previous item; the other slot's MMAs keep the tensor pipe busy.
    int bad_next = 0;  // the prepared item has a block index out of range
    auto prepare = [&](const TcItem& J, int qb) {
      {
        const bool rv = r < J.nq;
        const uint16_t* qrow = p.Q + ((size_t)J.bh * p.N + J.q0 + (rv ? r : 0)) * D + h * (D / 2);
        uint32_t qv[D / 4];
#pragma unroll
        for (int i = 0; i < D / 16; ++i) {
          const uint4 a = rv ? ldg_nc_v4(qrow + 8 * i) : make_uint4(0, 0, 0, 0);
          qv[4 * i] = a.x;
          qv[4 * i + 1] = a.y;
          qv[4 * i + 2] = a.z;
          qv[4 * i + 3] = a.w;
        }
#pragma unroll
        for (int c = 0; c < C::kQPieces; ++c)
          tc::tmem_st_16x32bx2_x16_sync<D / 4>(tbase + lanes + C::kColQ + qb * (D / 2) + 16 * c, qv + 16 * c);
        tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&qfull[2 * s + qb]);
      }
      if (!J.dense && (p.pooled || J.cnt > 0 || n_xh > 0)) {
        uint32_t* bm = bm2 + qb * nbwp;
        for (int i = lane; i < nbwp; i += 32) bm[i] = 0u;
        __syncwarp();
        if (lane == 0 && w == 0 && p.cnt[J.row] != J.cnt) set_error(SPARK_EDEVICE_INDEX);
        const int32_t* ip = p.idx + J.row * (size_t)p.kcap;
        int bad = 0;
        for (int j0 = 0; j0 < J.cnt; j0 += 128) {
          int bv[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int j = j0 + 32 * i + lane;
            bv[i] = j < J.cnt ? ip[j] : 0;
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int j = j0 + 32 * i + lane;
            if (j < J.cnt) {
              if (bv[i] >= 0 && bv[i] < p.nb) atomicOr(&bm[bv[i] >> 5], 1u << (bv[i] & 31));
              else bad = 1;
            }
          }
        }
        if (__any_sync(0xffffffffu, bad)) {
          bad_next = 1;
          if (lane == 0) set_error(SPARK_EDEVICE_INDEX);
        }
        __syncwarp();
      }
    };

    uint32_t ndone = 0;  // non-empty items whose epilogue ran
    auto epilogue = [&](const TcItem& I, float m_run, float l_run) -> bool {
      // odone completes once per item, after its last PV; it cannot run an item ahead
      // because the next item's PVs need this slot's P tiles.
      if (!tc::mbar_wait_warp(&odone[s], ndone & 1, abort_flag, p.wait_clocks)) return false;
      ++ndone;
      tc::tc_fence_after();
      uint32_t o[D / 2];
      if constexpr (D == 128)
        tc::tmem_ld_16x32bx2_x64_sync<64>(tbase + lanes + C::kColO, o);
      else
        tc::tmem_ld_16x32bx2_x32_sync<32>(tbase + lanes + C::kColO, o);
      // O is in registers: the next item's first PV may overwrite it
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&ofree[s]);
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
      if (write) {
        uint16_t* dst = p.O + ((size_t)I.bh * p.N + orow) * D + h * (D / 2);
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[8 * c]) * inv, __uint_as_float(o[8 * c + 1]) * inv);
          v.y = pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv);
          v.z = pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv);
          v.w = pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv);
          *reinterpret_cast<uint4*>(dst + 8 * c) = v;
        }
        if (h == 0 && p.lse != nullptr)
          p.lse[(size_t)I.bh * p.N + orow] = l_tot > 0.f ? (m_run + __log2f(l_tot)) * kLn2 : -INFINITY;
      }
      return true;
    };

    // Items of this slot in the queue's order; an item with nothing to attend to gets
    // O = 0, LSE = -inf.
    uint32_t qj = 0;
    auto next_item = [&](TcItem* I) -> bool {
      while (true) {
        int id;
        if (!queue[s].read(qj, abort_flag, &id, false, p.wait_clocks)) {
          ok = false;
          return false;
        }
        ++qj;
        if (id < 0) return false;
        *I = tc_item(p, id);
        if (I->ntiles > 0) return true;
        if (r < I->nq) {
          int orow = I->q0 + r;
          bool wr = true;
          if (!I->dense && p.perm != nullptr) {
            orow = p.perm[(size_t)I->bh * nv + I->q0 + r];
            wr = orow >= 0 && orow < nv;
          }
          if (wr) {
            const uint4 z = make_uint4(0, 0, 0, 0);
            uint16_t* dst = p.O + ((size_t)I->bh * p.N + orow) * D + h * (D / 2);
#pragma unroll
            for (int c = 0; c < D / 16; ++c) *reinterpret_cast<uint4*>(dst + 8 * c) = z;
            if (h == 0 && p.lse != nullptr) p.lse[(size_t)I->bh * p.N + orow] = -INFINITY;
          }
        }
      }
    };

    uint32_t g = 0;  // tiles processed by this slot (all items)
    uint32_t n = 0;  // non-empty items of this slot so far
    TcItem I, prev;
    prev.ntiles = 0;
    bool have_prev = false;
    float m_prev = -INFINITY, l_prev = 0.f;
    bool have = next_item(&I);
    if (have) prepare(I, 0);
    int cur_bad = bad_next;
    bad_next = 0;
    while (ok && have) {
      // the slot's next item (published before this item's first copies were issued)
      TcItem nxt;
      const bool have_nxt = next_item(&nxt);
      if (!ok) break;
      const uint32_t* bm = bm2 + (n & 1) * nbwp;

      float m_run = -INFINITY, l_run = 0.f;
      for (int t = 0; t < I.ntiles; ++t, ++g) {
        const uint32_t b = g & 1;
        // warm L1 with the biases of a pooled half (their loads follow the S wait)
        const int hi = 2 * t + h;
        const int kind = tc_half_kind(I, hi, n_dk, n_xh);
        const float* bias_src =
            p.bias + (size_t)I.bh * p.nbp + (kind == kHalfPooled ? (hi - I.cnt - n_dk - n_xh) * kBlock : 0);
        if (kind == kHalfPooled && lh < 2) prefetch_l1(bias_src + 32 * lh);
        if (!tc::mbar_wait_warp(&sfull[2 * s + b], (g >> 1) & 1, abort_flag, p.wait_clocks)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        // this thread's 64 keys: half h of the tile (columns 64h .. 64h+63 of the S buffer)
        // loaded as words, then converted: the scores are not read through a pointer of
        // another type (the compiler may reorder accesses it believes cannot alias)
        float x[64];
        {
          uint32_t xw[64];
          tc::tmem_ld_16x32bx2_x64_sync<64>(tbase + lanes + C::kColS + 128 * b, xw);
#pragma unroll
          for (int j = 0; j < 64; ++j) x[j] = __uint_as_float(xw[j]);
        }
        // ---- logits (base 2) and masks of this half
        // Exact and dense halves keep raw scores (the scale is folded into the exponent's
        // FFMA); pooled halves become scale*logit + beta*log2(e), with the selected blocks
        // masked (entries past nb carry a -inf bias).
        if (kind != kHalfPooled) {
          int valid = kBlock;
          if (kind == kHalfMissing) {
            valid = 0;
          } else if (kind == kHalfDense) {
            const int key0 = I.dense ? hi * kBlock : nv + (hi - I.cnt) * kBlock;
            valid = min(kBlock, p.N - key0);
          } else if (kind == kHalfExact && cur_bad) {
            const int bb = p.idx[I.row * (size_t)p.kcap + hi];
            if (bb < 0 || bb >= p.nb) valid = 0;
          }
          if (valid < kBlock) {
#pragma unroll
            for (int j = 0; j < 64; ++j)
              if (j >= valid) x[j] = -INFINITY;
          }
          if constexpr (kExtra) {
            if (kind == kHalfExtra) {
              const uint64_t keep = tc_extra_keep(p.xidx + (size_t)I.bh * p.ep, (hi - I.cnt - n_dk) * kBlock,
                                                  p.n_extra, bm);
#pragma unroll
              for (int j = 0; j < 64; ++j)
                if (!((keep >> j) & 1ull)) x[j] = -INFINITY;
            }
          }
        }
        if (kind == kHalfPooled) {
          const float4* bsrc = reinterpret_cast<const float4*>(bias_src);
          const int j0 = (hi - I.cnt - n_dk - n_xh) * kBlock;
          const int wb = j0 >> 5;  // j0 is a multiple of 64, wb + 1 < nbwp
          const uint32_t w0 = bm[wb], w1 = bm[wb + 1];
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            float bv[16];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float4 f = __ldg(bsrc + 4 * qq + i);
              bv[4 * i] = f.x;
              bv[4 * i + 1] = f.y;
              bv[4 * i + 2] = f.z;
              bv[4 * i + 3] = f.w;
            }
            const uint32_t wm = (qq < 2 ? w0 : w1) >> (16 * (qq & 1));
#pragma unroll
            for (int j = 0; j < 16; ++j)
              x[16 * qq + j] = ((wm >> j) & 1u) ? -INFINITY : fmaf(x[16 * qq + j], p.scale_log2, bv[j]);
          }
        }
        const float xs = kind == kHalfPooled ? 1.0f : p.scale_log2;  // factor still to apply
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
          if (!tc::mbar_wait_warp(&oready[s], (g - 1) & 1, abort_flag, p.wait_clocks)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t v[16];
            tc::tmem_ld_16x32bx2_x16_sync<D / 2>(tbase + lanes + C::kColO + 16 * c, v);
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha);
            tc::tmem_st_16x32bx2_x16_sync<D / 2>(tbase + lanes + C::kColO + 16 * c, v);
          }
        }
        if (need) {
          l_run *= alpha;
          m_run = m_new;
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
        // P over S (packed columns 32h .. 32h+31 of the buffer), 32 keys at a time
        {
          float2 l2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
          const float2 s2 = make_float2(xs, xs), m2 = make_float2(-m_use, -m_use);
#pragma unroll
          for (int hc = 0; hc < 2; ++hc) {
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int e = 32 * hc + 2 * j;
              const float2 a2 = tc::ffma2(make_float2(x[e], x[e + 1]), s2, m2);
              const float p0 = ex2f(a2.x);
              const float p1 = ex2f(a2.y);
              l2[j & 1] = tc::fadd2(l2[j & 1], make_float2(p0, p1));
              pk[j] = pack_bf16x2(p0, p1);
            }
            tc::tmem_st_16x32bx2_x16_sync<32>(tbase + lanes + C::kColS + 128 * b + 16 * hc, pk);
          }
          ls[0] = l2[0].x; ls[1] = l2[0].y; ls[2] = l2[1].x; ls[3] = l2[1].y;
        }
        l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&pfull[2 * s + b]);
        // ---- the previous item's epilogue, once this item's first P is on its way
        if (t == 0 && have_prev) {
          if (!epilogue(prev, m_prev, l_prev)) {
            ok = false;
            break;
          }
          have_prev = false;
        }
      }
      if (!ok) break;
      if (have_nxt) prepare(nxt, (n + 1) & 1);
      prev = I;
      have_prev = true;
      m_prev = m_run;
      l_prev = l_run;
      cur_bad = bad_next;
      bad_next = 0;
      I = nxt;
      have = have_nxt;
      ++n;
    }
    if (ok && have_prev) epilogue(prev, m_prev, l_prev);
  }

  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 9) tc::tmem_dealloc(tbase, C::kTmemCols);
}

}  // namespace spark
