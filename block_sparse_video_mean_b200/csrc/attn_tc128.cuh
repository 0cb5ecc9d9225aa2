// Exact + compressed block-sparse attention forward on the 128-query x 64-key route.
//
// Method: as attn_tc.cuh ("Spark-H3: speeding up MiniMax-H3 in ComfyUI with block-sparse
// attention", section "What Spark-Attn changes"), with the route geometry of the "H3
// Optimizations" README, section "Manual Sparse Sage recovery": a query tile of 128 rows
// (two consecutive video blocks, or 128 dense rows) shares one selection of 64-key
// blocks, so the whole tile is one A operand and every tensor-core MMA has M = 128 (the
// full-rate shape; M = 64 runs at half rate). Each K/V byte brought into shared memory
// now serves 128 queries instead of 64.
//
// Design (sm_100a), one persistent CTA per SM, one query tile at a time:
// * TMEM (512 columns): S/P double buffer (2 x 128 columns), O (D columns), Q double
//   buffer (2 x D/2 columns, bf16 pairs: the A operand of the S MMAs). Row r of the tile
//   is TMEM lane r.
// * Warp roles: warps 0-7 softmax (warp w owns rows 32 (w % 4) + 16 (w / 4) .. + 15 of its
//   lane quadrant; lanes 0-15 take keys 0-63 of those rows and lanes 16-31 keys 64-127,
//   through the 16-lane x 2 TMEM access shape), warp 8 fills the K ring, warp 10 the V
//   ring (TMA), warp 9 issues the S MMAs (and owns TMEM), warp 11 the PV MMAs. With two
//   issuers the tensor pipe gets S(t + 1) while PV(t) waits for its P.
// * Per tile of 128 keys: S = Q K^T (D/16 MMAs 128x128x16, Q from TMEM); each softmax
//   thread takes 64 keys of one row and the two halves of a row meet in one warp shuffle;
//   the running max is lazy (O is rescaled only when it grows by more than 2^8), so the
//   exponentials are taken against the running max first, with the row max alongside, and
//   redone (from the logits, still in registers) only on the rare tiles that raise it; the
//   softmax warps are bound by their instruction stream, so scale, subtract and row sums
//   use packed fp32 pairs; P is written as bf16 over the thread's own S columns (64h ..
//   64h + 31); O += P V (8 MMAs 128xDx16, the A columns of each key half taken from where
//   that half's P lives).
// * Every mbarrier wait is bounded; a timeout records SPARK_ETIMEOUT, raises the CTA abort
//   flag, the TMA roles drain their copies in flight and TMEM is released.
#pragma once
#include "attn_tc.cuh"

namespace spark {

template <int D>
struct Tc128Cfg {
  static constexpr int kStages = 2;
  static constexpr int kPanels = D / 64;
  static constexpr int kHalfBytes = 64 * 128;
  static constexpr int kTileBytes = 128 * D * 2;  // K (or V) of one 128-key tile
  static constexpr int kColS = 0;                 // S/P buffers at 0 and 128
  static constexpr int kColO = 256;
  static constexpr int kColQ = 256 + D;           // Q buffers at kColQ and kColQ + D/2
  static constexpr int kTmemCols = 512;
  static constexpr int kThreads = 384;
  static constexpr int kRingBytes = 2 * kStages * kTileBytes;
  static constexpr int kBarBytes = 1024;
};

template <int D>
__host__ __device__ inline size_t tc128_smem_bytes(int nb) {
  using C = Tc128Cfg<D>;
  return 1024 /*alignment slack*/ + C::kRingBytes + C::kBarBytes +
         (size_t)8 * 2 * tc_bitmap_words(nb) * 4;  // two bitmaps per softmax warp
}

// Item `it`, head-major: each head's dense items (128 dense query rows each, the longest
// items) and then its video query tiles (nt), so that the CTAs at work at any moment share
// one or two heads' K/V in L2.
__device__ __forceinline__ TcItem tc128_item(const TcParams& p, int it) {
  TcItem r;
  const int nv = p.nb * kBlock;
  const int n_dk = (p.N - nv + kBlock - 1) / kBlock;
  const int per_h = p.n_dq + p.nt;
  const int hb = it / per_h, jj = it - hb * per_h;
  if (jj < p.n_dq) {
    r.bh = hb;
    r.dense = 1;
    r.q0 = nv + jj * 128;
    r.cnt = 0;
    r.row = 0;
    r.nhalf = (p.N + kBlock - 1) / kBlock;
    r.nq = min(128, p.N - r.q0);
  } else {
    const int v = jj - p.n_dq;
    r.bh = hb;
    r.dense = 0;
    r.q0 = v * 128;
    r.row = (size_t)r.bh * p.nt + v;
    int c = p.cnt[r.row];
    c = c < 0 ? 0 : (c > p.kcap ? p.kcap : c);
    r.cnt = c;
    r.nhalf = c + n_dk + p.n_xh + (p.pooled ? p.nbp / kBlock : 0);
    r.nq = min(128, nv - r.q0);
  }
  r.ntiles = (r.nhalf + 1) / 2;
  return r;
}

// kExtra: the extra-token half kind is compiled in only when a launch has extra tokens
// (launches without them run code without it: it changes how the rest is compiled, and
// the 128-query kernel's results then varied from run to run within the tolerance).
template <int D, bool kExtra>
__global__ void __launch_bounds__(384, 1)
    attn_tc128_kernel(const __grid_constant__ TcMaps maps, const TcParams p) {
  const int n_xh = kExtra ? p.n_xh : 0;
  using C = Tc128Cfg<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ring = smem;
  unsigned char* vring = ring + C::kStages * C::kTileBytes;
  uint64_t* kfull = reinterpret_cast<uint64_t*>(ring + C::kRingBytes);
  uint64_t* vfull = kfull + C::kStages;
  uint64_t* kempty = vfull + C::kStages;  // K stage free: its S MMAs completed
  uint64_t* vempty = kempty + C::kStages; // V stage free: its PV MMAs completed
  uint64_t* sfull = vempty + C::kStages;  // [S buffer]: S of a tile is in TMEM
  uint64_t* pfull = sfull + 2;            // [S buffer]: the 8 softmax warps wrote P
  uint64_t* sfree = pfull + 2;            // [S buffer]: the PV MMAs reading P completed
  uint64_t* oready = sfree + 2;           // a PV completed
  uint64_t* qfull = oready + 1;           // [Q buffer]: the 8 softmax warps wrote Q
  uint64_t* ofree = qfull + 2;            // the epilogue has read O
  uint64_t* odone = ofree + 1;            // last PV of an item completed
  uint64_t* finbar = odone + 1;           // [issuer]: all its MMAs completed
  TcQueue queue;                          // items handed out at run time (warp 8 claims)
  queue.full = finbar + 2;
  queue.empty = queue.full + kQueueLen;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(queue.empty + kQueueLen);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  queue.ids = const_cast<int*>(abort_flag) + 1;
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(ring + C::kRingBytes + C::kBarBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      tc::mbar_init(&kfull[i], 1);
      tc::mbar_init(&vfull[i], 1);
      tc::mbar_init(&kempty[i], 1);
      tc::mbar_init(&vempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&sfull[i], 1);
      tc::mbar_init(&pfull[i], 8);
      tc::mbar_init(&sfree[i], 1);
      tc::mbar_init(&qfull[i], 8);
      tc::mbar_init(&finbar[i], 1);
    }
    tc::mbar_init(oready, 1);
    tc::mbar_init(ofree, 8);
    tc::mbar_init(odone, 1);
    for (int i = 0; i < kQueueLen; ++i) {
      tc::mbar_init(&queue.full[i], 1);
      tc::mbar_init(&queue.empty[i], 11);  // V producer, two issuers, 8 softmax warps
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

  // Registers: launched at 168 per thread (384 threads); the producer / issuer warpgroup
  // gives back down to 104 so the softmax warpgroups can grow to 200:
  // 128 x 104 + 256 x 200 = 64,512 = 384 x 168.
  if (warp >= 8) {
  tc::regs_dec<104>();
  if (warp == 8 || warp == 10) {
    // ================================================================ TMA producers
    const bool is_v = warp == 10;
    uint64_t* full = is_v ? vfull : kfull;
    uint64_t* empty = is_v ? vempty : kempty;
    unsigned char* rbase = is_v ? vring : ring;
    const CUtensorMap* map_x = is_v ? &maps.v : &maps.k;
    const CUtensorMap* map_p = is_v ? &maps.vp : &maps.kp;
    const CUtensorMap* map_e = is_v ? &maps.vx : &maps.kx;
    // The whole warp walks the tile sequence (warp 8 claims the items, warp 10 reads
    // them from the queue); the selected block indices are fetched 32 halves at a time,
    // one chunk ahead.
    uint32_t qj = 0;
    bool ok = true;
    auto take_nonempty = [&](TcItem* I) -> bool {
      while (true) {
        int id;
        if (!(is_v ? queue.read(qj, abort_flag, &id, false, p.wait_clocks) : queue.claim(qj, p, abort_flag, &id))) {
          ok = false;
          return false;
        }
        ++qj;
        if (id < 0) return false;
        *I = tc128_item(p, id);
        if (I->ntiles > 0) return true;
      }
    };
    // warp 8 keeps one non-empty item claimed ahead of the one it loads, so that every
    // reader of the queue finds the next item already published when it starts an item
    TcItem ahead_item = {};
    bool have_ahead = false;
    auto next_nonempty = [&](TcItem* I) -> bool {
      if (is_v) return take_nonempty(I);
      bool have_now;
      if (qj == 0) {
        have_now = take_nonempty(I);
      } else {
        have_now = have_ahead;
        *I = ahead_item;
      }
      have_ahead = have_now && take_nonempty(&ahead_item);
      return have_now && ok;
    };
    TcItem cur;
    bool have = next_nonempty(&cur);
    int t = 0;
    int ic = 0, in = 0;  // idx of halves 32c + lane (current / next chunk)
    if (have && !cur.dense) {
      ic = lane < cur.cnt ? p.idx[cur.row * (size_t)p.kcap + lane] : 0;
      in = 32 + lane < cur.cnt ? p.idx[cur.row * (size_t)p.kcap + 32 + lane] : 0;
    }
    uint32_t q = 0;
    while (ok && have) {
      const int stage = q % C::kStages;
      if (q >= (uint32_t)C::kStages &&
          !tc::mbar_wait(&empty[stage], ((q / C::kStages) - 1) & 1, abort_flag, p.wait_clocks)) {
        ok = false;
        break;
      }
      int y[2], src[2];  // src: 0 K/V, 1 pooled pack, 2 extra pack
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        int hi = 2 * t + hf;
        if (hi >= cur.nhalf) hi = 2 * t;  // a missing second half repeats the first (masked)
        const int bsel = __shfl_sync(0xffffffffu, ic, hi & 31);
        src[hf] = 0;
        if (cur.dense) {
          y[hf] = cur.bh * p.N + hi * kBlock;
        } else if (hi < cur.cnt) {
          y[hf] = cur.bh * p.N + ((bsel >= 0 && bsel < p.nb) ? bsel : 0) * kBlock;
        } else if (hi < cur.cnt + n_dk) {
          y[hf] = cur.bh * p.N + nv + (hi - cur.cnt) * kBlock;
        } else if (hi < cur.cnt + n_dk + n_xh) {
          src[hf] = 2;
          y[hf] = cur.bh * p.ep + (hi - cur.cnt - n_dk) * kBlock;
        } else {
          // pooled entries past nb read rows of the next head (or TMA zero fill); their
          // bias is -inf, so they carry no weight
          src[hf] = 1;
          y[hf] = cur.bh * p.nb + (hi - cur.cnt - n_dk - n_xh) * kBlock;
        }
      }
      // one box per lane: TMA issue throughput is per issuing lane and warp
      unsigned char* st = rbase + stage * C::kTileBytes;
      if (lane == 0) tc::mbar_expect_tx(&full[stage], C::kTileBytes);
      __syncwarp();
      if (lane < 2 * C::kPanels) {
        const int hf = lane / C::kPanels, pn = lane % C::kPanels;
        const int sk = hf ? src[1] : src[0];
        tc::tma_load_2d(st + pn * TcCfg<D>::kPanelBytes + hf * C::kHalfBytes,
                        sk == 1 ? map_p : (sk == 2 ? map_e : map_x), pn * 64, hf ? y[1] : y[0], &full[stage]);
      }
      __syncwarp();
      ++q;
      if (++t == cur.ntiles) {
        t = 0;
        have = next_nonempty(&cur);
        if (have && !cur.dense) {
          ic = lane < cur.cnt ? p.idx[cur.row * (size_t)p.kcap + lane] : 0;
          in = 32 + lane < cur.cnt ? p.idx[cur.row * (size_t)p.kcap + 32 + lane] : 0;
        }
      } else if ((t & 15) == 0 && !cur.dense && 2 * t < cur.cnt) {
        const int hn = 32 * ((t >> 4) + 1) + lane;
        ic = in;
        in = hn < cur.cnt ? p.idx[cur.row * (size_t)p.kcap + hn] : 0;
      }
    }
    if ((!ok || *abort_flag) && lane == 0) {
      // drain every copy that may still be in flight before the CTA leaves
      const uint32_t first = q > (uint32_t)C::kStages ? q - C::kStages : 0;
      for (uint32_t j = first; j < q; ++j) mbar_drain(&full[j % C::kStages], (j / C::kStages) & 1);
    }
  } else if (warp == 9 || warp == 11) {
    // ================================================================ MMA issuers
    // Warp 9 issues S(g) = Q K^T of every tile g, warp 11 O += P V; both walk the item
    // sequence, and tile g uses ring stage g % kStages and S buffer g % 2.
    if (lane == 0) {
      const bool is_pv = warp == 11;
      constexpr uint32_t idS = tc::make_idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idPV = tc::make_idesc_bf16(128, D, 0, 1);
      const uint32_t ring_addr = tc::smem_addr(ring);
      const uint32_t vring_addr = tc::smem_addr(vring);
      uint32_t qj = 0;
      bool ok = true;
      auto next_nonempty = [&](TcItem* I) -> bool {
        while (true) {
          int id;
          if (!queue.read(qj, abort_flag, &id, true, p.wait_clocks)) {
            ok = false;
            return false;
          }
          ++qj;
          if (id < 0) return false;
          *I = tc128_item(p, id);
          if (I->ntiles > 0) return true;
        }
      };
      TcItem cur;
      bool have = next_nonempty(&cur);
      uint32_t g = 0, nitem = 0;
      int t = 0;
      while (ok && have) {
        const uint32_t b = g & 1;
        const int stage = g % C::kStages;
        if (!is_pv) {
          const uint32_t qb = nitem & 1;
          bool good = t != 0 || tc::mbar_wait(&qfull[qb], (nitem >> 1) & 1, abort_flag, p.wait_clocks);
          good = good && tc::mbar_wait(&kfull[stage], (g / C::kStages) & 1, abort_flag, p.wait_clocks);
          // S buffer b is free once the PV of tile g - 2 (its P) completed
          good = good && (g < 2 || tc::mbar_wait(&sfree[b], ((g >> 1) - 1) & 1, abort_flag, p.wait_clocks));
          if (!good) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t st = ring_addr + stage * C::kTileBytes;
          const uint32_t qcol = C::kColQ + qb * (D / 2);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            tc::mma_ts(tbase + C::kColS + 128 * b, tbase + qcol + kk * 8, tc_kdesc<D>(st, kk), idS,
                       kk > 0 ? 1u : 0u);
          tc::mma_commit(&sfull[b]);
          tc::mma_commit(&kempty[stage]);
        } else {
          bool good = tc::mbar_wait(&pfull[b], (g >> 1) & 1, abort_flag, p.wait_clocks);
          good = good && tc::mbar_wait(&vfull[stage], (g / C::kStages) & 1, abort_flag, p.wait_clocks);
          // the first PV of an item overwrites O: the previous item's epilogue read it
          if (good && t == 0 && nitem > 0) good = tc::mbar_wait(ofree, (nitem - 1) & 1, abort_flag, p.wait_clocks);
          if (!good) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t st = vring_addr + stage * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            // keys 16kk .. 16kk + 15: P of key half kk / 4 lives at columns 64 (kk / 4) ..
            tc::mma_ts(tbase + C::kColO, tbase + C::kColS + 128 * b + 64 * (kk >> 2) + 8 * (kk & 3),
                       tc_vdesc<D>(st, kk), idPV, (t == 0 && kk == 0) ? 0u : 1u);
          // oready first: a softmax warp waits for it only on the tiles where it rescales O,
          // which is sound while PV(g - 2)'s oready arrival precedes its sfree arrival (the
          // one that lets S(g) start)
          tc::mma_commit(oready);
          tc::mma_commit(&vempty[stage]);
          tc::mma_commit(&sfree[b]);
          if (t + 1 == cur.ntiles) tc::mma_commit(odone);
        }
        ++g;
        if (++t == cur.ntiles) {
          t = 0;
          ++nitem;
          have = next_nonempty(&cur);
        }
      }
      // every MMA of this issuer must be complete before TMEM is released
      tc::mma_commit(&finbar[is_pv ? 1 : 0]);
      mbar_drain(&finbar[is_pv ? 1 : 0], 0);
    }
  }
  } else {
    tc::regs_inc<200>();
    // ================================================================ softmax
    const int row0 = 32 * (warp & 3) + 16 * (warp >> 2);  // the warp's 16 rows (one lane quadrant)
    const int r = row0 + (lane & 15);    // query row within the tile
    const int h = lane >> 4;             // key half of a tile, column half of O and Q
    const uint32_t lanes = (uint32_t)row0 << 16;
    const int nbwp = tc_bitmap_words(p.nb);
    uint32_t* bm2 = bitmap + warp * 2 * nbwp;  // this warp's two selection bitmaps
    bool ok = true;

    // ---- preparation of an item: the thread's half Q row into a TMEM Q buffer (then
    //      qfull), and the warp's selection bitmap. Runs at the end of the previous item.
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
        for (int c = 0; c < D / 64; ++c)
          tc::tmem_st_16x32bx2_x16_sync<D / 4>(tbase + lanes + C::kColQ + qb * (D / 2) + 16 * c, qv + 16 * c);
        tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&qfull[qb]);
      }
      if (!J.dense && (p.pooled || J.cnt > 0 || n_xh > 0)) {
        uint32_t* bm = bm2 + qb * nbwp;
        for (int i = lane; i < nbwp; i += 32) bm[i] = 0u;
        __syncwarp();
        if (lane == 0 && warp == 0 && p.cnt[J.row] != J.cnt) set_error(SPARK_EDEVICE_INDEX);
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
      if (!tc::mbar_wait_warp(odone, ndone & 1, abort_flag, p.wait_clocks)) return false;
      tc::tc_fence_after();
      uint32_t o[D / 2];
      if constexpr (D == 128)
        tc::tmem_ld_16x32bx2_x64_sync<64>(tbase + lanes + C::kColO, o);
      else
        tc::tmem_ld_16x32bx2_x32_sync<32>(tbase + lanes + C::kColO, o);
      // O is in registers: the next item's first PV may overwrite it
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(ofree);
      ++ndone;
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

    // Items in the queue's order; an item with nothing to attend to gets O = 0, LSE = -inf.
    uint32_t qj = 0;
    auto next_item = [&](TcItem* I) -> bool {
      while (true) {
        int id;
        if (!queue.read(qj, abort_flag, &id, false, p.wait_clocks)) {
          ok = false;
          return false;
        }
        ++qj;
        if (id < 0) return false;
        *I = tc128_item(p, id);
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

    uint32_t g = 0;  // tiles processed (all items)
    uint32_t n = 0;  // non-empty items so far
    TcItem I, prev;
    prev.ntiles = 0;
    bool have_prev = false;
    float m_prev = -INFINITY, l_prev = 0.f;
    bool have = next_item(&I);
    if (have) prepare(I, 0);
    int cur_bad = bad_next;
    bad_next = 0;
    while (ok && have) {
      // the next item (published before this item's first copies were issued)
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
        if (kind == kHalfPooled && lane < 2) prefetch_l1(bias_src + 32 * lane);
        if (!tc::mbar_wait_warp(&sfull[b], (g >> 1) & 1, abort_flag, p.wait_clocks)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        // this thread's 64 keys: half h of the tile (columns 64h .. 64h + 63 of the buffer)
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
        } else {
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
        // exponentials against the running max first (it rarely moves), the row max
        // alongside; when a row's max grew by more than 2^8 the warp redoes them
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
        auto exps = [&](float m_use) {
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
            tc::tmem_st_16x32bx2_x16_sync<64>(tbase + lanes + C::kColS + 128 * b + 16 * hc, pk);
          }
          ls[0] = l2[0].x; ls[1] = l2[0].y; ls[2] = l2[1].x; ls[3] = l2[1].y;
        };
        exps(m_run == -INFINITY ? 0.f : m_run);
        float mx;
        {
          float a0 = x[0], a1 = x[1], a2 = x[2], a3 = x[3];
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
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2f(m_run - m_new) : 1.0f;
          if (t > 0) {
            // rescale this thread's half of its O row once the previous PV has landed
            if (!tc::mbar_wait_warp(oready, (g - 1) & 1, abort_flag, p.wait_clocks)) {
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
          tc::tmem_wait_st();
          exps(m_run == -INFINITY ? 0.f : m_run);
        }
        l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&pfull[b]);
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
