// Block scores and selection: top-k keep ratio and the Sol-Attn per-head threshold.
//
// Method: "ComfyUI adds a core sparse-attention node and the Comfy Compiler", section
// "Block-sparse attention: one node, three backends": top-k keeps a fixed share of key
// blocks per query block; Sol-Attn keeps the blocks whose score lies tau standard
// deviations above the head's score mean.
//
// Scores S[i, j] = qbar_i . kbar_j * scale are formed in fp32 FMA (not on the tensor
// pipe: a bf16/tf32 product would move scores by ~1e-3, far beyond the 1e-4 window in
// which two blocks count as tied). A CTA holds the score rows of RT query blocks in
// shared memory as order-preserving uint32 keys; one warp per row then finds the k-th
// largest key from a warp-private 256-bin histogram of the row's values between its
// minimum and maximum and an exact ranking of the cut bin's keys (a 4-pass MSB radix select
// where that does not apply), and writes the kept indices with ballots (ties: lower index
// first) in the row's sweep order (select_sweep_start), which the attention kernels follow.
#pragma once
#include "spark_common.cuh"
#include "tc_util.cuh"

namespace spark {

constexpr int kSelThreads = 256;
constexpr int kSelJT = 64;  // score columns per staged kbar tile
constexpr int kSelKT = kSelJT + 1;  // padded row stride of the transposed tile (no bank conflicts)

// ---------------------------------------------------------------- tau: per-head moments
// acc[bh] += sum over the (r, c) entries of one 32 x 32 tile of Mq o Mk, where
// Mq = sum_i qbar_i qbar_i^T and Mk = sum_j kbar_j kbar_j^T (fp64). Summed over tiles,
// acc = tr(Mq Mk) = sum_{i,j} (qbar_i . kbar_j)^2.
template <int D>
__global__ void __launch_bounds__(256) moments_kernel(const float* __restrict__ q_pool,
                                                      const float* __restrict__ k_pool, int nq,
                                                      int nb, double* __restrict__ acc) {
  constexpr int T = 32;
  constexpr int TPD = D / T;
  const int tr = blockIdx.x / TPD, tc = blockIdx.x % TPD;
  const size_t bh = blockIdx.y;
  __shared__ float qa[T][T + 1], qb[T][T + 1], ka[T][T + 1], kb[T][T + 1];
  __shared__ double red[8];
  const int tid = threadIdx.x;
  const int r = tid / 8, c0 = (tid % 8) * 4;  // each thread: row r, columns c0..c0+3
  double mq[4] = {0, 0, 0, 0}, mk[4] = {0, 0, 0, 0};
  const float* qp = q_pool + bh * (size_t)nq * D;
  const float* kp = k_pool + bh * (size_t)nb * D;
  const int nmax = nq > nb ? nq : nb;
  for (int b0 = 0; b0 < nmax; b0 += T) {
    // stage 32 rows x 32 columns of each operand (rows tr*T.., cols tc*T..)
    for (int e = tid; e < T * T; e += 256) {
      const int bb = e / T, cc = e % T;
      const bool okq = b0 + bb < nq, okk = b0 + bb < nb;
      const size_t o = (size_t)(b0 + bb) * D;
      qa[bb][cc] = okq ? qp[o + tr * T + cc] : 0.f;
      qb[bb][cc] = okq ? qp[o + tc * T + cc] : 0.f;
      ka[bb][cc] = okk ? kp[o + tr * T + cc] : 0.f;
      kb[bb][cc] = okk ? kp[o + tc * T + cc] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int bb = 0; bb < T; ++bb) {
      const double xq = qa[bb][r], xk = ka[bb][r];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        mq[u] = fma(xq, (double)qb[bb][c0 + u], mq[u]);
        mk[u] = fma(xk, (double)kb[bb][c0 + u], mk[u]);
      }
    }
    __syncthreads();
  }
  double part = 0.0;
#pragma unroll
  for (int u = 0; u < 4; ++u) part = fma(mq[u], mk[u], part);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
  if ((tid & 31) == 0) red[tid >> 5] = part;
  __syncthreads();
  if (tid == 0) {
    double t = 0.0;
    for (int w = 0; w < 8; ++w) t += red[w];
    atomicAdd(acc + bh, t);
  }
}

// thr[bh] = mu + tau * sigma with mu = scale * (sum qbar) . (sum kbar) / (nq nb) and
// sigma^2 = scale^2 * tr(Mq Mk) / (nq nb) - mu^2 (population moments of all nq x nb
// scores; nq query rows: blocks, or tiles of the 128-query route).
template <int D>
__global__ void __launch_bounds__(D) tau_threshold_kernel(const float* __restrict__ q_pool,
                                                          const float* __restrict__ k_pool, int nq,
                                                          int nb, const double* __restrict__ acc,
                                                          double scale, double tau,
                                                          double* __restrict__ thr) {
  __shared__ double red[D / 32];
  const size_t bh = blockIdx.x;
  const int c = threadIdx.x;
  const float* qp = q_pool + bh * (size_t)nq * D;
  const float* kp = k_pool + bh * (size_t)nb * D;
  double sq = 0.0, sk = 0.0;
  for (int b = 0; b < nq; ++b) sq += qp[(size_t)b * D + c];
  for (int b = 0; b < nb; ++b) sk += kp[(size_t)b * D + c];
  double p = sq * sk;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
  if ((c & 31) == 0) red[c >> 5] = p;
  __syncthreads();
  if (c == 0) {
    double dot = 0.0;
    for (int w = 0; w < D / 32; ++w) dot += red[w];
    const double n2 = (double)nq * (double)nb;
    const double mu = scale * dot / n2;
    const double es2 = scale * scale * acc[bh] / n2;
    const double var = es2 - mu * mu;
    thr[bh] = mu + tau * sqrt(var > 0.0 ? var : 0.0);
  }
}

// ---------------------------------------------------------------- scores + selection
struct SelectParams {
  const float* q_pool;
  const float* k_pool;
  int32_t* idx;
  int32_t* cnt;
  const double* thr;  // [B*H] (tau mode)
  int nq, nb, kcap, k, mode, rt;  // nq score rows (query blocks or tiles), nb key blocks
  int sweep;  // query tiles the attention kernel runs at once (0: plain ascending rows)
  float scale;
};

// Start of row i's sweep order: the kept blocks of a row are written ascending from the
// first one at or above this position, then wrapping around to the ones below it. The
// attention kernels visit a row's blocks in the order written, and they run the query
// tiles of a head in ascending order, `sweep` at a time: as the start position advances
// by nb / sweep per row, the tiles at work at any moment read K/V near one position of
// the head, which then stays in L2 for all of them. Multiple of 32 (one warp chunk).
__host__ __device__ inline int select_sweep_start(int i, int nb, int sweep) {
  if (sweep <= 0) return 0;
  return (int)(((long long)(i % sweep) * nb) / sweep) & ~31;
}

// The bin of the 256-bin histogram h in which the count from the top reaches kk (1 <= kk
// <= the histogram's total), the count in the bins above it and the bin's own count; every
// lane gets all three. Lane l scans bins 255 - 8l .. 248 - 8l.
__device__ __forceinline__ void top_bin(const uint32_t* h, int kk, int lane, int* bin_out,
                                        int* above_out, uint32_t* count_out) {
  uint32_t cntb[8];
  uint32_t tot = 0;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    cntb[t] = h[255 - 8 * lane - t];
    tot += cntb[t];
  }
  uint32_t incl = tot;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  const uint32_t excl = incl - tot;
  const bool mine = excl < (uint32_t)kk && (uint32_t)kk <= incl;
  const uint32_t who = __ballot_sync(0xffffffffu, mine);
  const int src = __ffs(who) - 1;
  int bin = 0, above = 0;
  uint32_t c = 0;
  if (lane == src) {
    uint32_t run = excl;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      if (run + cntb[t] >= (uint32_t)kk) {
        bin = 255 - 8 * lane - t;
        above = (int)run;
        c = cntb[t];
        break;
      }
      run += cntb[t];
    }
  }
  *bin_out = __shfl_sync(0xffffffffu, bin, src);
  *above_out = __shfl_sync(0xffffffffu, above, src);
  *count_out = __shfl_sync(0xffffffffu, c, src);
}

// The top-k cut of the row kr[0 .. nb): its k-th largest key T and the number of keys
// equal to T that the top k keep (k minus the keys above T), by a 4-pass MSB radix select
// over the warp's 256-bin histogram h.
__device__ __forceinline__ void radix_cut(const uint32_t* kr, int nb, int k, uint32_t* h, int lane,
                                          uint32_t* T_out, int* take_out) {
  uint32_t prefix = 0, mask = 0;
  int kk = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int b = lane; b < 256; b += 32) h[b] = 0;
    __syncwarp();
    for (int j = lane; j < nb; j += 32) {
      const uint32_t key = kr[j];
      if ((key & mask) == prefix) atomicAdd(&h[(key >> shift) & 255u], 1u);
    }
    __syncwarp();
    int bin, above;
    uint32_t c;
    top_bin(h, kk, lane, &bin, &above, &c);
    kk -= above;
    prefix |= (uint32_t)bin << shift;
    mask |= 255u << shift;
    __syncwarp();
  }
  *T_out = prefix;
  *take_out = kk;
}

// The same cut from value bins, in one histogram pass instead of four: the row's scores are
// binned over [min, max] into 256 equal-width bins, bin(v) = min(floor((v - min) * 256 /
// (max - min)), 255) in fp32 with every operation rounded to nearest, which never
// decreases as the key grows, so every key in a bin above the cut bin lies above T. The
// cut bin's keys (a dozen or two on Gaussian-like rows; the radix select's first pass, on
// the sign and exponent bits, puts most of a row into two or three bins and serialises
// the warp's atomics) are gathered into h and ranked exactly. Returns false, with no
// result, when the row's range is not finite and positive or the cut bin holds more than
// 256 keys (many equal scores); the caller then runs radix_cut.
__device__ __forceinline__ bool binned_cut(const uint32_t* kr, int nb, int k, uint32_t* h, int lane,
                                           uint32_t* T_out, int* take_out) {
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int j = lane; j < nb; j += 32) {
    const uint32_t key = kr[j];
    kmin = min(kmin, key);
    kmax = max(kmax, key);
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  const float vmin = key_to_float(kmin), vmax = key_to_float(kmax);
  const float range = __fsub_rn(vmax, vmin);
  const float inv = __fdiv_rn(256.f, range);
  if (!(isfinite(vmin) && isfinite(vmax) && range > 0.f && isfinite(range) && isfinite(inv)))
    return false;
  auto bin_of = [&](uint32_t key) -> int {
    const float t = __fmul_rn(__fsub_rn(key_to_float(key), vmin), inv);  // in [0, 256]
    return min((int)t, 255);
  };
  for (int b = lane; b < 256; b += 32) h[b] = 0;
  __syncwarp();
  for (int j = lane; j < nb; j += 32) atomicAdd(&h[bin_of(kr[j])], 1u);
  __syncwarp();
  int bin, above;
  uint32_t cst;
  top_bin(h, k, lane, &bin, &above, &cst);
  __syncwarp();  // every lane has read h
  if (cst > 256u) return false;
  // the cut bin's keys to h[0 .. cst), in row order
  int base = 0;
  for (int j0 = 0; j0 < nb; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < nb ? kr[j] : 0u;
    const bool in = j < nb && bin_of(key) == bin;
    const uint32_t m = __ballot_sync(0xffffffffu, in);
    const int pos = base + __popc(m & lanemask_lt());
    if (in && pos < 256) h[pos] = key;
    base += __popc(m);
  }
  __syncwarp();
  // the candidate x with #(candidates > x) < kk <= #(candidates >= x) is T
  const int kk = k - above;  // 1 <= kk <= cst
  bool found = false;
  uint32_t T = 0;
  int take = 0;
  for (int i0 = 0; i0 < (int)cst; i0 += 32) {
    const int i = i0 + lane;
    uint32_t x = 0;
    int g = 0, e = 0;
    if (i < (int)cst) {
      x = h[i];
      for (int t = 0; t < (int)cst; ++t) {
        const uint32_t y = h[t];
        g += y > x ? 1 : 0;
        e += y >= x ? 1 : 0;
      }
    }
    const uint32_t hm = __ballot_sync(0xffffffffu, i < (int)cst && g < kk && kk <= e);
    if (hm) {
      const int src = __ffs(hm) - 1;
      T = __shfl_sync(0xffffffffu, x, src);
      take = kk - __shfl_sync(0xffffffffu, g, src);
      found = true;
      break;
    }
  }
  __syncwarp();  // h is read before the caller reuses it
  if (!found) return false;
  *T_out = T;
  *take_out = take;
  return true;
}

// One warp selects the kept blocks of one score row kr[0 .. nb) (order-preserving keys):
// top-k by the cut of binned_cut (radix_cut where that declines), or the head's tau
// threshold; writes the indices of the kept blocks to row orow of idx in the row's sweep
// order (select_sweep_start; at most kcap, the first ones in that order) and their count
// to cnt[orow]. Ties at the top-k cut go to the lower block indices whatever the order they
// are written in.
__device__ __forceinline__ void select_row_warp(const SelectParams& p, const uint32_t* kr,
                                                size_t bh, size_t orow, uint32_t* h, int lane) {
  const int nb = p.nb;
  int32_t* out = p.idx + orow * (size_t)p.kcap;
  uint32_t T = 0;
  int take_eq = 0;  // number of elements equal to T to keep (lowest indices first)
  const bool use_thr = (p.mode == SPARK_SELECT_TAU);
  const double thr = use_thr ? p.thr[bh] : 0.0;
  if (!use_thr) {
    if (!binned_cut(kr, nb, p.k, h, lane, &T, &take_eq)) radix_cut(kr, nb, p.k, h, lane, &T, &take_eq);
  }
  // ---- output pass in sweep order: chunks of 32 blocks from the start position to the
  // end of the row, then from 0. Ties are ranked by block index: the first segment starts
  // with the ties below the start position counted.
  const int i_row = (int)(orow - bh * (size_t)p.nq);
  const int start = select_sweep_start(i_row, nb, p.sweep);
  const int nch = (nb + 31) / 32;
  int eq_seen = 0;
  if (!use_thr) {
    for (int j0 = 0; j0 < start; j0 += 32) {
      const int j = j0 + lane;
      eq_seen += __popc(__ballot_sync(0xffffffffu, j < nb && kr[j] == T));
    }
  }
  int written = 0;
  for (int c = 0; c < nch; ++c) {
    int j0 = start + 32 * c;
    if (j0 >= 32 * nch) j0 -= 32 * nch;
    if (j0 == 0) eq_seen = 0;  // wrapped (or no rotation): ties ranked from the row start
    const int j = j0 + lane;
    bool keep = false;
    if (use_thr) {
      keep = j < nb && (double)key_to_float(kr[j]) > thr;
    } else {
      const uint32_t key = j < nb ? kr[j] : 0u;
      const bool eq = j < nb && key == T;
      const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
      const int rank = eq_seen + __popc(eqm & lanemask_lt());
      eq_seen += __popc(eqm);
      keep = j < nb && (key > T || (eq && rank < take_eq));
    }
    const uint32_t km = __ballot_sync(0xffffffffu, keep);
    const int pos = written + __popc(km & lanemask_lt());
    if (keep && pos < p.kcap) out[pos] = j;
    written += __popc(km);
  }
  if (lane == 0) {
    if (written > p.kcap) set_error(SPARK_ECAPACITY);
    p.cnt[orow] = min(written, p.kcap);
  }
}

// Dynamic shared memory: keys[rt][nbp] | qs[rt][D] | kt[D][kSelKT] | hist[8][256].
template <int D>
__global__ void __launch_bounds__(kSelThreads) score_select_kernel(SelectParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int RT = p.rt, nb = p.nb;
  const int nbp = (nb + 3) & ~3;
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem);
  float* qs = reinterpret_cast<float*>(keys + (size_t)RT * nbp);
  float* kt = qs + RT * D;
  uint32_t* hist = reinterpret_cast<uint32_t*>(kt + D * kSelKT);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t bh = blockIdx.y;
  const int row0 = blockIdx.x * RT;
  const int nrows = min(RT, p.nq - row0);
  const float* qp = p.q_pool + bh * (size_t)p.nq * D;
  const float* kp = p.k_pool + bh * (size_t)nb * D;

  for (int e = tid; e < RT * D; e += kSelThreads) {
    const int r = e / D;
    qs[e] = r < nrows ? qp[(size_t)(row0 + r) * D + (e % D)] : 0.f;
  }
  // ---- scores: thread -> column j = tid % 64 of the tile, rows rg, rg + 4, ...
  const int jj = tid % kSelJT, rg = tid / kSelJT;  // rg in [0, 4)
  for (int j0 = 0; j0 < nb; j0 += kSelJT) {
    __syncthreads();  // kt reuse
    for (int e = tid; e < kSelJT * D; e += kSelThreads) {
      const int j = e / D, c = e % D;  // coalesced read of kbar rows, transposed store
      kt[c * kSelKT + j] = (j0 + j < nb) ? kp[(size_t)(j0 + j) * D + c] : 0.f;
    }
    __syncthreads();
    const int j = j0 + jj;
    for (int r = rg; r < RT; r += 4) {
      float acc0 = 0.f, acc1 = 0.f;
      const float* qr = qs + r * D;
#pragma unroll 8
      for (int c = 0; c < D; c += 2) {
        acc0 = fmaf(qr[c], kt[c * kSelKT + jj], acc0);
        acc1 = fmaf(qr[c + 1], kt[(c + 1) * kSelKT + jj], acc1);
      }
      if (j < nb && r < nrows) keys[(size_t)r * nbp + j] = float_to_key((acc0 + acc1) * p.scale);
    }
  }
  __syncthreads();

  // ---- selection: warp w handles rows w, w + 8, ...
  uint32_t* h = hist + warp * 256;
  for (int r = warp; r < nrows; r += kSelThreads / 32)
    select_row_warp(p, keys + (size_t)r * nbp, bh, bh * (size_t)p.nq + row0 + r, h, lane);
}

// ---------------------------------------------------------------- scores, tiled
// Score tile of 64 query blocks x 128 key blocks of one head, written as order-preserving
// keys to skeys[bh][i][j] (row stride nbp). fp32 FMA with register tiling: each thread
// owns 4 rows x 8 columns; the d dimension is staged 32 at a time, transposed, so a
// thread reads its 4 q values and 8 k values of one d with three 16-byte loads. Every
// score sums its even and its odd d terms in two chains, in increasing d, as the fused
// kernel does.
constexpr int kScI = 64, kScJ = 128, kScDC = 32;

template <int D>
__global__ void __launch_bounds__(256) score_tile_kernel(const float* __restrict__ q_pool,
                                                         const float* __restrict__ k_pool, int nq,
                                                         int nb, int nbp, float scale,
                                                         uint32_t* __restrict__ skeys) {
  __shared__ __align__(16) float qs[kScDC][kScI];
  __shared__ __align__(16) float ks[kScDC][kScJ];
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  const size_t bh = blockIdx.z;
  const int i0 = blockIdx.y * kScI, j0 = blockIdx.x * kScJ;
  const float* qp = q_pool + bh * (size_t)nq * D;
  const float* kp = k_pool + bh * (size_t)nb * D;
  // accumulators in column pairs for the packed fp32 FMA (fma.rn.f32x2): each lane runs
  // exactly the fmaf chain of its own score
  float2 acc0[4][4], acc1[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int u = 0; u < 4; ++u) acc0[r][u] = acc1[r][u] = make_float2(0.f, 0.f);
  for (int d0 = 0; d0 < D; d0 += kScDC) {
    __syncthreads();
    // stage q rows i0.. (64 x 32) and k rows j0.. (128 x 32), transposed to [d][row]
    // consecutive lanes take consecutive rows, so the transposed stores hit 32 banks
    for (int e = tid; e < kScI * kScDC / 4; e += 256) {
      const int rr = e % kScI, cc = (e / kScI) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i0 + rr < nq) v = *reinterpret_cast<const float4*>(qp + (size_t)(i0 + rr) * D + d0 + cc);
      qs[cc][rr] = v.x;
      qs[cc + 1][rr] = v.y;
      qs[cc + 2][rr] = v.z;
      qs[cc + 3][rr] = v.w;
    }
    for (int e = tid; e < kScJ * kScDC / 4; e += 256) {
      const int rr = e % kScJ, cc = (e / kScJ) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + rr < nb) v = *reinterpret_cast<const float4*>(kp + (size_t)(j0 + rr) * D + d0 + cc);
      ks[cc][rr] = v.x;
      ks[cc + 1][rr] = v.y;
      ks[cc + 2][rr] = v.z;
      ks[cc + 3][rr] = v.w;
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < kScDC; c += 2) {
      const float4 qa = *reinterpret_cast<const float4*>(&qs[c][4 * ty]);
      const float4 qb = *reinterpret_cast<const float4*>(&qs[c + 1][4 * ty]);
      const float4 ka0 = *reinterpret_cast<const float4*>(&ks[c][4 * tx]);
      const float4 ka1 = *reinterpret_cast<const float4*>(&ks[c][64 + 4 * tx]);
      const float4 kb0 = *reinterpret_cast<const float4*>(&ks[c + 1][4 * tx]);
      const float4 kb1 = *reinterpret_cast<const float4*>(&ks[c + 1][64 + 4 * tx]);
      const float q0[4] = {qa.x, qa.y, qa.z, qa.w}, q1[4] = {qb.x, qb.y, qb.z, qb.w};
      const float2 k0[4] = {make_float2(ka0.x, ka0.y), make_float2(ka0.z, ka0.w),
                            make_float2(ka1.x, ka1.y), make_float2(ka1.z, ka1.w)};
      const float2 k1[4] = {make_float2(kb0.x, kb0.y), make_float2(kb0.z, kb0.w),
                            make_float2(kb1.x, kb1.y), make_float2(kb1.z, kb1.w)};
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          acc0[r][u] = tc::ffma2(make_float2(q0[r], q0[r]), k0[u], acc0[r][u]);
          acc1[r][u] = tc::ffma2(make_float2(q1[r], q1[r]), k1[u], acc1[r][u]);
        }
    }
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = i0 + 4 * ty + r;
    if (i >= nq) continue;
    uint32_t* dst = skeys + (bh * (size_t)nq + i) * nbp;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int j = j0 + 64 * half + 4 * tx;
      uint32_t kv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 a0 = acc0[r][2 * half + (e >> 1)], a1 = acc1[r][2 * half + (e >> 1)];
        kv[e] = float_to_key(((e & 1) ? a0.y + a1.y : a0.x + a1.x) * scale);
      }
      if (j + 3 < nbp) {
        *reinterpret_cast<uint4*>(dst + j) = make_uint4(kv[0], kv[1], kv[2], kv[3]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (j + e < nbp) dst[j + e] = kv[e];
      }
    }
  }
}

// Selection from materialised score rows: warp w of a CTA takes row 8 * blockIdx.x + w of
// head blockIdx.y, copies it to shared memory and selects (select_row_warp).
__global__ void __launch_bounds__(256) select_rows_kernel(SelectParams p,
                                                          const uint32_t* __restrict__ skeys,
                                                          int nbp) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* rows = reinterpret_cast<uint32_t*>(smem);
  uint32_t* hist = rows + 8 * (size_t)nbp;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t bh = blockIdx.y;
  const int i = blockIdx.x * 8 + warp;
  if (i >= p.nq) return;
  uint32_t* kr = rows + (size_t)warp * nbp;
  const uint4* src = reinterpret_cast<const uint4*>(skeys + (bh * (size_t)p.nq + i) * nbp);
  for (int e = lane; e < nbp / 4; e += 32) reinterpret_cast<uint4*>(kr)[e] = src[e];
  __syncwarp();
  select_row_warp(p, kr, bh, bh * (size_t)p.nq + i, hist + warp * 256, lane);
}

}  // namespace spark
