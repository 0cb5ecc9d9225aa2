// Spark-Reblock: data-dependent block layout by whitened median bisection.
//
// Method: "Spark-H3: speeding up MiniMax-H3 in ComfyUI with block-sparse attention",
// section "What Spark-Attn changes", Spark-Reblock bullet: two queries are alike when their
// attention-score patterns over the keys are alike, measured by the Mahalanobis cosine under
// the opposite side's (the keys') second moment; a hierarchical partitioner splits groups
// until every leaf holds the block size, in O(N log N), so the layout follows the input,
// layer and head. Section "Workflows": reblock_layout=q_reuse_k (keys reuse the query
// partition).
//
// Per (batch, head), level-synchronous:
//   M = mean_j k_j k_j^T (fp32 tile products, fp64 accumulation); M = L L^T (fp64 Cholesky,
//   retried with 1e-6 tr(M)/d on the diagonal, identity if that fails too);
//   x_i = L^T q_i / |L^T q_i| (fp32);
//   every node of m > 1 blocks: centred covariance of its x (fp64 accumulation), leading
//   eigenvector v (fp64 Lanczos; Householder tridiagonalisation, Sturm multisection and
//   inverse iteration when it does not converge), projections x.v signed so their third
//   central moment is >= 0, the
//   floor(m/2)*64-th smallest (projection, token) by radix select, stable partition;
//   leaves ordered by smallest token, tokens ascending; Q/K/V rows gathered.
// The tree shape depends only on nb, so the host walks it; nodes at most 64 blocks big are
// split together with their whole subtree by one CTA, larger nodes (the first few levels)
// accumulate their raw moment sums over many CTAs with fp64 atomics: the root and every
// left child over its tokens, every right child as its parent's sums minus its left
// sibling's.
#pragma once
#include <vector>

#include "spark_common.cuh"

namespace spark {
namespace rb {

constexpr int kThreads = 256;
constexpr int kSmallBlocks = 64;   // nodes up to this many blocks are split by one CTA subtree
constexpr int kChunkTok = 4096;    // tokens per CTA of the multi-CTA accumulations
constexpr int kTile = 64;          // tokens staged per covariance step

// Node (level, label) -> first block and block count, following the label bits from the
// root (bit 1 = right child). Returns false for labels no node carries at that level.
__host__ __device__ inline bool node_of(int nb, int level, int label, int* start, int* m) {
  int st = 0, mm = nb;
  for (int l = level - 1; l >= 0; --l) {
    const int bit = (label >> l) & 1;
    if (mm == 1) {
      if (bit) return false;
      continue;
    }
    const int ml = mm / 2;
    if (bit) {
      st += ml;
      mm -= ml;
    } else {
      mm = ml;
    }
  }
  *start = st;
  *m = mm;
  return true;
}

inline int num_levels(int nb) {
  int L = 0;
  while ((1 << L) < nb) ++L;
  return L;
}

// ------------------------------------------------------------------ block reductions
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
// Sum over the CTA; every thread gets the result. `red` holds kThreads/32 doubles.
__device__ __forceinline__ double block_sum_d(double v, double* red) {
  v = warp_sum_d(v);
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int i = 0; i < kThreads / 32; ++i) t += red[i];
  return t;
}

// ------------------------------------------------------------------ second moments
// Adds sum over `rows` of r r^T (and sum of r when S1 != nullptr) into fp64 accumulators
// held in shared memory (S2: D x D, S1: D). Rows are staged 64 at a time as fp32; thread
// (ti, tj) owns rows ti (D/16) .. + D/16 - 1 and columns tj + 16 b of S2, sums a tile in
// fp32, then adds it in fp64: consecutive tj touch consecutive doubles, so the fp64
// read-modify-writes are free of bank conflicts (a contiguous column block would put the
// 16 tj of a warp 8 doubles apart). Each element sums the same products in the same order
// whichever thread owns it.
// `load_row(i, dst)` writes row i (0 <= i < n) as D floats into dst.
template <int D, class LoadRow>
__device__ void accumulate_moments(int n, LoadRow load_row, float* stage, double* S2, double* S1) {
  constexpr int S = D / 16;
  constexpr int LD = D + 4;  // padded staging row
  const int tid = threadIdx.x;
  const int ti = tid / 16, tj = tid % 16;
  for (int t0 = 0; t0 < n; t0 += kTile) {
    const int nt = min(kTile, n - t0);
    __syncthreads();
    for (int r = tid / (D / 4); r < kTile; r += kThreads / (D / 4)) {
      float* dst = stage + r * LD;
      if (r < nt) {
        load_row(t0 + r, dst, tid % (D / 4));
      } else {
        reinterpret_cast<float4*>(dst)[tid % (D / 4)] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    __syncthreads();
    float acc[S][S];
#pragma unroll
    for (int a = 0; a < S; ++a)
#pragma unroll
      for (int b = 0; b < S; ++b) acc[a][b] = 0.f;
    for (int r = 0; r < kTile; ++r) {
      const float* row = stage + r * LD;
      float xa[S], xb[S];
#pragma unroll
      for (int a = 0; a < S; ++a) {
        xa[a] = row[ti * S + a];
        xb[a] = row[tj + 16 * a];
      }
#pragma unroll
      for (int a = 0; a < S; ++a)
#pragma unroll
        for (int b = 0; b < S; ++b) acc[a][b] = fmaf(xa[a], xb[b], acc[a][b]);
    }
#pragma unroll
    for (int a = 0; a < S; ++a)
#pragma unroll
      for (int b = 0; b < S; ++b) S2[(ti * S + a) * D + tj + 16 * b] += (double)acc[a][b];
    if (S1 != nullptr && tid < D) {
      float cs = 0.f;
      for (int r = 0; r < kTile; ++r) cs += stage[r * LD + tid];
      S1[tid] += (double)cs;
    }
  }
  __syncthreads();
}

// As accumulate_moments, for fp32 rows already in global memory (`row_ptr(i)`, 16-byte
// aligned, D floats): tiles are gathered with cp.async into two alternating stages, so the
// next tile's gather overlaps this tile's products. `stage` holds 2 x kTile x (D + 4) floats.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

template <int D, class RowPtr>
__device__ void accumulate_moments_rows(int n, RowPtr row_ptr, float* stage, double* S2, double* S1) {
  constexpr int S = D / 16;
  constexpr int LD = D + 4;  // padded staging row (16-byte multiple)
  constexpr int C4 = D / 4;  // 16-byte chunks per row
  const int tid = threadIdx.x;
  const int ti = tid / 16, tj = tid % 16;
  auto issue = [&](int t0, float* buf) {
    const int nt = min(kTile, n - t0);
    for (int e = tid; e < kTile * C4; e += kThreads) {
      const int r = e / C4, c4 = e % C4;
      float* dst = buf + r * LD + 4 * c4;
      if (r < nt) cp_async16(dst, row_ptr(t0 + r) + 4 * c4);
      else *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  const int ntiles = (n + kTile - 1) / kTile;
  if (ntiles > 0) issue(0, stage);
  cp_async_commit();
  for (int tt = 0; tt < ntiles; ++tt) {
    float* cur = stage + (tt & 1) * kTile * LD;
    if (tt + 1 < ntiles) issue((tt + 1) * kTile, stage + ((tt + 1) & 1) * kTile * LD);
    cp_async_commit();
    cp_async_wait1();
    __syncthreads();
    float acc[S][S];
#pragma unroll
    for (int a = 0; a < S; ++a)
#pragma unroll
      for (int b = 0; b < S; ++b) acc[a][b] = 0.f;
    for (int r = 0; r < kTile; ++r) {
      const float* row = cur + r * LD;
      float xa[S], xb[S];
#pragma unroll
      for (int a = 0; a < S; a += 4) {
        const float4 va = *reinterpret_cast<const float4*>(row + ti * S + a);
        xa[a] = va.x; xa[a + 1] = va.y; xa[a + 2] = va.z; xa[a + 3] = va.w;
      }
#pragma unroll
      for (int b = 0; b < S; ++b) xb[b] = row[tj + 16 * b];
#pragma unroll
      for (int a = 0; a < S; ++a)
#pragma unroll
        for (int b = 0; b < S; ++b) acc[a][b] = fmaf(xa[a], xb[b], acc[a][b]);
    }
#pragma unroll
    for (int a = 0; a < S; ++a)
#pragma unroll
      for (int b = 0; b < S; ++b) S2[(ti * S + a) * D + tj + 16 * b] += (double)acc[a][b];
    if (S1 != nullptr && tid < D) {
      float cs = 0.f;
      for (int r = 0; r < kTile; ++r) cs += cur[r * LD + tid];
      S1[tid] += (double)cs;
    }
    __syncthreads();  // this stage is refilled two tiles later
  }
}

// Key second moment of one head: grid (chunks, B*H); fp64 atomics into macc[bh][D][D].
template <int D>
__global__ void __launch_bounds__(kThreads) kmoment_kernel(const uint16_t* __restrict__ K, int N, int nv,
                                                           double* __restrict__ macc) {
  extern __shared__ __align__(16) unsigned char smem[];
  double* S2 = reinterpret_cast<double*>(smem);
  float* stage = reinterpret_cast<float*>(S2 + D * D);
  const size_t bh = blockIdx.y;
  const int r0 = blockIdx.x * kChunkTok;
  const int n = min(kChunkTok, nv - r0);
  if (n <= 0) return;
  for (int i = threadIdx.x; i < D * D; i += kThreads) S2[i] = 0.0;
  const uint16_t* kb = K + (bh * N + r0) * D;
  auto load = [&](int i, float* dst, int c4) {
    const uint2 u = *reinterpret_cast<const uint2*>(kb + (size_t)i * D + 4 * c4);
    dst[4 * c4 + 0] = __uint_as_float(u.x << 16);
    dst[4 * c4 + 1] = __uint_as_float(u.x & 0xffff0000u);
    dst[4 * c4 + 2] = __uint_as_float(u.y << 16);
    dst[4 * c4 + 3] = __uint_as_float(u.y & 0xffff0000u);
  };
  accumulate_moments<D>(n, load, stage, S2, nullptr);
  double* dst = macc + bh * D * D;
  for (int i = threadIdx.x; i < D * D; i += kThreads) atomicAdd(dst + i, S2[i]);
}

// In-place lower Cholesky of A (fp64, D x D in shared memory). Returns false on a
// non-positive pivot.
template <int D>
__device__ bool cholesky_inplace(double* A, int* fail) {
  const int tid = threadIdx.x;
  if (tid == 0) *fail = 0;
  __syncthreads();
  for (int j = 0; j < D; ++j) {
    if (tid == 0) {
      const double dj = A[j * D + j];
      if (!(dj > 0.0)) *fail = 1;
      A[j * D + j] = dj > 0.0 ? sqrt(dj) : 1.0;
    }
    __syncthreads();
    if (*fail) return false;
    const double piv = A[j * D + j];
    for (int i = j + 1 + tid; i < D; i += kThreads) A[i * D + j] /= piv;
    __syncthreads();
    const int m = D - j - 1;
    for (int e = tid; e < m * m; e += kThreads) {
      const int i = j + 1 + e / m, k = j + 1 + e % m;
      if (k <= i) A[i * D + k] -= A[i * D + j] * A[k * D + j];
    }
    __syncthreads();
  }
  return true;
}

// L of each head (fp32 row-major, upper triangle zero): grid B*H.
template <int D>
__global__ void __launch_bounds__(kThreads) cholesky_kernel(const double* __restrict__ macc, int nv,
                                                            float* __restrict__ lmat) {
  extern __shared__ __align__(16) unsigned char smem[];
  double* A = reinterpret_cast<double*>(smem);
  __shared__ int fail;
  __shared__ double red[kThreads / 32];
  const size_t bh = blockIdx.x;
  const double* src = macc + bh * D * D;
  const double inv_n = nv > 0 ? 1.0 / nv : 0.0;
  bool ok = false;
  for (int attempt = 0; attempt < 2 && !ok; ++attempt) {
    double tr = 0.0;
    for (int i = threadIdx.x; i < D; i += kThreads) tr += src[i * D + i] * inv_n;
    tr = block_sum_d(tr, red);
    const double jitter = attempt == 0 ? 0.0 : 1e-6 * tr / D;
    for (int e = threadIdx.x; e < D * D; e += kThreads)
      A[e] = src[e] * inv_n + ((e / D == e % D) ? jitter : 0.0);
    __syncthreads();
    ok = cholesky_inplace<D>(A, &fail);
  }
  float* L = lmat + bh * D * D;
  for (int e = threadIdx.x; e < D * D; e += kThreads) {
    const int i = e / D, k = e % D;
    L[e] = ok ? (k <= i ? (float)A[e] : 0.f) : (i == k ? 1.f : 0.f);
  }
}

// x_i = L^T q_i / |L^T q_i| for the video rows of every head; also tok[i] = i and the
// level-0 tree labels. grid (ceil(nv / kWhTok), B*H). L stays in shared memory for the
// CTA's kWhTok tokens, taken 64 at a time: thread (ty, tx) computes tokens 4 ty .. 4 ty + 3
// x columns 4 tx .. 4 tx + 3 and 64 + 4 tx .. 64 + 4 tx + 3, summing k in increasing order.
constexpr int kWhTok = 256;
template <int D>
__global__ void __launch_bounds__(kThreads)
    whiten_kernel(const uint16_t* __restrict__ Q, int N, int nv, const float* __restrict__ lmat,
                  float* __restrict__ X, int32_t* __restrict__ tok, int32_t* __restrict__ tree0,
                  size_t tree_head_stride) {
  static_assert(D == 128 || D == 64, "head dim");
  extern __shared__ __align__(16) unsigned char smem[];
  float* Ls = reinterpret_cast<float*>(smem);  // D x D
  float* qs = Ls + D * D;                      // [D][64]: the tile's queries, transposed
  constexpr int CW = D / 32;                   // columns per thread in each half
  const size_t bh = blockIdx.y;
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  const float* L = lmat + bh * D * D;
  for (int e = tid; e < D * D / 4; e += kThreads)
    reinterpret_cast<float4*>(Ls)[e] = reinterpret_cast<const float4*>(L)[e];
  for (int t0 = blockIdx.x * kWhTok; t0 < min(nv, (int)(blockIdx.x + 1) * kWhTok); t0 += 64) {
    __syncthreads();  // qs reuse (and Ls on the first pass)
    for (int e = tid; e < 64 * D / 2; e += kThreads) {
      const int r = e / (D / 2), c2 = e % (D / 2);
      const int t = t0 + r;
      uint32_t u = 0;
      if (t < nv) u = *reinterpret_cast<const uint32_t*>(Q + (bh * N + t) * D + 2 * c2);
      qs[(2 * c2) * 64 + r] = __uint_as_float(u << 16);
      qs[(2 * c2 + 1) * 64 + r] = __uint_as_float(u & 0xffff0000u);
    }
    __syncthreads();
    float acc[4][2 * CW];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 2 * CW; ++c) acc[r][c] = 0.f;
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
      const float4 q4 = *reinterpret_cast<const float4*>(qs + k * 64 + 4 * ty);
      const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
      float lv[2 * CW];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int c = 0; c < CW; c += 2) {
          const float2 l2 = *reinterpret_cast<const float2*>(Ls + k * D + hh * (D / 2) + CW * tx + c);
          lv[hh * CW + c] = l2.x;
          lv[hh * CW + c + 1] = l2.y;
        }
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 2 * CW; ++c) acc[r][c] = fmaf(qv[r], lv[c], acc[r][c]);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < 2 * CW; ++c) ss = fmaf(acc[r][c], acc[r][c], ss);
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
      const int t = t0 + 4 * ty + r;
      if (t < nv) {
        float* xr = X + (bh * nv + t) * D;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int c = 0; c < CW; c += 2)
            *reinterpret_cast<float2*>(xr + hh * (D / 2) + CW * tx + c) =
                make_float2(acc[r][hh * CW + c] * inv, acc[r][hh * CW + c + 1] * inv);
        if (tx == 0) {
          tok[bh * nv + t] = t;
          if (tree0 != nullptr) tree0[bh * tree_head_stride + t] = 0;
        }
      }
    }
  }
}

// ------------------------------------------------------------------ node covariance
// C = centred covariance (fp64, D x D) and mu = mean of the n whitened rows x[tok[i]].
template <int D>
__device__ void node_covariance(const float* __restrict__ Xh, const int32_t* __restrict__ tseg,
                                int n, float* stage, double* C, double* mu) {
  for (int i = threadIdx.x; i < D * D; i += kThreads) C[i] = 0.0;
  for (int i = threadIdx.x; i < D; i += kThreads) mu[i] = 0.0;
  auto rowp = [&](int i) { return Xh + (size_t)tseg[i] * D; };
  accumulate_moments_rows<D>(n, rowp, stage, C, mu);
  const double inv = 1.0 / n;
  for (int i = threadIdx.x; i < D; i += kThreads) mu[i] *= inv;
  __syncthreads();
  for (int e = threadIdx.x; e < D * D; e += kThreads) C[e] = C[e] * inv - mu[e / D] * mu[e % D];
  __syncthreads();
}

// ------------------------------------------------------------------ leading eigenvector
// Scratch layout (doubles): a, e, e2, beta, u, w, y, dd, du, du2, dl (D each), red (8),
// misc (8); piv (D ints) after that.
template <int D>
struct EigScratch {
  static constexpr int kDoubles = 11 * D + 16;
  static constexpr int kBytes = kDoubles * 8 + D * 4;
};

// 1/x in fp64 by two Newton-Raphson steps r <- r (2 - x r) from the fp32 reciprocal
// (relative error 2^-24 -> 2^-48 -> below fp64 rounding); magnitudes outside the fp32
// range take the plain division.
__device__ __forceinline__ double rcp_nr(double x) {
  const double ax = fabs(x);
  if (!(ax > 1e-36 && ax < 1e36)) return 1.0 / x;
  double r = (double)__frcp_rn((float)x);
  r = r * fma(-x, r, 2.0);
  r = r * fma(-x, r, 2.0);
  return r;
}

// Eigenvalues of the tridiagonal (a, e) below x, counted as sign changes of the Sturm
// sequence p_0 = 1, p_1 = a_0 - x, p_{i+1} = (a_i - x) p_i - e_{i-1}^2 p_{i-1}. The ratio
// p_{i+1} / p_i is pivot i of the LDL^T factorisation of T - xI, so this counts negative
// pivots without a division: one FMA per step on the dependency chain. A pivot below pivmin
// in magnitude becomes -pivmin, as in the division form; signs are read from the sign bits
// (a term scaled down to zero keeps its sign). Every 4 steps the pair (p_i, p_{i-1}) is
// multiplied by the exact power of two that brings the larger to [1, 2); the entries are a
// covariance of whitened rows, O(1), so 4 steps can neither overflow nor lose the pair.
__device__ __forceinline__ int sturm_count(const double* a, const double* e2, int n, double x,
                                           double pivmin) {
  constexpr double kTrueMin = 4.9406564584124654e-324;
  double pm = 1.0;      // p_{i-1}
  double p = a[0] - x;  // p_i
  if (fabs(p) < pivmin) p = -pivmin;
  int c = signbit(p) ? 1 : 0;
  for (int i = 1; i < n; ++i) {
    const double lim = fmax(pivmin * fabs(p), kTrueMin);
    double pn = fma(a[i] - x, p, -e2[i - 1] * pm);
    if (fabs(pn) < lim) pn = signbit(p) ? lim : -lim;
    c += (signbit(pn) != signbit(p)) ? 1 : 0;
    pm = p;
    p = pn;
    if ((i & 3) == 0) {
      const double m = fmax(fabs(p), fabs(pm));
      int ex = (int)((__double2hiint(m) >> 20) & 0x7ff) - 1023;
      ex = min(max(ex, -1022), 1022);
      const double s = __hiloint2double((1023 - ex) << 20, 0);  // 2^-ex
      p *= s;
      pm *= s;
    }
  }
  return c;
}

// Unit eigenvector of the largest eigenvalue of the symmetric matrix C (fp64, shared
// memory, destroyed) into v (shared). Householder tridiagonalisation T = H^T C H, the
// largest eigenvalue of T by multisection on Sturm counts, its eigenvector by inverse
// iteration (tridiagonal LU with partial pivoting), then v = H y.
template <int D>
__device__ void eigen_top(double* C, double* scr, double* v) {
  double* a = scr;
  double* e = a + D;
  double* e2 = e + D;
  double* bt = e2 + D;
  double* u = bt + D;
  double* w = u + D;
  double* y = w + D;
  double* dd = y + D;
  double* du = dd + D;
  double* du2 = du + D;
  double* dl = du2 + D;
  double* red = dl + D;
  double* misc = red + 8;
  int* piv = reinterpret_cast<int*>(misc + 8);
  const int tid = threadIdx.x;

  // ---- tridiagonalisation, with the matrix in registers: thread (ty, tx) of a 16 x 16
  //      grid holds C[ty + 16 ra][tx + 16 rb] (ra, rb < D / 16). Per step k the column
  //      below the diagonal becomes the Householder vector u (kept in column k for the
  //      back-transformation), p = beta C u is reduced across the 16 threads of a row
  //      group with shuffles, and the trailing block takes the rank-2 update
  //      C -= u w^T + w u^T with w = p - (beta/2)(u.p) u.
  {
    constexpr int R = D / 16;
    const int ty = tid >> 4, tx = tid & 15, lane = tid & 31;
    double c[R][R];
#pragma unroll
    for (int ra = 0; ra < R; ++ra)
#pragma unroll
      for (int rb = 0; rb < R; ++rb) c[ra][rb] = C[(ty + 16 * ra) * D + tx + 16 * rb];
    // k = 16 kb + kl: kb is unrolled so every register index is a compile-time constant
#pragma unroll
    for (int kb = 0; kb < R; ++kb) {
      for (int kl = 0; kl < 16; ++kl) {
        const int k = 16 * kb + kl;
        if (k >= D - 2) break;
        // u and p alternate between two buffers so that one barrier before and one
        // after the matrix-vector product suffice; every warp derives alpha, beta and
        // u.p itself (identical arithmetic, identical results)
        double* ub = (kl & 1) ? y : u;
        double* pb = (kl & 1) ? dd : w;
        // column k below the diagonal into ub (zero at and above the diagonal)
        if (tx == kl) {
#pragma unroll
          for (int ra = 0; ra < R; ++ra) {
            const int i = ty + 16 * ra;
            if (i > k) ub[i] = c[ra][kb];
          }
        }
        if (tid <= k) ub[tid] = 0.0;
        __syncthreads();
        double ss = 0.0;
        for (int i = k + 1 + lane; i < D; i += 32) ss += ub[i] * ub[i];
        ss = warp_sum_d(ss);
        const double x0 = ub[k + 1];
        const double tail = ss - x0 * x0;
        if (!(tail > 1e-300 * (ss + 1e-300))) {  // column already reduced (uniform)
          if (tid == 0) {
            bt[k] = 0.0;
            e[k] = x0;
          }
          continue;
        }
        const double alpha = -copysign(sqrt(ss), x0);
        const double u0 = x0 - alpha;
        const double beta = 2.0 / (tail + u0 * u0);
        if (tid == 0) {
          bt[k] = beta;
          e[k] = alpha;
        }
        // row and column groups below kb hold only indices <= k: the trailing block starts
        // at group kb (a compile-time constant of this unrolled iteration)
        double uj[R];
#pragma unroll
        for (int rb = kb; rb < R; ++rb) {
          const int j = tx + 16 * rb;
          uj[rb] = j == k + 1 ? u0 : ub[j];
        }
#pragma unroll
        for (int ra = kb; ra < R; ++ra) {
          double sacc = 0.0;
#pragma unroll
          for (int rb = kb; rb < R; ++rb) sacc = fma(c[ra][rb], uj[rb], sacc);
#pragma unroll
          for (int off = 8; off > 0; off >>= 1) sacc += __shfl_xor_sync(0xffffffffu, sacc, off);
          if (tx == 0) pb[ty + 16 * ra] = beta * sacc;  // p (rows at or above k are unused)
        }
        __syncthreads();
        double dt = 0.0;
        for (int i = k + 1 + lane; i < D; i += 32) dt += (i == k + 1 ? u0 : ub[i]) * pb[i];
        const double kc = 0.5 * beta * warp_sum_d(dt);
        double wj[R];
#pragma unroll
        for (int rb = kb; rb < R; ++rb) {
          const int j = tx + 16 * rb;
          wj[rb] = j > k ? pb[j] - kc * uj[rb] : 0.0;
        }
#pragma unroll
        for (int ra = kb; ra < R; ++ra) {
          const int i = ty + 16 * ra;
          const double ui = i == k + 1 ? u0 : ub[i];
          const double wi = i > k ? pb[i] - kc * ui : 0.0;
#pragma unroll
          for (int rb = kb; rb < R; ++rb) c[ra][rb] = fma(-ui, wj[rb], fma(-wi, uj[rb], c[ra][rb]));
        }
        // the Householder vector's first entry replaces C[k + 1][k] (row k + 1 lies in
        // row group kb, or kb + 1 when kl = 15)
        if (tx == kl && ty == ((k + 1) & 15)) {
          if (kl < 15) {
            c[kb][kb] = u0;
          } else if (kb + 1 < R) {
            c[(kb + 1) < R ? kb + 1 : kb][kb] = u0;
          }
        }
      }
    }
    __syncthreads();
    // stored transposed: the Householder vector of step k is then row k of C, contiguous
#pragma unroll
    for (int ra = 0; ra < R; ++ra)
#pragma unroll
      for (int rb = 0; rb < R; ++rb) C[(tx + 16 * rb) * D + ty + 16 * ra] = c[ra][rb];
    __syncthreads();
  }
  for (int i = tid; i < D; i += kThreads) a[i] = C[i * D + i];
  if (tid == 0) e[D - 2] = C[(D - 2) * D + (D - 1)];
  __syncthreads();
  for (int i = tid; i < D - 1; i += kThreads) e2[i] = e[i] * e[i];

  // ---- largest eigenvalue of T: Gershgorin interval, then multisection
  double glo = 1e300, ghi = -1e300, emax = 0.0;
  for (int i = tid; i < D; i += kThreads) {
    const double r = (i > 0 ? fabs(e[i - 1]) : 0.0) + (i < D - 1 ? fabs(e[i]) : 0.0);
    glo = fmin(glo, a[i] - r);
    ghi = fmax(ghi, a[i] + r);
    if (i < D - 1) emax = fmax(emax, e[i] * e[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    glo = fmin(glo, __shfl_xor_sync(0xffffffffu, glo, o));
    ghi = fmax(ghi, __shfl_xor_sync(0xffffffffu, ghi, o));
    emax = fmax(emax, __shfl_xor_sync(0xffffffffu, emax, o));
  }
  __syncthreads();
  if ((tid & 31) == 0) {
    red[tid >> 5] = glo;
    w[tid >> 5] = ghi;
    y[tid >> 5] = emax;
  }
  __syncthreads();
  if (tid == 0) {
    double lo = red[0], hi = w[0], em = y[0];
    for (int i = 1; i < kThreads / 32; ++i) {
      lo = fmin(lo, red[i]);
      hi = fmax(hi, w[i]);
      em = fmax(em, y[i]);
    }
    const double span = fmax(fabs(lo), fabs(hi)) + 1e-300;
    misc[0] = lo - 1e-12 * span;
    misc[1] = hi + 1e-12 * span;
    misc[2] = 2.2250738585072014e-308 * fmax(1.0, em);
  }
  __syncthreads();
  const double pivmin = misc[2];
  for (int round = 0; round < 12; ++round) {
    const double lo = misc[0], hi = misc[1];
    if (hi - lo <= 1e-11 * fmax(fabs(lo), fabs(hi))) break;  // ample for the shift below
    const double x = lo + (hi - lo) * (double)(tid + 1) / (double)(kThreads + 1);
    const int c = sturm_count(a, e2, D, x, pivmin);
    double clo = (c <= D - 1) ? x : -1e300;  // at or below the top eigenvalue
    double chi = (c == D) ? x : 1e300;       // above it
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      clo = fmax(clo, __shfl_xor_sync(0xffffffffu, clo, o));
      chi = fmin(chi, __shfl_xor_sync(0xffffffffu, chi, o));
    }
    __syncthreads();
    if ((tid & 31) == 0) {
      red[tid >> 5] = clo;
      w[tid >> 5] = chi;
    }
    __syncthreads();
    if (tid == 0) {
      double nlo = misc[0], nhi = misc[1];
      for (int i = 0; i < kThreads / 32; ++i) {
        nlo = fmax(nlo, red[i]);
        nhi = fmin(nhi, w[i]);
      }
      misc[0] = nlo;
      misc[1] = nhi;
    }
    __syncthreads();
  }
  const double theta = 0.5 * (misc[0] + misc[1]);

  // ---- eigenvector of T by inverse iteration (one thread; O(D) per solve)
  if (tid == 0) {
    const double tiny = 1e-30 * (fabs(theta) + 1e-300);
    for (int i = 0; i < D; ++i) {
      dd[i] = a[i] - theta;
      if (i < D - 1) dl[i] = du[i] = e[i];
      du2[i] = 0.0;
    }
    for (int i = 0; i < D - 1; ++i) {
      if (fabs(dd[i]) >= fabs(dl[i])) {
        if (dd[i] == 0.0) dd[i] = tiny;
        const double f = dl[i] * rcp_nr(dd[i]);
        dl[i] = f;
        dd[i + 1] -= f * du[i];
        piv[i] = 0;
      } else {
        const double f = dd[i] * rcp_nr(dl[i]);
        dd[i] = dl[i];
        dl[i] = f;
        const double tmp = du[i];
        du[i] = dd[i + 1];
        dd[i + 1] = tmp - f * dd[i + 1];
        if (i < D - 2) {
          du2[i] = du[i + 1];
          du[i + 1] = -f * du[i + 1];
        }
        piv[i] = 1;
      }
    }
    if (dd[D - 1] == 0.0) dd[D - 1] = tiny;
    for (int i = 0; i < D; ++i) dd[i] = rcp_nr(dd[i]);  // the solves multiply by 1 / pivot
    for (int i = 0; i < D; ++i) y[i] = 1.0 + 0.001 * i;
    for (int it = 0; it < 2; ++it) {  // each solve shrinks other components by (lambda1-theta)/gap
      for (int i = 0; i < D - 1; ++i) {
        if (piv[i] == 0) {
          y[i + 1] -= dl[i] * y[i];
        } else {
          const double tmp = y[i] - dl[i] * y[i + 1];
          y[i] = y[i + 1];
          y[i + 1] = tmp;
        }
      }
      y[D - 1] *= dd[D - 1];
      y[D - 2] = (y[D - 2] - du[D - 2] * y[D - 1]) * dd[D - 2];
      for (int i = D - 3; i >= 0; --i) y[i] = (y[i] - du[i] * y[i + 1] - du2[i] * y[i + 2]) * dd[i];
      double nn = 0.0;
      for (int i = 0; i < D; ++i) nn += y[i] * y[i];
      const double inv = 1.0 / sqrt(nn);
      for (int i = 0; i < D; ++i) y[i] *= inv;
    }
  }
  __syncthreads();

  // ---- back-transform v = H_0 ... H_{D-3} y (one warp; lane l keeps y[l + 32 j] in
  //      registers, the Householder vector of step k is row k of C)
  if (tid < 32) {
    constexpr int YJ = D / 32;
    double yr[YJ];
#pragma unroll
    for (int j = 0; j < YJ; ++j) yr[j] = y[tid + 32 * j];
    for (int k = D - 3; k >= 0; --k) {
      const double b = bt[k];
      if (b == 0.0) continue;
      const double* hk = C + k * D;
      double hv[YJ];
      double s = 0.0;
#pragma unroll
      for (int j = 0; j < YJ; ++j) {
        const int e = tid + 32 * j;
        hv[j] = e > k ? hk[e] : 0.0;
        s = fma(hv[j], yr[j], s);
      }
      s = warp_sum_d(s) * b;
#pragma unroll
      for (int j = 0; j < YJ; ++j) yr[j] = fma(-s, hv[j], yr[j]);
    }
    double nn = 0.0;
#pragma unroll
    for (int j = 0; j < YJ; ++j) nn = fma(yr[j], yr[j], nn);
    nn = warp_sum_d(nn);
    const double inv = 1.0 / sqrt(nn);
#pragma unroll
    for (int j = 0; j < YJ; ++j) v[tid + 32 * j] = yr[j] * inv;
  }
  __syncthreads();
}

// ------------------------------------------------------------------ Lanczos
// Leading eigenvector by the Lanczos method (Lanczos 1950; the three-term recurrence with
// one local re-orthogonalisation against the newest vector), with C in registers as in
// eigen_top. Pass 1 runs the recurrence and checks the top eigenpair (theta, s) of the
// Lanczos tridiagonal T_n every kLzCheck steps from kLzFirst on (multisection on Sturm
// counts, inverse iteration) until the Ritz residual beta_n |s_n| is below kLzTol * theta. Pass 2 runs the
// same recurrence again from the same start - the same operations in the same order, so
// the same vectors bit for bit - and sums the Ritz vector v = sum_j s_j q_j in fp64 as it
// goes, so no basis is stored. The true residual |C v - theta v| is then measured; the call
// returns false, with C untouched in shared memory, when it is above kLzAccept * theta or
// nothing converged within kMax steps, and the caller runs eigen_top. With the residual
// below 1e-9 theta the eigenvector error is below 1e-9 / relative gap: 1e-5 at the 1e-4
// gap under which a node counts as a tie.
constexpr int kLzCheck = 16;
// first check after 48 steps: on whitened covariances (nearly flat spectra) none of 503
// solves sampled at 1344x768x240 converged in fewer, and a check (a multisection and an
// inverse iteration) costs as much as about 30 steps
constexpr int kLzFirst = 3 * kLzCheck;
constexpr double kLzTol = 1e-12;
constexpr double kLzAccept = 1e-9;

template <int D>
struct LzScratch {
  static constexpr int kMax = 2 * D;  // Lanczos steps at most
  static constexpr int kDoubles = 9 * kMax + 3 * D + 32;  // (2 D used for C q)
  static constexpr int kBytes = kDoubles * 8 + kMax * 4;
};

// Largest eigenvalue of the n x n tridiagonal (a, e; e2 = e^2) by multisection on Sturm
// counts over the Gershgorin interval (all threads). Returns the midpoint of the bracket.
__device__ double tridiag_top_value(const double* a, const double* e, const double* e2, int n,
                                    double* red, double* misc) {
  const int tid = threadIdx.x;
  double glo = 1e300, ghi = -1e300, emax = 0.0;
  for (int i = tid; i < n; i += kThreads) {
    const double r = (i > 0 ? fabs(e[i - 1]) : 0.0) + (i < n - 1 ? fabs(e[i]) : 0.0);
    glo = fmin(glo, a[i] - r);
    ghi = fmax(ghi, a[i] + r);
    if (i < n - 1) emax = fmax(emax, e2[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    glo = fmin(glo, __shfl_xor_sync(0xffffffffu, glo, o));
    ghi = fmax(ghi, __shfl_xor_sync(0xffffffffu, ghi, o));
    emax = fmax(emax, __shfl_xor_sync(0xffffffffu, emax, o));
  }
  if ((tid & 31) == 0) {
    red[tid >> 5] = glo;
    red[8 + (tid >> 5)] = ghi;
    red[16 + (tid >> 5)] = emax;
  }
  __syncthreads();
  if (tid == 0) {
    double lo = red[0], hi = red[8], em = red[16];
    for (int i = 1; i < kThreads / 32; ++i) {
      lo = fmin(lo, red[i]);
      hi = fmax(hi, red[8 + i]);
      em = fmax(em, red[16 + i]);
    }
    const double span = fmax(fabs(lo), fabs(hi)) + 1e-300;
    misc[0] = lo - 1e-12 * span;
    misc[1] = hi + 1e-12 * span;
    misc[2] = 2.2250738585072014e-308 * fmax(1.0, em);
  }
  __syncthreads();
  const double pivmin = misc[2];
  for (int round = 0; round < 12; ++round) {
    const double lo = misc[0], hi = misc[1];
    if (hi - lo <= 1e-14 * fmax(fabs(lo), fabs(hi))) break;
    const double x = lo + (hi - lo) * (double)(tid + 1) / (double)(kThreads + 1);
    const int c = sturm_count(a, e2, n, x, pivmin);
    double clo = (c <= n - 1) ? x : -1e300;  // at or below the top eigenvalue
    double chi = (c == n) ? x : 1e300;       // above it
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      clo = fmax(clo, __shfl_xor_sync(0xffffffffu, clo, o));
      chi = fmin(chi, __shfl_xor_sync(0xffffffffu, chi, o));
    }
    __syncthreads();
    if ((tid & 31) == 0) {
      red[tid >> 5] = clo;
      red[8 + (tid >> 5)] = chi;
    }
    __syncthreads();
    if (tid == 0) {
      double nlo = misc[0], nhi = misc[1];
      for (int i = 0; i < kThreads / 32; ++i) {
        nlo = fmax(nlo, red[i]);
        nhi = fmin(nhi, red[8 + i]);
      }
      misc[0] = nlo;
      misc[1] = nhi;
    }
    __syncthreads();
  }
  const double theta = 0.5 * (misc[0] + misc[1]);
  __syncthreads();
  return theta;
}

// Unit eigenvector y of the n x n tridiagonal (a, e) at the eigenvalue theta by two steps
// of inverse iteration (LU with partial pivoting, Newton-refined reciprocals); one thread.
// The factorisation and both solves carry their recurrences in registers (the next pivot,
// the next superdiagonal entry, the neighbouring solution entries) and keep in shared
// memory only what a later pass reads, so no step waits on a shared-memory round trip;
// the operations and their order are those of the plain LAPACK-style loops.
__device__ void tridiag_inverse_iteration(const double* a, const double* e, int n, double theta,
                                          double* dd, double* du, double* du2, double* dl, int* piv,
                                          double* y) {
  const double tiny = 1e-30 * (fabs(theta) + 1e-300);
  // factorisation: dd holds the reciprocals of the pivots
  double d0 = a[0] - theta;               // pivot candidate of row i
  double u0 = n > 1 ? e[0] : 0.0;         // superdiagonal entry of row i
  for (int i = 0; i < n - 1; ++i) {
    const double li = e[i];               // subdiagonal entry below row i
    const double dn = a[i + 1] - theta;   // diagonal of row i + 1
    const double un = i < n - 2 ? e[i + 1] : 0.0;  // superdiagonal of row i + 1
    if (fabs(d0) >= fabs(li)) {
      if (d0 == 0.0) d0 = tiny;
      const double r = rcp_nr(d0);
      const double f = li * r;
      dd[i] = r;
      dl[i] = f;
      du[i] = u0;
      du2[i] = 0.0;
      piv[i] = 0;
      d0 = dn - f * u0;
      u0 = un;
    } else {
      const double r = rcp_nr(li);
      const double f = d0 * r;
      dd[i] = r;
      dl[i] = f;
      du[i] = dn;
      du2[i] = un;
      piv[i] = 1;
      d0 = u0 - f * dn;
      u0 = -f * un;
    }
  }
  if (d0 == 0.0) d0 = tiny;
  dd[n - 1] = rcp_nr(d0);
  for (int i = 0; i < n; ++i) y[i] = 1.0 + 0.001 * i;
  for (int it = 0; it < 2; ++it) {
    // forward: apply the row interchanges and L^-1; yi carries y[i]
    double yi = y[0];
    for (int i = 0; i < n - 1; ++i) {
      const double yn = y[i + 1];
      if (piv[i] == 0) {
        y[i] = yi;
        yi = yn - dl[i] * yi;
      } else {
        y[i] = yn;
        yi = yi - dl[i] * yn;
      }
    }
    y[n - 1] = yi;
    // back substitution with U (diagonal reciprocals dd, superdiagonals du, du2)
    double y1 = y[n - 1] * dd[n - 1];      // y[i + 1]
    y[n - 1] = y1;
    double y2 = 0.0;                        // y[i + 2]
    if (n >= 2) {
      const double t = (y[n - 2] - du[n - 2] * y1) * dd[n - 2];
      y[n - 2] = t;
      y2 = y1;
      y1 = t;
    }
    for (int i = n - 3; i >= 0; --i) {
      const double t = (y[i] - du[i] * y1 - du2[i] * y2) * dd[i];
      y[i] = t;
      y2 = y1;
      y1 = t;
    }
    double nn = 0.0;
    for (int i = 0; i < n; ++i) nn += y[i] * y[i];
    const double inv = 1.0 / sqrt(nn);
    for (int i = 0; i < n; ++i) y[i] *= inv;
  }
}

// Returns true with the unit leading eigenvector of the symmetric C (fp64, shared memory)
// in v; false when the Lanczos iteration did not reach the accepted residual, with C as it
// was. `work`: LzScratch<D>::kBytes bytes of shared memory. While C is in registers its
// buffer holds the first D Lanczos vectors in fp64; when more steps are needed the Ritz
// vector is summed by a second pass of the same recurrence instead.
template <int D>
__device__ bool eigen_top_lanczos(double* C, double* v, unsigned char* work) {
  using L = LzScratch<D>;
  constexpr int R = D / 16;
  constexpr int M = D / 32;  // vector entries per lane (every warp holds whole vectors)
  constexpr int K = L::kMax;
  double* al = reinterpret_cast<double*>(work);  // alpha_j
  double* be = al + K;                            // beta_j
  double* b2 = be + K;
  double* s = b2 + K;
  double* dd = s + K;
  double* du = dd + K;
  double* du2 = du + K;
  double* dl = du2 + K;
  double* ev = dl + K;                            // off-diagonal copy for the solves
  double* wv = ev + K;                            // C q_j, double-buffered (2 D)
  double* red = wv + 3 * D;                       // 24
  double* misc = red + 24;                        // 8
  int* piv = reinterpret_cast<int*>(misc + 8);
  double* basis = C;                              // q_j, j < D, once C is in registers
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15, lane = tid & 31, warp = tid >> 5;

  double c[R][R];
#pragma unroll
  for (int ra = 0; ra < R; ++ra)
#pragma unroll
    for (int rb = 0; rb < R; ++rb) c[ra][rb] = C[(ty + 16 * ra) * D + tx + 16 * rb];
  __syncthreads();  // every thread has C in registers: its buffer is free

  // Lanczos state, identical in every warp: lane l holds entries l + 32 m of q_j, q_{j-1}
  double q[M], qp[M];
  double beta_prev = 0.0;
  auto start = [&]() {  // all-positive, slowly varying start vector, normalised
    double nn = 0.0;
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const int i = lane + 32 * m;
      q[m] = 1.0 + 0.37 * (double)((i * 7919) % 97) / 97.0;
      qp[m] = 0.0;
      nn = fma(q[m], q[m], nn);
    }
    nn = warp_sum_d(nn);
    const double inv = 1.0 / sqrt(nn);
#pragma unroll
    for (int m = 0; m < M; ++m) q[m] *= inv;
    beta_prev = 0.0;
  };
  // one step from q_j to q_{j+1} (one barrier); stores alpha_j and beta_j (warp 0) and
  // returns whether the Krylov space became invariant
  auto step = [&](int j) -> bool {
    double* w_out = wv + (j & 1) * D;
    {
      // the thread's columns tx + 16 rb: entry e lives in lane e % 32, slot e / 32
      double qv[R];
#pragma unroll
      for (int rb = 0; rb < R; ++rb) qv[rb] = __shfl_sync(0xffffffffu, q[rb >> 1], tx + 16 * (rb & 1));
#pragma unroll
      for (int ra = 0; ra < R; ++ra) {
        double acc = 0.0;
#pragma unroll
        for (int rb = 0; rb < R; ++rb) acc = fma(c[ra][rb], qv[rb], acc);
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (tx == 0) w_out[ty + 16 * ra] = acc;
      }
    }
    __syncthreads();
    double r[M], w[M];
#pragma unroll
    for (int m = 0; m < M; ++m) w[m] = w_out[lane + 32 * m];
    // two reductions per step, each of two sums at once: (q.w, q.q), then (q.r, r.r)
    double t0 = 0.0, t1 = 0.0;
#pragma unroll
    for (int m = 0; m < M; ++m) {
      t0 = fma(q[m], w[m], t0);
      t1 = fma(q[m], q[m], t1);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      t0 += __shfl_xor_sync(0xffffffffu, t0, o);
      t1 += __shfl_xor_sync(0xffffffffu, t1, o);
    }
    double alpha = t0;
#pragma unroll
    for (int m = 0; m < M; ++m) r[m] = w[m] - alpha * q[m] - beta_prev * qp[m];
    double u0 = 0.0, u1 = 0.0;  // one local re-orthogonalisation against q_j
#pragma unroll
    for (int m = 0; m < M; ++m) {
      u0 = fma(q[m], r[m], u0);
      u1 = fma(r[m], r[m], u1);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      u0 += __shfl_xor_sync(0xffffffffu, u0, o);
      u1 += __shfl_xor_sync(0xffffffffu, u1, o);
    }
    const double c2 = u0;
#pragma unroll
    for (int m = 0; m < M; ++m) r[m] -= c2 * q[m];
    alpha += c2;
    // |r - c2 q|^2 = r.r - 2 c2 (q.r) + c2^2 (q.q), with q.r = c2
    const double beta = sqrt(fmax(u1 - c2 * c2 * (2.0 - t1), 0.0));
    const bool invariant = !(beta > 1e-13 * (fabs(alpha) + 1e-300));
    const double inv = invariant ? 0.0 : 1.0 / beta;
    if (warp == 0 && lane == 0) {
      al[j] = alpha;
      be[j] = beta;
      b2[j] = beta * beta;
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
      qp[m] = q[m];
      q[m] = r[m] * inv;
    }
    beta_prev = beta;
    return invariant;
  };

  // ---- pass 1: steps until the Ritz pair has converged (the first D vectors kept)
  start();
  int n = 0;
  double theta = 0.0;
  bool done = false;
  for (int j = 0; j < K && !done; ++j) {
    if (warp == 0 && j < D) {
#pragma unroll
      for (int m = 0; m < M; ++m) basis[j * D + lane + 32 * m] = q[m];
    }
    const bool invariant = step(j);
    n = j + 1;
    if (invariant || (n >= kLzFirst && n % kLzCheck == 0) || n == K) {
      __syncthreads();  // al / be of step j are written
      theta = tridiag_top_value(al, be, b2, n, red, misc);
      if (tid == 0) {
        for (int i = 0; i < n; ++i) ev[i] = be[i];
        tridiag_inverse_iteration(al, ev, n, theta, dd, du, du2, dl, piv, s);
        const double rho = invariant ? 0.0 : fabs(be[n - 1] * s[n - 1]);
        misc[3] = (rho <= kLzTol * fabs(theta) || n == K || invariant) ? 1.0 : 0.0;
      }
      __syncthreads();
      done = misc[3] != 0.0;
      __syncthreads();
    }
  }
  // ---- Ritz vector v = sum_j s_j q_j: from the kept vectors, or by a second pass of the
  //      same recurrence (the same vectors bit for bit)
  double acc[M];
#pragma unroll
  for (int m = 0; m < M; ++m) acc[m] = 0.0;
  if (n <= D) {
    for (int j = 0; j < n; ++j) {
      const double sj = s[j];
#pragma unroll
      for (int m = 0; m < M; ++m) acc[m] = fma(sj, basis[j * D + lane + 32 * m], acc[m]);
    }
  } else {
    start();
    for (int j = 0; j < n; ++j) {
      const double sj = s[j];
#pragma unroll
      for (int m = 0; m < M; ++m) acc[m] = fma(sj, q[m], acc[m]);
      if (j + 1 < n) step(j);
    }
  }
  {
    double t = 0.0;
#pragma unroll
    for (int m = 0; m < M; ++m) t = fma(acc[m], acc[m], t);
    const double inv = 1.0 / sqrt(warp_sum_d(t));
    if (warp == 0) {
#pragma unroll
      for (int m = 0; m < M; ++m) v[lane + 32 * m] = acc[m] * inv;
    }
  }
  __syncthreads();
  // ---- true residual |C v - theta v| (C still in registers)
  bool accepted;
  {
    double vv[R];
#pragma unroll
    for (int rb = 0; rb < R; ++rb) vv[rb] = v[tx + 16 * rb];
    double part = 0.0;
#pragma unroll
    for (int ra = 0; ra < R; ++ra) {
      double a2 = 0.0;
#pragma unroll
      for (int rb = 0; rb < R; ++rb) a2 = fma(c[ra][rb], vv[rb], a2);
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) a2 += __shfl_xor_sync(0xffffffffu, a2, off);
      const double rr = a2 - theta * v[ty + 16 * ra];
      if (tx == 0) part = fma(rr, rr, part);
    }
    const double tot = block_sum_d(part, red);
    accepted = fabs(theta) > 0.0 && sqrt(tot) <= kLzAccept * fabs(theta);
  }
  if (!accepted) {
    // give C back to the full solver
#pragma unroll
    for (int ra = 0; ra < R; ++ra)
#pragma unroll
      for (int rb = 0; rb < R; ++rb) C[(ty + 16 * ra) * D + tx + 16 * rb] = c[ra][rb];
  }
  __syncthreads();
  return accepted;
}

// The leading eigenvector: Lanczos first, the full tridiagonalisation solve as fallback.
template <int D>
__device__ __forceinline__ void leading_eigvec(double* C, double* scr, unsigned char* work, double* v) {
  if (!eigen_top_lanczos<D>(C, v, work)) eigen_top<D>(C, scr, v);
}

// ------------------------------------------------------------------ one bisection
struct SplitScratch {
  int hist[256];
  int warp_tot[kThreads / 32];
  double red[kThreads / 32];
  int sel[4];  // bin, remaining rank, count of equal keys, chosen token
};

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Radix select over the n values key(i) (uint32) restricted to filt(i): returns the
// r-th smallest (1-based) and leaves in sc->sel[1] its rank among equal values and in
// sc->sel[2] how many values equal it.
template <class KeyF, class FiltF>
__device__ uint32_t radix_select(int n, int r, KeyF key, FiltF filt, SplitScratch* sc) {
  uint32_t prefix = 0, mask = 0;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int b = threadIdx.x; b < 256; b += kThreads) sc->hist[b] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kThreads) {
      if (!filt(i)) continue;
      const uint32_t k = key(i);
      if ((k & mask) == prefix) atomicAdd(&sc->hist[(k >> shift) & 255u], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int cum = 0, b = 0;
      for (; b < 255; ++b) {
        if (cum + sc->hist[b] >= r) break;
        cum += sc->hist[b];
      }
      sc->sel[0] = b;
      sc->sel[1] = r - cum;
      sc->sel[2] = sc->hist[b];
    }
    __syncthreads();
    prefix |= (uint32_t)sc->sel[0] << shift;
    mask |= 255u << shift;
    r = sc->sel[1];
    __syncthreads();
  }
  return prefix;
}

// Projections proj[i] = x[tin[i]] . v of n tokens (fp64 dot products, stored as fp32) by
// the CTA; returns the thread's share of their fp64 sum. 8 lanes per token, 4 tokens per
// warp at a time (PL = D / 8 components per lane, as float4 loads), so each warp keeps
// several row gathers in flight.
template <int D>
__device__ double project_tokens(const double* v, const float* __restrict__ Xh, const int32_t* tin,
                                 float* proj, int n) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int PL = D / 8;
  const int sub = lane >> 3, sl = lane & 7;
  double vl[PL];
#pragma unroll
  for (int j = 0; j < PL; ++j) vl[j] = v[sl * PL + j];
  double psum = 0.0;
  for (int i0 = 4 * warp; i0 < n; i0 += 4 * (kThreads / 32)) {
    const int i = i0 + sub;
    double d = 0.0;
    if (i < n) {
      const float4* xr = reinterpret_cast<const float4*>(Xh + (size_t)tin[i] * D + sl * PL);
#pragma unroll
      for (int j = 0; j < PL / 4; ++j) {
        const float4 x4 = xr[j];
        d = fma((double)x4.x, vl[4 * j], d);
        d = fma((double)x4.y, vl[4 * j + 1], d);
        d = fma((double)x4.z, vl[4 * j + 2], d);
        d = fma((double)x4.w, vl[4 * j + 3], d);
      }
    }
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
    if (sl == 0 && i < n) {
      proj[i] = (float)d;
      psum += d;
    }
  }
  return psum;
}

// Splits one node of m > 1 blocks (n = 64 m tokens) whose projections are in proj and
// whose projection mean is pbar: sign from the third central moment, the floor(m/2)*64-th
// smallest (projection, token) and a stable partition of tin into tout (left part first).
// Writes the children's labels 2c / 2c + 1 into tree_next when it is not null.
__device__ void split_projected(const int32_t* tin, int32_t* tout, const float* proj, double pbar, int n,
                                int m, int label, int32_t* tree_next, SplitScratch* sc) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  double m3 = 0.0;
  for (int i = tid; i < n; i += kThreads) {
    const double c = (double)proj[i] - pbar;
    m3 += c * c * c;
  }
  m3 = block_sum_d(m3, sc->red);
  const float sgn = m3 < 0.0 ? -1.f : 1.f;
  const int cut = (m / 2) * kBlock;
  auto pkey = [&](int i) { return order_key(sgn * proj[i]); };
  auto all = [](int) { return true; };
  const uint32_t T = radix_select(n, cut, pkey, all, sc);
  const int r_eq = sc->sel[1], n_eq = sc->sel[2];
  __syncthreads();
  uint32_t Ttok = 0xffffffffu;  // ties at T: the r_eq lowest tokens go left
  if (n_eq > r_eq) {
    auto tkey = [&](int i) { return (uint32_t)tin[i]; };
    auto eq = [&](int i) { return pkey(i) == T; };
    Ttok = radix_select(n, r_eq, tkey, eq, sc);
  }
  // stable partition
  int nl_base = 0;
  for (int base = 0; base < n; base += kThreads) {
    const int i = base + tid;
    int t = 0;
    bool left = false;
    if (i < n) {
      t = tin[i];
      const uint32_t k = pkey(i);
      left = k < T || (k == T && (uint32_t)t <= Ttok);
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, left);
    const int wrank = __popc(bal & ((1u << lane) - 1u));
    __syncthreads();
    if (lane == 0) sc->warp_tot[warp] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int q = 0; q < kThreads / 32; ++q) {
      const int c = sc->warp_tot[q];
      before += q < warp ? c : 0;
      total += c;
    }
    if (i < n) {
      const int lrank = nl_base + before + wrank;
      const int pos = left ? lrank : cut + (i - lrank);
      tout[pos] = t;
      if (tree_next != nullptr) tree_next[t] = 2 * label + (left ? 0 : 1);
    }
    nl_base += total;
  }
  __syncthreads();
}

// Projections on v by the CTA, then the split (small nodes: one CTA does both).
template <int D>
__device__ void split_node(const double* v, const float* __restrict__ Xh, const int32_t* tin,
                           int32_t* tout, float* proj, int n, int m, int label,
                           int32_t* tree_next, SplitScratch* sc) {
  const double psum = project_tokens<D>(v, Xh, tin, proj, n);
  __syncthreads();
  const double pbar = block_sum_d(psum, sc->red) / n;
  split_projected(tin, tout, proj, pbar, n, m, label, tree_next, sc);
}

// A leaf carried to the next level: same tokens, label 2c.
__device__ __forceinline__ void carry_leaf(const int32_t* tin, int32_t* tout, int label,
                                           int32_t* tree_next) {
  for (int i = threadIdx.x; i < kBlock; i += kThreads) {
    const int t = tin[i];
    tout[i] = t;
    if (tree_next != nullptr) tree_next[t] = 2 * label;
  }
}

// Shared memory of the split kernels: C (D x D doubles), mu, v, eigen scratch, staging,
// split scratch.
template <int D>
struct SplitSmem {
  static constexpr int kC = D * D * 8;
  static constexpr int kVec = 2 * D * 8;
  static constexpr int kStage = 2 * kTile * (D + 4) * 4;  // also the Lanczos scratch
  static_assert(kStage >= LzScratch<D>::kBytes, "Lanczos scratch exceeds the staging buffer");
  static constexpr int kBytes = kC + kVec + EigScratch<D>::kBytes + kStage + (int)sizeof(SplitScratch) + 64;
};

struct LevelArgs {
  const float* X;     // [BH][nv][D]
  const int32_t* tin; // [BH][nv]
  int32_t* tout;
  float* proj;        // [BH][nv]
  int32_t* tree;      // [BH][L+1][nv] or null
  int nv, nb, level, levels;
};

template <int D>
__device__ __forceinline__ void carve(unsigned char* smem, double** C, double** mu, double** v,
                                      double** scr, float** stage, SplitScratch** sc) {
  using S = SplitSmem<D>;
  *C = reinterpret_cast<double*>(smem);
  *mu = reinterpret_cast<double*>(smem + S::kC);
  *v = *mu + D;
  *scr = reinterpret_cast<double*>(smem + S::kC + S::kVec);
  *stage = reinterpret_cast<float*>(smem + S::kC + S::kVec + EigScratch<D>::kBytes);
  *sc = reinterpret_cast<SplitScratch*>(smem + S::kC + S::kVec + EigScratch<D>::kBytes + S::kStage);
}

// Large levels, step 1: raw sums of the summed nodes (labels stride * i: every node at the
// root, the left children below it) over chunks of their tokens, fp64 atomics into
// nacc[node][bh] = (S2 = sum x x^T [D x D], S1 = sum x [D]). grid (summed nodes * cpn, BH).
// A left leaf is summed too: its right sibling (3-block parents) needs it.
template <int D>
__global__ void __launch_bounds__(kThreads) node_moments_kernel(LevelArgs a, int cpn, int stride,
                                                                double* __restrict__ nacc) {
  extern __shared__ __align__(16) unsigned char smem[];
  double* S2 = reinterpret_cast<double*>(smem);
  double* S1 = S2 + D * D;
  float* stage = reinterpret_cast<float*>(S1 + D);
  const int c = stride * (blockIdx.x / cpn), chunk = blockIdx.x % cpn;
  const size_t bh = blockIdx.y;
  int st, m;
  if (!node_of(a.nb, a.level, c, &st, &m) || m < 1 || (stride == 1 && m == 1)) return;
  const int t0 = chunk * kChunkTok;
  const int n = min(kChunkTok, m * kBlock - t0);
  if (n <= 0) return;
  for (int i = threadIdx.x; i < D * D + D; i += kThreads) S2[i] = 0.0;
  const float* Xh = a.X + bh * (size_t)a.nv * D;
  const int32_t* tseg = a.tin + bh * (size_t)a.nv + st * kBlock + t0;
  auto rowp = [&](int i) { return Xh + (size_t)tseg[i] * D; };
  accumulate_moments_rows<D>(n, rowp, stage, S2, S1);
  double* dst = nacc + ((size_t)c * gridDim.y + bh) * (D * D + D);
  for (int i = threadIdx.x; i < D * D + D; i += kThreads) atomicAdd(dst + i, S2[i]);
}

// Large levels, step 2: one CTA per node finishes the covariance (a right child's sums are
// its parent's minus its left sibling's; they are kept for its children) and writes the
// leading eigenvector to vbuf[node][bh]. grid (nodes, BH).
template <int D>
__global__ void __launch_bounds__(kThreads) node_eig_kernel(LevelArgs a, double* __restrict__ nacc,
                                                            const double* __restrict__ nacc_up,
                                                            double* __restrict__ vbuf) {
  extern __shared__ __align__(16) unsigned char smem[];
  double *C, *mu, *v, *scr;
  float* stage;
  SplitScratch* sc;
  carve<D>(smem, &C, &mu, &v, &scr, &stage, &sc);
  const int c = blockIdx.x;
  const size_t bh = blockIdx.y;
  int st, m;
  if (!node_of(a.nb, a.level, c, &st, &m) || m == 1) return;
  const int n = m * kBlock;
  double* src = nacc + ((size_t)c * gridDim.y + bh) * (D * D + D);
  if (nacc_up != nullptr && (c & 1)) {
    const double* up = nacc_up + ((size_t)(c >> 1) * gridDim.y + bh) * (D * D + D);
    const double* left = nacc + ((size_t)(c - 1) * gridDim.y + bh) * (D * D + D);
    for (int e = threadIdx.x; e < D * D + D; e += kThreads) src[e] = up[e] - left[e];
    __syncthreads();
  }
  const double inv = 1.0 / n;
  for (int i = threadIdx.x; i < D; i += kThreads) mu[i] = src[D * D + i] * inv;
  __syncthreads();
  for (int e = threadIdx.x; e < D * D; e += kThreads) C[e] = src[e] * inv - mu[e / D] * mu[e % D];
  __syncthreads();
  leading_eigvec<D>(C, scr, reinterpret_cast<unsigned char*>(stage), v);
  double* vout = vbuf + ((size_t)c * gridDim.y + bh) * D;
  for (int i = threadIdx.x; i < D; i += kThreads) vout[i] = v[i];
}

// Large levels, step 3: projections of every node's tokens on its eigenvector, in chunks of
// kChunkTok tokens per CTA (one CTA per node would keep too few row gathers in flight for
// the 10^5 tokens of a top-level node). grid (nodes * cpn, BH).
template <int D>
__global__ void __launch_bounds__(kThreads) node_project_kernel(LevelArgs a, int cpn, const double* __restrict__ vbuf) {
  const int c = blockIdx.x / cpn, chunk = blockIdx.x % cpn;
  const size_t bh = blockIdx.y;
  int st, m;
  if (!node_of(a.nb, a.level, c, &st, &m) || m == 1) return;
  const int t0 = chunk * kChunkTok;
  const int n = min(kChunkTok, m * kBlock - t0);
  if (n <= 0) return;
  const size_t hoff = bh * (size_t)a.nv + st * kBlock + t0;
  project_tokens<D>(vbuf + ((size_t)c * gridDim.y + bh) * D, a.X + bh * (size_t)a.nv * D, a.tin + hoff,
                    a.proj + hoff, n);
}

// Large levels, step 4: one CTA per node splits it from its projections (or carries a
// leaf). grid (nodes, BH).
__global__ void __launch_bounds__(kThreads) node_split_kernel(LevelArgs a) {
  __shared__ SplitScratch sc;
  const int c = blockIdx.x;
  const size_t bh = blockIdx.y;
  int st, m;
  if (!node_of(a.nb, a.level, c, &st, &m)) return;
  const size_t hoff = bh * (size_t)a.nv + st * kBlock;
  int32_t* tree_next = a.tree ? a.tree + bh * (size_t)(a.levels + 1) * a.nv + (size_t)(a.level + 1) * a.nv : nullptr;
  if (m == 1) {
    carry_leaf(a.tin + hoff, a.tout + hoff, c, tree_next);
    return;
  }
  const int n = m * kBlock;
  const float* proj = a.proj + hoff;
  double psum = 0.0;
  for (int i = threadIdx.x; i < n; i += kThreads) psum += (double)proj[i];
  const double pbar = block_sum_d(psum, sc.red) / n;
  split_projected(a.tin + hoff, a.tout + hoff, proj, pbar, n, m, c, tree_next, &sc);
}

// Small nodes: one CTA per node of level `level` splits it and its whole subtree down to
// single blocks, reading and writing the token arrays tok[lev & 1] -> tok[(lev + 1) & 1].
template <int D>
__global__ void __launch_bounds__(kThreads) subtree_kernel(LevelArgs a, int32_t* tok0, int32_t* tok1) {
  extern __shared__ __align__(16) unsigned char smem[];
  double *C, *mu, *v, *scr;
  float* stage;
  SplitScratch* sc;
  carve<D>(smem, &C, &mu, &v, &scr, &stage, &sc);
  const int c0 = blockIdx.x;
  const size_t bh = blockIdx.y;
  int st0, m0;
  if (!node_of(a.nb, a.level, c0, &st0, &m0)) return;
  const float* Xh = a.X + bh * (size_t)a.nv * D;
  for (int lev = a.level; lev < a.levels; ++lev) {
    const int span = 1 << (lev - a.level);
    const int32_t* tin = (lev & 1) ? tok1 : tok0;
    int32_t* tout = (lev & 1) ? tok0 : tok1;
    int32_t* tree_next = a.tree ? a.tree + bh * (size_t)(a.levels + 1) * a.nv + (size_t)(lev + 1) * a.nv : nullptr;
    for (int cc = c0 * span; cc < (c0 + 1) * span; ++cc) {
      int st, m;
      if (!node_of(a.nb, lev, cc, &st, &m)) continue;
      const size_t hoff = bh * (size_t)a.nv + st * kBlock;
      if (m == 1) {
        carry_leaf(tin + hoff, tout + hoff, cc, tree_next);
        __syncthreads();
        continue;
      }
      const int n = m * kBlock;
      node_covariance<D>(Xh, tin + hoff, n, stage, C, mu);
      leading_eigvec<D>(C, scr, reinterpret_cast<unsigned char*>(stage), v);
      split_node<D>(v, Xh, tin + hoff, tout + hoff, a.proj + hoff, n, m, cc, tree_next, sc);
    }
    __syncthreads();  // the next level reads what this level wrote (same CTA)
    __threadfence_block();
  }
}

// ------------------------------------------------------------------ canonical order
// Sorts the 64 tokens of every leaf ascending (in place) and marks each leaf's smallest
// token: mark[bh][token] = leaf + 1. One warp per leaf; grid (ceil(nb / 8), BH).
__global__ void __launch_bounds__(kThreads) leaf_sort_kernel(int32_t* tok, int nv, int nb, int32_t* mark) {
  __shared__ int32_t buf[kThreads / 32][kBlock];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int leaf = blockIdx.x * (kThreads / 32) + warp;
  if (leaf >= nb) return;
  const size_t bh = blockIdx.y;
  int32_t* seg = tok + bh * (size_t)nv + (size_t)leaf * kBlock;
  const int a = seg[lane], b = seg[lane + 32];
  buf[warp][lane] = a;
  buf[warp][lane + 32] = b;
  __syncwarp();
  int ra = 0, rb = 0;  // tokens are distinct: rank = number of smaller tokens
  for (int j = 0; j < kBlock; ++j) {
    const int x = buf[warp][j];
    ra += x < a;
    rb += x < b;
  }
  __syncwarp();
  seg[ra] = a;
  seg[rb] = b;
  if (ra == 0) mark[bh * (size_t)nv + a] = leaf + 1;
  if (rb == 0) mark[bh * (size_t)nv + b] = leaf + 1;
}

// perm lists the leaves by their smallest token: a scan over the marks in token order.
// One CTA of 1024 threads per head.
__global__ void __launch_bounds__(1024) leaf_order_kernel(const int32_t* __restrict__ tok,
                                                          const int32_t* __restrict__ mark, int nv,
                                                          int32_t* __restrict__ order) {
  __shared__ int wsum[32];
  __shared__ int base;
  const size_t bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) base = 0;
  __syncthreads();
  for (int t0 = 0; t0 < nv; t0 += 1024) {
    const int t = t0 + tid;
    const int mk = t < nv ? mark[bh * (size_t)nv + t] : 0;
    const uint32_t bal = __ballot_sync(0xffffffffu, mk != 0);
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    int before = base;
    for (int q = 0; q < warp; ++q) before += wsum[q];
    if (mk != 0) order[bh * (size_t)(nv / kBlock) + before + __popc(bal & ((1u << lane) - 1u))] = mk - 1;
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int q = 0; q < 32; ++q) tot += wsum[q];
      base += tot;
    }
    __syncthreads();
  }
}

// perm[bh][r * 64 + j] = tok[bh][order[r] * 64 + j]. grid (ceil(nv / 256), BH).
__global__ void __launch_bounds__(kThreads) perm_kernel(const int32_t* __restrict__ tok,
                                                        const int32_t* __restrict__ order, int nv,
                                                        int32_t* __restrict__ perm) {
  const size_t bh = blockIdx.y;
  const int p = blockIdx.x * kThreads + threadIdx.x;
  if (p >= nv) return;
  const int leaf = order[bh * (size_t)(nv / kBlock) + p / kBlock];
  perm[bh * (size_t)nv + p] = tok[bh * (size_t)nv + (size_t)leaf * kBlock + (p % kBlock)];
}

// Qp/Kp/Vp rows p < nv come from rows perm[p]; dense rows are copied. 16 bytes per thread.
// Q rows follow perm, K and V rows follow perm_kv (the same array under q_reuse_k).
template <int D>
__global__ void __launch_bounds__(kThreads) gather_kernel(const uint16_t* __restrict__ Q, const uint16_t* __restrict__ K,
                                                          const uint16_t* __restrict__ V, const int32_t* __restrict__ perm,
                                                          const int32_t* __restrict__ perm_kv, int N, int nv,
                                                          uint16_t* __restrict__ Qp, uint16_t* __restrict__ Kp,
                                                          uint16_t* __restrict__ Vp) {
  constexpr int CH = D / 8;
  const size_t bh = blockIdx.y;
  const long long e = (long long)blockIdx.x * kThreads + threadIdx.x;
  if (e >= (long long)N * CH) return;
  const int p = (int)(e / CH), c = (int)(e % CH);
  const int sq = p < nv ? perm[bh * (size_t)nv + p] : p;
  const int sk = p < nv ? perm_kv[bh * (size_t)nv + p] : p;
  const size_t dof = (bh * N + p) * D + c * 8;
  *reinterpret_cast<uint4*>(Qp + dof) = ldg_nc_v4(Q + (bh * N + sq) * D + c * 8);
  *reinterpret_cast<uint4*>(Kp + dof) = ldg_nc_v4(K + (bh * N + sk) * D + c * 8);
  *reinterpret_cast<uint4*>(Vp + dof) = ldg_nc_v4(V + (bh * N + sk) * D + c * 8);
}

// ------------------------------------------------------------------ host side
struct Plan {
  int levels = 0, first_small = 0;  // levels < first_small use the multi-CTA path
  int max_large_nodes = 0;
  std::vector<int> cpn;             // chunks per node at each large level
  size_t off_macc, off_lmat, off_x, off_tok0, off_tok1, off_proj, off_nacc, off_nacc2, off_vbuf, off_mark, off_order,
      total;
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

inline Plan make_plan(int bh, int nb, int d) {
  Plan P;
  const size_t nv = (size_t)nb * kBlock;
  P.levels = num_levels(nb);
  P.first_small = P.levels;
  for (int l = 0; l < P.levels; ++l) {
    int maxm = 0;
    for (int c = 0; c < (1 << l); ++c) {
      int st, m;
      if (node_of(nb, l, c, &st, &m)) maxm = m > maxm ? m : maxm;
    }
    if (maxm <= kSmallBlocks) {
      P.first_small = l;
      break;
    }
    P.cpn.push_back((maxm * kBlock + kChunkTok - 1) / kChunkTok);
  }
  P.max_large_nodes = P.first_small > 0 ? (1 << (P.first_small - 1)) : 0;
  size_t o = 0;
  P.off_macc = o;  o = align256(o + (size_t)bh * d * d * 8);
  P.off_lmat = o;  o = align256(o + (size_t)bh * d * d * 4);
  P.off_x = o;     o = align256(o + (size_t)bh * nv * d * 4);
  P.off_tok0 = o;  o = align256(o + (size_t)bh * nv * 4);
  P.off_tok1 = o;  o = align256(o + (size_t)bh * nv * 4);
  P.off_proj = o;  o = align256(o + (size_t)bh * nv * 4);
  P.off_nacc = o;  o = align256(o + (size_t)P.max_large_nodes * bh * ((size_t)d * d + d) * 8);
  P.off_nacc2 = o; o = align256(o + (size_t)P.max_large_nodes * bh * ((size_t)d * d + d) * 8);
  P.off_vbuf = o;  o = align256(o + (size_t)P.max_large_nodes * bh * d * 8);
  P.off_mark = o;  o = align256(o + (size_t)bh * nv * 4);
  P.off_order = o; o = align256(o + (size_t)bh * nb * 4);
  P.total = o;
  return P;
}

}  // namespace rb

inline size_t reblock_workspace_bytes(int bh, int nb, int d) {
  if (nb <= 0) return 0;
  return rb::make_plan(bh, nb, d).total;
}

// Partition of the video rows of A (whitened by the second moment of the video rows of
// Bm) into 64-row leaves: perm (and tree, when not null).
template <int D>
int partition_run(int bh, int N, int nb, const uint16_t* A, const uint16_t* Bm, int32_t* perm,
                  int32_t* tree, void* ws, cudaStream_t cs) {
  using namespace rb;
  const uint16_t* Q = A;  // the rows being partitioned
  const uint16_t* K = Bm; // the rows whose second moment whitens them
  const int nv = nb * kBlock;
  if (nb > 0) {
    const Plan P = make_plan(bh, nb, D);
    unsigned char* w = static_cast<unsigned char*>(ws);
    double* macc = reinterpret_cast<double*>(w + P.off_macc);
    float* lmat = reinterpret_cast<float*>(w + P.off_lmat);
    float* X = reinterpret_cast<float*>(w + P.off_x);
    int32_t* tok0 = reinterpret_cast<int32_t*>(w + P.off_tok0);
    int32_t* tok1 = reinterpret_cast<int32_t*>(w + P.off_tok1);
    float* proj = reinterpret_cast<float*>(w + P.off_proj);
    double* nacc_buf[2] = {reinterpret_cast<double*>(w + P.off_nacc), reinterpret_cast<double*>(w + P.off_nacc2)};
    double* vbuf = reinterpret_cast<double*>(w + P.off_vbuf);
    int32_t* mark = reinterpret_cast<int32_t*>(w + P.off_mark);
    int32_t* order = reinterpret_cast<int32_t*>(w + P.off_order);
    const size_t tree_stride = (size_t)(P.levels + 1) * nv;

    if (cudaMemsetAsync(macc, 0, (size_t)bh * D * D * 8, cs) != cudaSuccess) return SPARK_ECUDA;
    if (cudaMemsetAsync(mark, 0, (size_t)bh * nv * 4, cs) != cudaSuccess) return SPARK_ECUDA;
    const int smem_km = D * D * 8 + kTile * (D + 4) * 4;
    cudaFuncSetAttribute(kmoment_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_km);
    kmoment_kernel<D><<<dim3((nv + kChunkTok - 1) / kChunkTok, bh), kThreads, smem_km, cs>>>(K, N, nv, macc);
    cudaFuncSetAttribute(cholesky_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, D * D * 8);
    cholesky_kernel<D><<<bh, kThreads, D * D * 8, cs>>>(macc, nv, lmat);
    const int smem_wh = D * D * 4 + 64 * D * 4;
    cudaFuncSetAttribute(whiten_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_wh);
    whiten_kernel<D><<<dim3((nv + kWhTok - 1) / kWhTok, bh), kThreads, smem_wh, cs>>>(Q, N, nv, lmat, X, tok0, tree,
                                                                                    tree_stride);
    SPARK_LAUNCH_CHECK();
    note_launches(3);

    LevelArgs a;
    a.X = X;
    a.proj = proj;
    a.tree = tree;
    a.nv = nv;
    a.nb = nb;
    a.levels = P.levels;
    const int smem_split = SplitSmem<D>::kBytes;
    cudaFuncSetAttribute(node_eig_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_split);
    cudaFuncSetAttribute(subtree_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_split);
    const int smem_nm = (D * D + D) * 8 + 2 * kTile * (D + 4) * 4;
    cudaFuncSetAttribute(node_moments_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_nm);
    // level l keeps its nodes' raw sums in nacc_buf[l & 1]; below the root only the left
    // children are summed over their tokens, a right child's sums are its parent's minus its
    // left sibling's (node_eig_kernel derives and stores them); then the eigenvectors (one
    // CTA per node), the projections (many CTAs per node) and the splits (one CTA per node)
    for (int l = 0; l < P.first_small; ++l) {
      a.level = l;
      a.tin = (l & 1) ? tok1 : tok0;
      a.tout = (l & 1) ? tok0 : tok1;
      const int nodes = 1 << l;
      double* nacc = nacc_buf[l & 1];
      const double* nacc_up = l > 0 ? nacc_buf[(l - 1) & 1] : nullptr;
      if (cudaMemsetAsync(nacc, 0, (size_t)nodes * bh * ((size_t)D * D + D) * 8, cs) != cudaSuccess)
        return SPARK_ECUDA;
      const int summed = l > 0 ? nodes / 2 : 1;
      node_moments_kernel<D><<<dim3(summed * P.cpn[l], bh), kThreads, smem_nm, cs>>>(a, P.cpn[l], l > 0 ? 2 : 1, nacc);
      node_eig_kernel<D><<<dim3(nodes, bh), kThreads, smem_split, cs>>>(a, nacc, nacc_up, vbuf);
      node_project_kernel<D><<<dim3(nodes * P.cpn[l], bh), kThreads, 0, cs>>>(a, P.cpn[l], vbuf);
      node_split_kernel<<<dim3(nodes, bh), kThreads, 0, cs>>>(a);
      SPARK_LAUNCH_CHECK();
      note_launches(4);
    }
    if (P.first_small < P.levels) {
      a.level = P.first_small;
      subtree_kernel<D><<<dim3(1 << P.first_small, bh), kThreads, smem_split, cs>>>(a, tok0, tok1);
      SPARK_LAUNCH_CHECK();
      note_launches(1);
    }
    int32_t* final_tok = (P.levels & 1) ? tok1 : tok0;
    leaf_sort_kernel<<<dim3((nb + 7) / 8, bh), kThreads, 0, cs>>>(final_tok, nv, nb, mark);
    leaf_order_kernel<<<bh, 1024, 0, cs>>>(final_tok, mark, nv, order);
    perm_kernel<<<dim3((nv + kThreads - 1) / kThreads, bh), kThreads, 0, cs>>>(final_tok, order, nv, perm);
    SPARK_LAUNCH_CHECK();
    note_launches(3);
  }
  return SPARK_OK;
}

// q_reuse_k when perm_k is null (K and V follow the query partition); otherwise the keys
// get their own partition (whitened by the queries' second moment) in perm_k.
template <int D>
int reblock_run(int bh, int N, int nb, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                int32_t* perm, int32_t* perm_k, uint16_t* Qp, uint16_t* Kp, uint16_t* Vp,
                int32_t* tree, void* ws, cudaStream_t cs) {
  using namespace rb;
  const int nv = nb * kBlock;
  int st = partition_run<D>(bh, N, nb, Q, K, perm, tree, ws, cs);
  if (st != SPARK_OK) return st;
  if (perm_k != nullptr) {
    st = partition_run<D>(bh, N, nb, K, Q, perm_k, nullptr, ws, cs);
    if (st != SPARK_OK) return st;
  }
  const long long chunks = (long long)N * (D / 8);
  gather_kernel<D><<<dim3((unsigned)((chunks + kThreads - 1) / kThreads), bh), kThreads, 0, cs>>>(
      Q, K, V, perm, perm_k != nullptr ? perm_k : perm, N, nv, Qp, Kp, Vp);
  SPARK_LAUNCH_CHECK();
  note_launches(1);
  return SPARK_OK;
}

inline int reblock_launch(int bh, int N, int nb, int d, const uint16_t* Q, const uint16_t* K,
                          const uint16_t* V, int32_t* perm, int32_t* perm_k, uint16_t* Qp,
                          uint16_t* Kp, uint16_t* Vp, int32_t* tree, void* ws, cudaStream_t stream) {
  return d == 128 ? reblock_run<128>(bh, N, nb, Q, K, V, perm, perm_k, Qp, Kp, Vp, tree, ws, stream)
                  : reblock_run<64>(bh, N, nb, Q, K, V, perm, perm_k, Qp, Kp, Vp, tree, ws, stream);
}

}  // namespace spark
