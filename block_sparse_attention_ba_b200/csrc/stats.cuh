// stats.cuh — K6: per-block mean and diagonal (per-dimension) variance.
//
// Stage one of BA-Att pools Q and K block-wise before any scoring, and the
// covariance correction needs each block's per-dimension variance
// ("Efficient Long-Context Modeling in DLMs via Block Approximate Sparse
// Attention": abstract; "Core claim").
//
// One CTA of 256 threads per (head, block). The block's rows are read once
// from HBM with 16-byte vector loads, all issued up front and kept in
// registers; the mean and then the centred second moment are reduced from
// those registers (an exact two-pass variance with a single HBM read).
// Q heads and K heads are handled by one launch: CTAs [0, B*Hq*nq) do Q.
#pragma once

#include "common.cuh"

#ifndef BA_STATS_EVICT_FIRST
#define BA_STATS_EVICT_FIRST 1
#endif

namespace baatt {

constexpr int kStatsThreads = 256;

template <typename T, int D, int RPT>
__global__ void __launch_bounds__(kStatsThreads) stats_kernel(const T *__restrict__ Q, const T *__restrict__ K,
                                                              float *__restrict__ q_mean, float *__restrict__ q_var,
                                                              float *__restrict__ k_mean, float *__restrict__ k_var,
                                                              int B, int Hq, int Hkv, int N, int N_alloc, int block,
                                                              int nb, int kblock, int nbk) {
  constexpr int VEC = Elem<T>::kVec;
  constexpr int COLS = D / VEC;                   // 16-byte vectors per row
  constexpr int RPP = kStatsThreads / COLS;       // rows covered per pass
  __shared__ float red[RPP][D];
  __shared__ float mean_s[D];

  const long long n_q_ctas = static_cast<long long>(B) * Hq * nb;
  long long cta = blockIdx.x;
  const bool is_q = cta < n_q_ctas;
  if (!is_q) cta -= n_q_ctas;
  const int nbx = is_q ? nb : nbk, bsize = is_q ? block : kblock;    // query or key blocks
  const int blk = static_cast<int>(cta % nbx);
  const long long bh = cta / nbx;                // b*H + h
  const T *X = is_q ? Q : K;
  float *out_mean = is_q ? q_mean : k_mean;
  float *out_var = is_q ? q_var : k_var;

  const int row0 = blk * bsize;
  const int n_rows = min(bsize, N - row0);
  const int tid = threadIdx.x;
  const int col = tid % COLS;
  const int rsub = tid / COLS;
  const T *base = X + (bh * N_alloc + row0) * static_cast<long long>(D) + col * VEC;

  uint4 v[RPT];
#pragma unroll
  for (int k = 0; k < RPT; ++k) {
    const int r = rsub + k * RPP;
    if (r < n_rows) {
      v[k] = __ldg(reinterpret_cast<const uint4 *>(base + static_cast<long long>(r) * D));
    } else {
      v[k] = make_uint4(0, 0, 0, 0);
    }
  }

  // pass 1: sum
  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
#pragma unroll
  for (int k = 0; k < RPT; ++k) {
    float f[VEC];
    Elem<T>::unpack(v[k], f);
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] += f[e];
  }
#pragma unroll
  for (int e = 0; e < VEC; ++e) red[rsub][col * VEC + e] = acc[e];
  __syncthreads();
  const float inv_n = 1.f / static_cast<float>(n_rows);
  if (tid < D) {
    float s = 0.f;
#pragma unroll 8
    for (int r = 0; r < RPP; ++r) s += red[r][tid];
    mean_s[tid] = s * inv_n;
  }
  __syncthreads();

  // pass 2: centred sum of squares over the same registers
  float mu[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    mu[e] = mean_s[col * VEC + e];
    acc[e] = 0.f;
  }
#pragma unroll
  for (int k = 0; k < RPT; ++k) {
    const int r = rsub + k * RPP;
    if (r < n_rows) {
      float f[VEC];
      Elem<T>::unpack(v[k], f);
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const float dv = f[e] - mu[e];
        acc[e] = fmaf(dv, dv, acc[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < VEC; ++e) red[rsub][col * VEC + e] = acc[e];
  __syncthreads();
  if (tid < D) {
    float s = 0.f;
#pragma unroll 8
    for (int r = 0; r < RPP; ++r) s += red[r][tid];
    const long long o = (bh * nbx + blk) * static_cast<long long>(D) + tid;
    out_mean[o] = mean_s[tid];
    out_var[o] = s * inv_n;
  }
}

// Streaming variant for blocks of at most 32 KB (every bf16 d=128 shape up to
// block 128): a persistent CTA walks the (head, block) items with a stride of
// the grid size; each item is one contiguous slab of rows, fetched with a
// single bulk copy (cp.async.bulk) into a 3-stage shared-memory ring, so that
// three slabs per CTA are in flight while the current one is reduced.
//
// The reduction takes one CTA barrier per item. Each thread reduces its own
// rows exactly (two passes over registers: local sum S_t, then the centred
// second moment M2_t about S_t / n_t); the lanes of a warp that share columns
// are merged with shuffles, and the 8 warp partials of a column are merged by
// one thread after the barrier, using the pairwise update for centred moments
// (Chan, Golub and LeVeque, "Algorithms for computing the sample variance"):
//   n = na + nb,  S = Sa + Sb,  M2 = M2a + M2b + (Sa/na - Sb/nb)^2 na nb / n.
// The partials are double-buffered, so the same barrier that publishes this
// item's partials also frees the ring stage and the other partial buffer.
constexpr int kStatsStages = 3;
constexpr uint32_t kStatsStageBytes = 32768;
constexpr int kStatsWarps = kStatsThreads / 32;

// Valid rows among r = rsub + k*rpp (k < rpt) of a block with n_rows rows.
__device__ __forceinline__ int stats_rows_of(int rsub, int rpp, int rpt, int n_rows) {
  return n_rows > rsub ? min(rpt, (n_rows - rsub + rpp - 1) / rpp) : 0;
}

// Moments of this thread's rows (r = rsub + k*RPP) of a complete block, with
// the packed .f32x2 instructions (two columns per instruction), then merged
// over the lanes of the warp that hold the same columns. Every count is a
// compile-time constant here.
template <typename T, int D>
__device__ __forceinline__ void stats_moments_full(const T *slab, int rsub, int col, float (&ps)[Elem<T>::kVec],
                                                   float (&pm2)[Elem<T>::kVec]) {
  constexpr int VEC = Elem<T>::kVec, P = VEC / 2;
  constexpr int COLS = D / VEC, RPP = kStatsThreads / COLS;
  constexpr int RPT = static_cast<int>(kStatsStageBytes / (D * sizeof(T))) / RPP;
  uint64_t x[RPT][P];
#pragma unroll
  for (int k = 0; k < RPT; ++k)
    Elem<T>::unpack2(*reinterpret_cast<const uint4 *>(slab + (rsub + k * RPP) * D + col * VEC), x[k]);
  const float inv = 1.f / static_cast<float>(RPT);
  const uint64_t neg_inv2 = pack_f32x2(-inv, -inv), zero2 = pack_f32x2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < P; ++i) {
    uint64_t s2 = x[0][i];
#pragma unroll
    for (int k = 1; k < RPT; ++k) s2 = add_f32x2(s2, x[k][i]);
    const uint64_t neg_mu = fma_f32x2(s2, neg_inv2, zero2);
    uint64_t q2 = zero2;
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
      const uint64_t dv = add_f32x2(x[k][i], neg_mu);
      q2 = fma_f32x2(dv, dv, q2);
    }
    ps[2 * i] = lo_f32(s2);
    ps[2 * i + 1] = hi_f32(s2);
    pm2[2 * i] = lo_f32(q2);
    pm2[2 * i + 1] = hi_f32(q2);
  }
  int na = RPT;
#pragma unroll
  for (int off = COLS; off < 32; off <<= 1) {    // equal counts: M2 += (Sa - Sb)^2 / (2 na)
    const float c = 0.5f / static_cast<float>(na);
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const float sb = __shfl_xor_sync(0xFFFFFFFFu, ps[e], off);
      const float mb = __shfl_xor_sync(0xFFFFFFFFu, pm2[e], off);
      const float dm = ps[e] - sb;
      pm2[e] = fmaf(dm * dm, c, pm2[e] + mb);
      ps[e] += sb;
    }
    na *= 2;
  }
}

// The same for the last, partly filled block of a head: rows at or beyond
// n_rows are left out of every count.
template <typename T, int D>
__device__ __forceinline__ void stats_moments_ragged(const T *slab, int n_rows, int rsub, int col,
                                                  float (&ps)[Elem<T>::kVec], float (&pm2)[Elem<T>::kVec]) {
  constexpr int VEC = Elem<T>::kVec;
  constexpr int COLS = D / VEC, RPP = kStatsThreads / COLS;
  constexpr int RPT = static_cast<int>(kStatsStageBytes / (D * sizeof(T))) / RPP;
  float f[RPT][VEC];
#pragma unroll
  for (int k = 0; k < RPT; ++k) {
    const int r = rsub + k * RPP;
    const uint4 v = r < n_rows ? *reinterpret_cast<const uint4 *>(slab + r * D + col * VEC) : make_uint4(0, 0, 0, 0);
    Elem<T>::unpack(v, f[k]);
  }
  const int nt = stats_rows_of(rsub, RPP, RPT, n_rows);
  const float inv_nt = nt > 0 ? 1.f / static_cast<float>(nt) : 0.f;
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    float a = 0.f;
#pragma unroll
    for (int k = 0; k < RPT; ++k) a += f[k][e];              // padded rows hold 0
    ps[e] = a;
    const float mu = a * inv_nt;
    float q = 0.f;
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
      const float dv = f[k][e] - mu;
      q = (rsub + k * RPP < n_rows) ? fmaf(dv, dv, q) : q;
    }
    pm2[e] = q;
  }
  int na = nt;
#pragma unroll
  for (int off = COLS; off < 32; off <<= 1) {
    const int nb_ = __shfl_xor_sync(0xFFFFFFFFu, na, off);
    const int n = na + nb_;
    const float ia = na > 0 ? 1.f / static_cast<float>(na) : 0.f;
    const float ib = nb_ > 0 ? 1.f / static_cast<float>(nb_) : 0.f;
    const float c = (na > 0 && nb_ > 0) ? static_cast<float>(na) * static_cast<float>(nb_) / static_cast<float>(n)
                                        : 0.f;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const float sb = __shfl_xor_sync(0xFFFFFFFFu, ps[e], off);
      const float mb = __shfl_xor_sync(0xFFFFFFFFu, pm2[e], off);
      const float dm = ps[e] * ia - sb * ib;
      pm2[e] = fmaf(dm * dm, c, pm2[e] + mb);
      ps[e] += sb;
    }
    na = n;
  }
}

// Optional output of the statistics pass: the augmented score features of
// every block, so that the score GEMM reads them instead of deriving them per
// tile. Plane p2 = 2p + h holds part p (0..2) as bf16, h = 0 the high and
// h = 1 the low half of x = hi + lo (hi = RN(x), lo = RN(x - hi)); a plane is
// [rows][D] with rows = B*H*nb, Q and K in separate arrays:
//   Q parts: s*mean, (s^2/2)*var, (s^2/2)*mean*mean
//   K parts: mean, mean*mean + var, var
struct FeatOut {
  __nv_bfloat16 *q, *k;        // nullptr: no feature output
  float s, hs2;                // sm_scale and 0.5 * sm_scale * sm_scale
  long long q_rows, k_rows;    // rows per plane
};

__device__ __forceinline__ void store_feat(__nv_bfloat16 *base, long long plane_elems, long long at, float x0, float x1,
                                           float x2) {
  const float x[3] = {x0, x1, x2};
#pragma unroll
  for (int p = 0; p < 3; ++p) {
    const __nv_bfloat16 hi = __float2bfloat16_rn(x[p]);
    const __nv_bfloat16 lo = __float2bfloat16_rn(x[p] - __bfloat162float(hi));
    base[(2 * p) * plane_elems + at] = hi;
    base[(2 * p + 1) * plane_elems + at] = lo;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kStatsThreads, 2)
    stats_bulk_kernel(const T *__restrict__ Q, const T *__restrict__ K, float *__restrict__ q_mean,
                      float *__restrict__ q_var, float *__restrict__ k_mean, float *__restrict__ k_var, int B,
                      int Hq, int Hkv, int N, int N_alloc, int block, int nb, int kblock, int nbk,
                      FeatOut feat) {
  constexpr int VEC = Elem<T>::kVec;
  constexpr int COLS = D / VEC;                     // threads per row (16-byte vectors)
  constexpr int RPP = kStatsThreads / COLS;         // rows per pass of the CTA
  constexpr int RPT = static_cast<int>(kStatsStageBytes / (D * sizeof(T))) / RPP;
  constexpr int RPW = 32 / COLS;                    // row subsets (rsub values) per warp
  static_assert(COLS <= 32 && 32 % COLS == 0, "a row must map onto whole lanes of a warp");
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ float part_s[2][kStatsWarps][D];
  __shared__ float part_m2[2][kStatsWarps][D];
  __shared__ uint64_t full[kStatsStages];
  __shared__ int abort_flag;
  // the decoded item of each ring stage, written by the issuing thread before
  // its expect_tx arrive (release) and read after the full wait (acquire)
  __shared__ long long meta_orow[kStatsStages];
  __shared__ int meta_rows[kStatsStages];

  const long long n_q = static_cast<long long>(B) * Hq * nb;
  const long long total = n_q + static_cast<long long>(B) * Hkv * nbk;
  const int tid = threadIdx.x, col = tid % COLS, rsub = tid / COLS, warp = tid >> 5;
  const uint32_t ring = smem_u32(stage_mem);

  // item w -> source slab, valid rows, output row offset, Q-or-K
  auto locate = [&](long long w, const T *&src, int &n_rows, long long &orow, bool &is_q) {
    is_q = w < n_q;
    const long long c = is_q ? w : w - n_q;
    const int nbx = is_q ? nb : nbk, bsize = is_q ? block : kblock;   // query or key blocks
    const int blk = static_cast<int>(c % nbx);
    const long long bh = c / nbx;
    src = (is_q ? Q : K) + (bh * N_alloc + static_cast<long long>(blk) * bsize) * D;
    n_rows = min(bsize, N - blk * bsize);
    orow = (bh * nbx + blk) * static_cast<long long>(D);
  };
  auto issue = [&](long long w, int s) {
    const T *src;
    int n_rows;
    long long orow;
    bool is_q;
    locate(w, src, n_rows, orow, is_q);
    const uint32_t bytes = static_cast<uint32_t>(n_rows) * D * sizeof(T);
    meta_orow[s] = is_q ? orow : -1 - orow;             // sign carries Q-or-K
    meta_rows[s] = n_rows;
    mbar_arrive_expect_tx(smem_u32(&full[s]), bytes);
#if BA_STATS_EVICT_FIRST
    // Q and K are read exactly once here: stream them through L2 at evict-first
    // priority so that lines still resident from earlier kernels (for example
    // an attention output not yet written back) are not displaced by them
    bulk_load_hint(ring + s * kStatsStageBytes, src, bytes, smem_u32(&full[s]), l2_evict_first_policy());
#else
    bulk_load(ring + s * kStatsStageBytes, src, bytes, smem_u32(&full[s]));
#endif
  };

  long long last_issued = -1;             // thread 0: newest item handed to the copy engine
  if (tid == 0) {
    for (int s = 0; s < kStatsStages; ++s) mbar_init(smem_u32(&full[s]), 1);
    abort_flag = 0;
    fence_mbar_init();
    for (int s = 0; s < kStatsStages; ++s) {
      const long long w = blockIdx.x + static_cast<long long>(s) * gridDim.x;
      if (w < total) {
        issue(w, s);
        last_issued = w;
      }
    }
  }
  __syncthreads();

  int it = 0;
  for (long long w = blockIdx.x; w < total; w += gridDim.x, ++it) {
    const int s = it % kStatsStages, pb = it & 1;
    const bool ok = mbar_wait_bounded(smem_u32(&full[s]), (it / kStatsStages) & 1, &abort_flag);
    const long long mo = meta_orow[s];
    const int n_rows = meta_rows[s];
    const bool is_q = mo >= 0;
    const long long orow = is_q ? mo : -1 - mo;

    // this thread's rows: exact local sum and centred second moment, merged
    // over the lanes of the warp that hold the same columns
    const T *slab = reinterpret_cast<const T *>(stage_mem + s * kStatsStageBytes);
    const bool full_block = n_rows == RPP * RPT;
    float ps[VEC], pm2[VEC];
    if (full_block) {
      stats_moments_full<T, D>(slab, rsub, col, ps, pm2);
    } else {
      stats_moments_ragged<T, D>(slab, n_rows, rsub, col, ps, pm2);
    }
    if ((tid & 31) < COLS) {
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        part_s[pb][warp][col * VEC + e] = ps[e];
        part_m2[pb][warp][col * VEC + e] = pm2[e];
      }
    }
    // one barrier: partials published, ring stage s consumed by every thread
    if (__syncthreads_or(!ok)) break;
    if (tid == 0) {
      const long long wn = w + static_cast<long long>(kStatsStages) * gridDim.x;
      if (wn < total) {
        fence_proxy_async_smem();             // the reads above before the bulk write
        issue(wn, s);
        last_issued = wn;
      }
    }
    if (tid < D) {
      float S = 0.f;
#pragma unroll
      for (int q = 0; q < kStatsWarps; ++q) S += part_s[pb][q][tid];
      float mean, M2 = 0.f;
      if (full_block) {                       // every warp holds RPW * RPT rows
        constexpr float kNw = static_cast<float>(RPW * RPT), kInvNw = 1.f / kNw;
        constexpr float kInvN = 1.f / static_cast<float>(RPP * RPT);
        mean = S * kInvN;
#pragma unroll
        for (int q = 0; q < kStatsWarps; ++q) {
          const float t = fmaf(-kNw, mean, part_s[pb][q][tid]);
          M2 += fmaf(t * t, kInvNw, part_m2[pb][q][tid]);
        }
        M2 *= kInvN;
      } else {
        mean = S / static_cast<float>(n_rows);
#pragma unroll
        for (int q = 0; q < kStatsWarps; ++q) {
          int nq = 0;
#pragma unroll
          for (int u = 0; u < RPW; ++u) nq += stats_rows_of(q * RPW + u, RPP, RPT, n_rows);
          const float t = fmaf(-static_cast<float>(nq), mean, part_s[pb][q][tid]);
          M2 += part_m2[pb][q][tid] + (nq > 0 ? t * t / static_cast<float>(nq) : 0.f);
        }
        M2 /= static_cast<float>(n_rows);
      }
      (is_q ? q_mean : k_mean)[orow + tid] = mean;
      (is_q ? q_var : k_var)[orow + tid] = M2;
      if (feat.q != nullptr) {
        if (is_q)
          store_feat(feat.q, feat.q_rows * D, orow + tid, __fmul_rn(feat.s, mean), __fmul_rn(feat.hs2, M2),
                     __fmul_rn(__fmul_rn(feat.hs2, mean), mean));
        else
          store_feat(feat.k, feat.k_rows * D, orow + tid, mean, __fmaf_rn(mean, mean, M2), M2);
      }
    }
  }
  // after an abandoned wait, let every issued copy land before exiting
  // (the newest kStatsStages items issued, each in its own stage)
  if (tid == 0 && abort_flag) {
    for (long long w = last_issued; w >= blockIdx.x && w > last_issued - kStatsStages * static_cast<long long>(gridDim.x);
         w -= gridDim.x) {
      const long long idx = (w - blockIdx.x) / gridDim.x;
      mbar_wait_bounded(smem_u32(&full[idx % kStatsStages]), (idx / kStatsStages) & 1, nullptr);
    }
  }
}

// One warp per block (the statistics pass of the one-copy path): the warp's
// lanes own D/32 columns each across all rows of the block, so no value
// crosses lanes and no barrier joins warps. Each lane accumulates, in fp32,
// the deviations d = x - c from the block's first row c (exact in fp32 for
// bf16 and small for fp32 inputs), S1 = sum d and S2 = sum d^2 over two
// interleaved accumulator sets; then
//   mean = c + S1/n,  var = (S2 - S1 * (S1/n)) / n   (clamped at 0).
// A column that does not vary gives d = 0 and a variance of exactly 0.
// Each warp double-buffers its own 32 KB bulk copies (two ring stages with
// their own mbarriers); kStatsWarpsPerCta warps share a CTA and its shared
// memory, one CTA per SM.
constexpr int kStatsWarpsPerCta = 3;
constexpr long long kStatsWarpMinBlocks = 16384;     // blocks of work from which the warp kernel is used

template <typename T, int D>
__global__ void __launch_bounds__(kStatsWarpsPerCta * 32, 1)
    stats_warp_kernel(const T *__restrict__ Q, const T *__restrict__ K, float *__restrict__ q_mean,
                      float *__restrict__ q_var, float *__restrict__ k_mean, float *__restrict__ k_var, int B,
                      int Hq, int Hkv, int N, int N_alloc, int block, int nb, int kblock, int nbk, FeatOut feat) {
  constexpr int E = D / 32;                         // columns per lane
  constexpr int P = E / 2;                          // packed fp32 pairs per lane
  constexpr int RB = D * static_cast<int>(sizeof(T));   // bytes per row
  static_assert(E == 2 || E == 4, "head dimension");
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ uint64_t full[kStatsWarpsPerCta][2];
  __shared__ long long meta_orow[kStatsWarpsPerCta][2];
  __shared__ int meta_rows[kStatsWarpsPerCta][2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ring = smem_u32(stage_mem) + static_cast<uint32_t>(warp) * 2u * kStatsStageBytes;
  const long long n_q = static_cast<long long>(B) * Hq * nb;
  const long long total = n_q + static_cast<long long>(B) * Hkv * nbk;
  const long long tw = static_cast<long long>(gridDim.x) * kStatsWarpsPerCta;
  const long long gw = static_cast<long long>(blockIdx.x) * kStatsWarpsPerCta + warp;
  const uint64_t policy = l2_evict_first_policy();

  // item w -> its slab (Q rows of a query block or K rows of a key block)
  auto issue = [&](long long w, int st) {
    const bool is_q = w < n_q;
    const long long c = is_q ? w : w - n_q;
    const int nbx = is_q ? nb : nbk, bsize = is_q ? block : kblock;
    const int blk = static_cast<int>(c % nbx);
    const long long bh = c / nbx;
    const T *src = (is_q ? Q : K) + (bh * N_alloc + static_cast<long long>(blk) * bsize) * D;
    const int n_rows = min(bsize, N - blk * bsize);
    const long long orow = (bh * nbx + blk) * static_cast<long long>(D);
    meta_orow[warp][st] = is_q ? orow : -1 - orow;   // sign carries Q-or-K
    meta_rows[warp][st] = n_rows;
    mbar_arrive_expect_tx(smem_u32(&full[warp][st]), static_cast<uint32_t>(n_rows) * RB);
    bulk_load_hint(ring + st * kStatsStageBytes, src, static_cast<uint32_t>(n_rows) * RB, smem_u32(&full[warp][st]),
                   policy);
  };

  long long issued = 0, consumed = 0;               // this warp's items handed to the copy engine / read
  if (lane == 0) {
    mbar_init(smem_u32(&full[warp][0]), 1);
    mbar_init(smem_u32(&full[warp][1]), 1);
    fence_mbar_init();
    for (int st = 0; st < 2; ++st)
      if (gw + st * tw < total) issue(gw + st * tw, st);
  }
  issued = (gw < total) + (gw + tw < total);
  __syncwarp();

  bool ok = true;
  for (long long w = gw; w < total; w += tw) {
    const int st = static_cast<int>(consumed & 1);
    const bool got = mbar_wait_bounded(smem_u32(&full[warp][st]), static_cast<uint32_t>((consumed >> 1) & 1), nullptr);
    if (!__all_sync(0xFFFFFFFFu, got)) {
      ok = false;
      break;
    }
    const long long mo = meta_orow[warp][st];
    const int n = meta_rows[warp][st];
    const bool is_q = mo >= 0;
    const long long orow = is_q ? mo : -1 - mo;
    const uint8_t *rows = stage_mem + (static_cast<size_t>(warp) * 2 + st) * kStatsStageBytes + lane * E * sizeof(T);

    // this lane's E columns of row r as P packed fp32 pairs
    auto row_pairs = [&](int r, uint64_t (&x)[P]) {
      const uint8_t *a = rows + static_cast<size_t>(r) * RB;
      if constexpr (sizeof(T) == 2) {
        if constexpr (E == 4) {
          const uint2 v = *reinterpret_cast<const uint2 *>(a);
          x[0] = pack_u32x2(v.x << 16, v.x & 0xFFFF0000u);
          x[1] = pack_u32x2(v.y << 16, v.y & 0xFFFF0000u);
        } else {
          const uint32_t v = *reinterpret_cast<const uint32_t *>(a);
          x[0] = pack_u32x2(v << 16, v & 0xFFFF0000u);
        }
      } else {
        if constexpr (E == 4) {
          const uint4 v = *reinterpret_cast<const uint4 *>(a);
          x[0] = pack_u32x2(v.x, v.y);
          x[1] = pack_u32x2(v.z, v.w);
        } else {
          const uint2 v = *reinterpret_cast<const uint2 *>(a);
          x[0] = pack_u32x2(v.x, v.y);
        }
      }
    };
    uint64_t c[P], nc[P], s1[2][P], s2[2][P];
    row_pairs(0, c);
#pragma unroll
    for (int i = 0; i < P; ++i) {
      nc[i] = pack_f32x2(-lo_f32(c[i]), -hi_f32(c[i]));
      s1[0][i] = s1[1][i] = s2[0][i] = s2[1][i] = 0ull;       // +0.0f pairs
    }
    int r = 1;
#pragma unroll 4
    for (; r + 1 < n; r += 2) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint64_t x[P];
        row_pairs(r + h, x);
#pragma unroll
        for (int i = 0; i < P; ++i) {
          const uint64_t d = add_f32x2(x[i], nc[i]);
          s1[h][i] = add_f32x2(s1[h][i], d);
          s2[h][i] = fma_f32x2(d, d, s2[h][i]);
        }
      }
    }
    if (r < n) {
      uint64_t x[P];
      row_pairs(r, x);
#pragma unroll
      for (int i = 0; i < P; ++i) {
        const uint64_t d = add_f32x2(x[i], nc[i]);
        s1[0][i] = add_f32x2(s1[0][i], d);
        s2[0][i] = fma_f32x2(d, d, s2[0][i]);
      }
    }
    __syncwarp();                                   // every lane is done with this stage
    ++consumed;
    if (lane == 0 && w + 2 * tw < total) {
      fence_proxy_async_smem();                     // the reads above before the bulk write
      issue(w + 2 * tw, st);
    }
    if (w + 2 * tw < total) ++issued;

    const float inv_n = 1.f / static_cast<float>(n);
    float mean[E], var[E];
#pragma unroll
    for (int i = 0; i < P; ++i) {
      const uint64_t S1 = add_f32x2(s1[0][i], s1[1][i]), S2 = add_f32x2(s2[0][i], s2[1][i]);
      const float a1[2] = {lo_f32(S1), hi_f32(S1)}, a2[2] = {lo_f32(S2), hi_f32(S2)};
      const float cc[2] = {lo_f32(c[i]), hi_f32(c[i])};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float md = a1[e] * inv_n;
        mean[2 * i + e] = cc[e] + md;
        var[2 * i + e] = fmaxf(fmaf(-a1[e], md, a2[e]) * inv_n, 0.f);
      }
    }
    float *om = (is_q ? q_mean : k_mean) + orow + lane * E;
    float *ov = (is_q ? q_var : k_var) + orow + lane * E;
    if constexpr (E == 4) {
      *reinterpret_cast<float4 *>(om) = make_float4(mean[0], mean[1], mean[2], mean[3]);
      *reinterpret_cast<float4 *>(ov) = make_float4(var[0], var[1], var[2], var[3]);
    } else {
      *reinterpret_cast<float2 *>(om) = make_float2(mean[0], mean[1]);
      *reinterpret_cast<float2 *>(ov) = make_float2(var[0], var[1]);
    }
    if (feat.q != nullptr) {
      // the lane's E columns of each plane packed into one store: a warp
      // writes each plane's D contiguous values at once
      float x[3][E];
#pragma unroll
      for (int e = 0; e < E; ++e) {
        if (is_q) {
          x[0][e] = __fmul_rn(feat.s, mean[e]);
          x[1][e] = __fmul_rn(feat.hs2, var[e]);
          x[2][e] = __fmul_rn(__fmul_rn(feat.hs2, mean[e]), mean[e]);
        } else {
          x[0][e] = mean[e];
          x[1][e] = __fmaf_rn(mean[e], mean[e], var[e]);
          x[2][e] = var[e];
        }
      }
      __nv_bfloat16 *base = is_q ? feat.q : feat.k;
      const long long plane = (is_q ? feat.q_rows : feat.k_rows) * D;
#pragma unroll
      for (int pp = 0; pp < 3; ++pp) {
        uint32_t hw[E / 2], lw[E / 2];
#pragma unroll
        for (int e = 0; e < E; e += 2) {
          const __nv_bfloat16 h0 = __float2bfloat16_rn(x[pp][e]), h1 = __float2bfloat16_rn(x[pp][e + 1]);
          const __nv_bfloat16 l0 = __float2bfloat16_rn(x[pp][e] - __bfloat162float(h0));
          const __nv_bfloat16 l1 = __float2bfloat16_rn(x[pp][e + 1] - __bfloat162float(h1));
          hw[e / 2] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
                      (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
          lw[e / 2] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) |
                      (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
        }
        __nv_bfloat16 *ph = base + (2 * pp) * plane + orow + lane * E;
        __nv_bfloat16 *pl = base + (2 * pp + 1) * plane + orow + lane * E;
        if constexpr (E == 4) {
          *reinterpret_cast<uint2 *>(ph) = make_uint2(hw[0], hw[1]);
          *reinterpret_cast<uint2 *>(pl) = make_uint2(lw[0], lw[1]);
        } else {
          *reinterpret_cast<uint32_t *>(ph) = hw[0];
          *reinterpret_cast<uint32_t *>(pl) = lw[0];
        }
      }
    }
  }
  // after an abandoned wait, let this warp's copies in flight land first
  if (!ok && lane == 0) {
    for (long long u = consumed; u < issued; ++u)
      mbar_wait_bounded(smem_u32(&full[warp][u & 1]), static_cast<uint32_t>((u >> 1) & 1), nullptr);
  }
}

// Rows each thread holds for a given block size (power-of-two bucket).
template <typename T, int D>
inline int stats_rpt_needed(int block) {
  constexpr int RPP = kStatsThreads / (D / Elem<T>::kVec);
  return (block + RPP - 1) / RPP;
}

// Whether the one-copy-per-block kernel (the one that can also write the
// score features) serves this block size.
template <typename T, int D>
constexpr bool stats_bulk_fits(int block) {
  return static_cast<size_t>(block) * D * sizeof(T) <= kStatsStageBytes;
}

template <typename T, int D>
cudaError_t launch_stats(const T *Q, const T *K, float *qm, float *qv, float *km, float *kv, int B, int Hq, int Hkv,
                         int N, int N_alloc, int block, int kblock, int num_sms, cudaStream_t stream,
                         FeatOut feat = FeatOut{nullptr, nullptr, 0.f, 0.f, 0, 0}) {
  const int nb = (N + block - 1) / block, nbk = (N + kblock - 1) / kblock;
  const long long grid = static_cast<long long>(B) * Hq * nb + static_cast<long long>(B) * Hkv * nbk;
  const int bmax = block > kblock ? block : kblock;
  // The warp-per-block kernel has no cross-warp merge and reaches ~0.97 of
  // HBM on long runs (128K: 40960 blocks); below ~16K blocks its three warps
  // per SM ramp up and drain more slowly than the CTA-per-block kernel.
  if (stats_bulk_fits<T, D>(bmax) && grid >= kStatsWarpMinBlocks) {
    const size_t smem = static_cast<size_t>(kStatsWarpsPerCta) * 2 * kStatsStageBytes;
    cudaError_t e = cudaFuncSetAttribute(stats_warp_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const long long warps = (grid + 0);                 // one warp per block
    const long long ctas_needed = (warps + kStatsWarpsPerCta - 1) / kStatsWarpsPerCta;
    const unsigned g = static_cast<unsigned>(ctas_needed < num_sms ? ctas_needed : num_sms);
    stats_warp_kernel<T, D><<<g, kStatsWarpsPerCta * 32, smem, stream>>>(Q, K, qm, qv, km, kv, B, Hq, Hkv, N, N_alloc,
                                                                       block, nb, kblock, nbk, feat);
    return cudaGetLastError();
  }
  if (stats_bulk_fits<T, D>(bmax)) {
    const size_t smem = static_cast<size_t>(kStatsStages) * kStatsStageBytes;
    cudaError_t e = cudaFuncSetAttribute(stats_bulk_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, stats_bulk_kernel<T, D>, kStatsThreads, smem);
    if (e != cudaSuccess) return e;
    const long long persistent = static_cast<long long>(num_sms) * (per_sm > 0 ? per_sm : 1);
    const unsigned g = static_cast<unsigned>(grid < persistent ? grid : persistent);
    stats_bulk_kernel<T, D><<<g, kStatsThreads, smem, stream>>>(Q, K, qm, qv, km, kv, B, Hq, Hkv, N, N_alloc, block,
                                                                 nb, kblock, nbk, feat);
    return cudaGetLastError();
  }
  if (feat.q != nullptr) return cudaErrorInvalidValue;    // features only from the one-copy kernel
  const int need = stats_rpt_needed<T, D>(bmax);
  dim3 g(static_cast<unsigned>(grid));
  if (need <= 2) {
    stats_kernel<T, D, 2><<<g, kStatsThreads, 0, stream>>>(Q, K, qm, qv, km, kv, B, Hq, Hkv, N, N_alloc, block, nb,
                                                              kblock, nbk);
  } else if (need <= 4) {
    stats_kernel<T, D, 4><<<g, kStatsThreads, 0, stream>>>(Q, K, qm, qv, km, kv, B, Hq, Hkv, N, N_alloc, block, nb,
                                                              kblock, nbk);
  } else if (need <= 8) {
    stats_kernel<T, D, 8><<<g, kStatsThreads, 0, stream>>>(Q, K, qm, qv, km, kv, B, Hq, Hkv, N, N_alloc, block, nb,
                                                              kblock, nbk);
  } else if (need <= 16) {
    stats_kernel<T, D, 16><<<g, kStatsThreads, 0, stream>>>(Q, K, qm, qv, km, kv, B, Hq, Hkv, N, N_alloc, block, nb,
                                                              kblock, nbk);
  } else {
    stats_kernel<T, D, 32><<<g, kStatsThreads, 0, stream>>>(Q, K, qm, qv, km, kv, B, Hq, Hkv, N, N_alloc, block, nb,
                                                              kblock, nbk);
  }
  return cudaGetLastError();
}

}  // namespace baatt
