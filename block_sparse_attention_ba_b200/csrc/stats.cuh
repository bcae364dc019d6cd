// stats.cuh — K6: per-block mean and diagonal (per-dimension) variance.
//
// Stage one of BA-Att pools Q and K block-wise before any scoring, and the
// covariance correction needs each block's per-dimension variance
// ("Efficient Long-Context Modeling in DLMs via Block Approximate Sparse
// Attention": abstract; "Core claim").
//
// One warp per (head, block) item, persistent over items, Q and K items in
// one launch (items [0, B*Hq*nq) are Q). The warp's lanes own D/32 columns
// each across all rows of the block, so no value crosses lanes and no
// barrier joins warps. Each lane accumulates, in fp32, the deviations
// d = x - c from the block's first row c (exact in fp32 for bf16 inputs and
// small for fp32 ones), S1 = sum d and S2 = sum d^2 over two accumulator sets
// (even rows, odd rows); then
//   mean = c + S1/n,  var = (S2 - S1 * (S1/n)) / n   (clamped at 0).
// A column that does not vary gives d = 0 and a variance of exactly 0.
//
// A block is streamed from HBM in chunks of 32 KB / SPLIT by cp.async.bulk
// (evict-first), each warp double-buffering its own chunks (two ring stages
// with their own mbarriers) in 192 KB of shared memory per CTA, one CTA of
// 3 * SPLIT warps per SM. The chunks of a block are consumed in row order
// and a chunk holds an even number of rows, so the sums do not depend on
// SPLIT or on the block size. Smaller chunks (SPLIT 4) give twelve warps per
// SM, which ramp up and drain faster on short runs; on long runs 32 KB
// chunks (SPLIT 1) keep fewer, longer streams in flight and reach ~0.97 of
// HBM. Once its first copies are issued, each CTA lets a programmatic
// dependent (the score GEMM of ba_att_selector) launch as SMs free up.
#pragma once

#include "common.cuh"
#include "pdl.cuh"

#ifndef BA_STATS_LONG_RUN_ITEMS
#define BA_STATS_LONG_RUN_ITEMS 16384
#endif

namespace baatt {

constexpr uint32_t kStatsStageBytes = 32768;          // shared memory per warp and ring stage at SPLIT 1
constexpr size_t kStatsSmem = 6 * static_cast<size_t>(kStatsStageBytes);   // 3 warps x 2 stages at SPLIT 1
constexpr long long kStatsLongRunItems = BA_STATS_LONG_RUN_ITEMS;   // from here on: 32 KB chunks

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

// Per-lane pieces of the statistics pass (stats_warp_kernel). A lane owns
// E = D/32 columns of a block, as P = E/2 packed fp32 pairs.
template <typename T, int D>
struct LaneStats {
  static constexpr int E = D / 32;
  static constexpr int P = E / 2;
  static constexpr int RB = D * static_cast<int>(sizeof(T));   // bytes per row
  uint64_t c[P], nc[P], s1[2][P], s2[2][P];

  // this lane's E columns of row r of a staged chunk as P packed fp32 pairs
  __device__ __forceinline__ static void row_pairs(const uint8_t *rows, int r, uint64_t (&x)[P]) {
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
  }

  __device__ __forceinline__ void clear() {
#pragma unroll
    for (int i = 0; i < P; ++i) c[i] = nc[i] = s1[0][i] = s1[1][i] = s2[0][i] = s2[1][i] = 0ull;
  }

  // Adds the nr rows of one staged chunk (rows: this lane's first column of
  // the chunk's row 0); the first chunk of a block also takes its first row
  // as the shift c. Rows go in pairs (even row -> set 0, odd row -> set 1;
  // the first row contributes exactly +0).
  __device__ __forceinline__ void add_chunk(const uint8_t *rows, int nr, bool first_chunk) {
    if (first_chunk) {
      row_pairs(rows, 0, c);
#pragma unroll
      for (int i = 0; i < P; ++i) {
        nc[i] = pack_f32x2(-lo_f32(c[i]), -hi_f32(c[i]));
        s1[0][i] = s1[1][i] = s2[0][i] = s2[1][i] = 0ull;     // +0.0f pairs
      }
    }
    int r = 0;
#pragma unroll 4
    for (; r + 1 < nr; r += 2) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint64_t x[P];
        row_pairs(rows, r + h, x);
#pragma unroll
        for (int i = 0; i < P; ++i) {
          const uint64_t d = add_f32x2(x[i], nc[i]);
          s1[h][i] = add_f32x2(s1[h][i], d);
          s2[h][i] = fma_f32x2(d, d, s2[h][i]);
        }
      }
    }
    if (r < nr) {
      uint64_t x[P];
      row_pairs(rows, r, x);
#pragma unroll
      for (int i = 0; i < P; ++i) {
        const uint64_t d = add_f32x2(x[i], nc[i]);
        s1[0][i] = add_f32x2(s1[0][i], d);
        s2[0][i] = fma_f32x2(d, d, s2[0][i]);
      }
    }
  }

  // mean = c + S1/n, var = (S2 - S1*(S1/n))/n clamped at 0, for a block of n rows
  __device__ __forceinline__ void finish(int n, float (&mean)[E], float (&var)[E]) const {
    const float inv_n = 1.f / static_cast<float>(n);
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
  }
};

// Writes one lane's E columns of a block's mean and variance (at element
// offset orow + lane*E of the mean/var arrays) and, with feat.q set, the
// block's augmented score features (the lane's columns of each plane packed
// into one store, so a warp writes each plane's D contiguous values at once).
template <int D>
__device__ __forceinline__ void write_block_stats(bool is_q, long long orow, int lane, const float (&mean)[D / 32],
                                                  const float (&var)[D / 32], float *q_mean, float *q_var,
                                                  float *k_mean, float *k_var, const FeatOut &feat) {
  constexpr int E = D / 32;
  float *om = (is_q ? q_mean : k_mean) + orow + lane * E;
  float *ov = (is_q ? q_var : k_var) + orow + lane * E;
  if constexpr (E == 4) {
    *reinterpret_cast<float4 *>(om) = make_float4(mean[0], mean[1], mean[2], mean[3]);
    *reinterpret_cast<float4 *>(ov) = make_float4(var[0], var[1], var[2], var[3]);
  } else {
    *reinterpret_cast<float2 *>(om) = make_float2(mean[0], mean[1]);
    *reinterpret_cast<float2 *>(ov) = make_float2(var[0], var[1]);
  }
  if (feat.q == nullptr) return;
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

template <typename T, int D, int SPLIT>
__global__ void __launch_bounds__(3 * SPLIT * 32, 1)
    stats_warp_kernel(const T *__restrict__ Q, const T *__restrict__ K, float *__restrict__ q_mean,
                      float *__restrict__ q_var, float *__restrict__ k_mean, float *__restrict__ k_var, int B,
                      int Hq, int Hkv, int N, int N_alloc, int block, int nb, int kblock, int nbk, FeatOut feat) {
  static_assert(SPLIT == 1 || SPLIT == 2 || SPLIT == 4, "chunks per 32 KB");
  constexpr int E = D / 32;                         // columns per lane
  constexpr int RB = D * static_cast<int>(sizeof(T));   // bytes per row
  constexpr int W = 3 * SPLIT;                      // warps per CTA
  constexpr uint32_t CB = kStatsStageBytes / SPLIT; // bytes per chunk
  constexpr int CR = static_cast<int>(CB) / RB;     // rows per chunk
  static_assert(E == 2 || E == 4, "head dimension");
  static_assert(CR >= 2 && CR % 2 == 0, "a chunk holds an even number of rows");
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ uint64_t full[W][2];
  __shared__ long long meta_orow[W][2];
  __shared__ int meta_rows[W][2];
  __shared__ int meta_chunk[W][2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ring = smem_u32(stage_mem) + static_cast<uint32_t>(warp) * 2u * CB;
  const long long n_q = static_cast<long long>(B) * Hq * nb;
  const long long total = n_q + static_cast<long long>(B) * Hkv * nbk;
  const long long tw = static_cast<long long>(gridDim.x) * W;
  const uint64_t policy = l2_evict_first_policy();

  // the next chunk to hand to the copy engine: item iw (Q rows of a query
  // block or K rows of a key block), chunk ic of it; every lane keeps the
  // same cursor, lane 0 issues
  long long iw = static_cast<long long>(blockIdx.x) * W + warp;
  int ic = 0;
  const T *isrc = nullptr;
  long long iorow = 0;                              // output row offset; the sign carries Q-or-K
  int irows = 0;
  auto load_item = [&]() {
    if (iw >= total) return;
    const bool is_q = iw < n_q;
    const long long c = is_q ? iw : iw - n_q;
    const int nbx = is_q ? nb : nbk, bsize = is_q ? block : kblock;
    const int blk = static_cast<int>(c % nbx);
    const long long bh = c / nbx;
    isrc = (is_q ? Q : K) + (bh * N_alloc + static_cast<long long>(blk) * bsize) * D;
    irows = min(bsize, N - blk * bsize);
    const long long orow = (bh * nbx + blk) * static_cast<long long>(D);
    iorow = is_q ? orow : -1 - orow;
  };
  auto issue_next = [&](int st) -> int {
    if (iw >= total) return 0;
    const int r0 = ic * CR, nr = min(CR, irows - r0);
    if (lane == 0) {
      meta_orow[warp][st] = iorow;
      meta_rows[warp][st] = irows;
      meta_chunk[warp][st] = ic;
      mbar_arrive_expect_tx(smem_u32(&full[warp][st]), static_cast<uint32_t>(nr) * RB);
      bulk_load_hint(ring + st * CB, isrc + static_cast<long long>(r0) * D,
                     static_cast<uint32_t>(nr) * RB, smem_u32(&full[warp][st]), policy);
    }
    if (r0 + CR >= irows) {
      iw += tw;
      ic = 0;
      load_item();
    } else {
      ++ic;
    }
    return 1;
  };

  long long issued = 0, consumed = 0;               // this warp's chunks handed to the copy engine / read
  if (lane == 0) {
    mbar_init(smem_u32(&full[warp][0]), 1);
    mbar_init(smem_u32(&full[warp][1]), 1);
    fence_mbar_init();
  }
  __syncwarp();
  load_item();
  issued += issue_next(0);
  issued += issue_next(1);
  pdl_allow_dependents();                           // the score GEMM may launch as SMs free up

  LaneStats<T, D> acc;
  acc.clear();
  bool ok = true;
  while (consumed < issued) {
    const int st = static_cast<int>(consumed & 1);
    const bool got = mbar_wait_bounded(smem_u32(&full[warp][st]), static_cast<uint32_t>((consumed >> 1) & 1), nullptr);
    if (!__all_sync(0xFFFFFFFFu, got)) {
      ok = false;
      break;
    }
    const long long mo = meta_orow[warp][st];
    const int n = meta_rows[warp][st];
    const int r0 = meta_chunk[warp][st] * CR;
    const int nr = min(CR, n - r0);
    const bool is_q = mo >= 0;
    const long long orow = is_q ? mo : -1 - mo;
    const uint8_t *rows = stage_mem + (static_cast<size_t>(warp) * 2 + st) * CB + lane * E * sizeof(T);
    acc.add_chunk(rows, nr, r0 == 0);              // a new block: its first row is the shift
    __syncwarp();                                   // every lane is done with this stage
    ++consumed;
    if (lane == 0 && iw < total) fence_proxy_async_smem();   // the reads above before the bulk write
    issued += issue_next(st);
    if (r0 + nr < n) continue;                      // the block goes on in the next chunk

    float mean[E], var[E];
    acc.finish(n, mean, var);
    write_block_stats<D>(is_q, orow, lane, mean, var, q_mean, q_var, k_mean, k_var, feat);
  }
  // after an abandoned wait, let this warp's copies in flight land first
  if (!ok && lane == 0) {
    for (long long u = consumed; u < issued; ++u)
      mbar_wait_bounded(smem_u32(&full[warp][u & 1]), static_cast<uint32_t>((u >> 1) & 1), nullptr);
  }
}


template <typename T, int D, int SPLIT>
cudaError_t launch_stats_split(const T *Q, const T *K, float *qm, float *qv, float *km, float *kv, int B, int Hq,
                               int Hkv, int N, int N_alloc, int block, int nb, int kblock, int nbk, long long items,
                               int num_sms, cudaStream_t stream, FeatOut feat) {
  constexpr int W = 3 * SPLIT;
  const cudaError_t e = cudaFuncSetAttribute(stats_warp_kernel<T, D, SPLIT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kStatsSmem));
  if (e != cudaSuccess) return e;
  const long long ctas = (items + W - 1) / W;
  const unsigned g = static_cast<unsigned>(ctas < num_sms ? ctas : num_sms);
  stats_warp_kernel<T, D, SPLIT><<<g, W * 32, kStatsSmem, stream>>>(Q, K, qm, qv, km, kv, B, Hq, Hkv, N, N_alloc,
                                                                    block, nb, kblock, nbk, feat);
  return cudaGetLastError();
}

// Statistics of every Q and K block, optionally with the score features.
template <typename T, int D>
cudaError_t launch_stats(const T *Q, const T *K, float *qm, float *qv, float *km, float *kv, int B, int Hq, int Hkv,
                         int N, int N_alloc, int block, int kblock, int num_sms, cudaStream_t stream,
                         FeatOut feat = FeatOut{nullptr, nullptr, 0.f, 0.f, 0, 0}) {
  const int nb = (N + block - 1) / block, nbk = (N + kblock - 1) / kblock;
  const long long items = static_cast<long long>(B) * Hq * nb + static_cast<long long>(B) * Hkv * nbk;
  if (items >= kStatsLongRunItems)
    return launch_stats_split<T, D, 1>(Q, K, qm, qv, km, kv, B, Hq, Hkv, N, N_alloc, block, nb, kblock, nbk, items,
                                       num_sms, stream, feat);
  return launch_stats_split<T, D, 4>(Q, K, qm, qv, km, kv, B, Hq, Hkv, N, N_alloc, block, nb, kblock, nbk, items,
                                     num_sms, stream, feat);
}

}  // namespace baatt
