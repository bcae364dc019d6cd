// select_tc.cuh — K7 on the tensor cores: covariance-compensated block
// scores as a tiled tcgen05 GEMM; the exact per-row top-k follows as its own
// launch (topk_rows_kernel in select.cuh).
//
// Operator ("Efficient Long-Context Modeling in DLMs via Block Approximate
// Sparse Attention": abstract; "Core claim"; Figure 2):
//   S~[i,j] = qt_i . kt_j + ln m_j, summed over 3d augmented features
//   qt_i = [ s qbar_i , (s^2/2) vq_i , (s^2/2) qbar_i^2 ]
//   kt_j = [ kbar_j , kbar_j^2 + vk_j , vk_j ]
// ranked per query block, ties to the lower key block, top k kept ascending.
//
// One CTA = one (batch, head) x 128 query blocks (MMA M, the TMEM lanes) x NT
// key blocks (MMA N, 64 or 128 TMEM columns): grid (ceil(nq/128) *
// ceil(nk/NT), Hq, B), which covers any nq, nk up to the host limit.
//  - The feature order inside the 3d-long dot product is free, so the
//    features are taken in groups of 64 dimensions: one read of the fp32
//    statistics for dimensions [64g, 64g+64) yields all three feature parts
//    of that group, written as three 64-wide K slices.
//  - fp32-level accuracy on bf16 tensor cores: every operand is split
//    x = hi + lo (two bf16s, 16 significant bits) and S accumulates
//    hi*hi + hi*lo + lo*hi in fp32 (the dropped lo*lo is ~2^-16 relative).
//  - Operands go straight from registers into the 128-byte-swizzled K-major
//    shared-memory layout; one thread issues the MMAs and commits to an
//    mbarrier. The statistics of the next group are loaded into registers
//    before that mbarrier is waited on, so the loads overlap the MMAs.
//  - The fp32 scores are read from TMEM (warp w: lane quadrant w%4, a quarter
//    of the columns) and stored straight to the score map, ln m_j added.
#pragma once

#include "common.cuh"
#include "pdl.cuh"
#include "select.cuh"

namespace baatt {
namespace seltc {

constexpr int kThreads = 512;
constexpr int kRows = 128;                              // query blocks per tile
constexpr uint32_t kABytes = kRows * 128;               // 128 rows x 64 bf16
template <int NT>
struct Tile {
  static constexpr uint32_t kBBytes = NT * 128;         // NT rows x 64 bf16
  static constexpr uint32_t kPart = 2 * kABytes + 2 * kBBytes;
  static constexpr uint32_t kDynSmem = 3 * kPart + 1024;
  static constexpr int kTasksPerThread = (kRows + NT) * 8 / kThreads;
  static_assert((kRows + NT) * 8 % kThreads == 0, "tasks must split evenly over the threads");
  static_assert((kRows * 8) % kThreads == 0, "A and B tasks must not share an iteration");
};

// x = hi + lo for 8 consecutive values, hi = RN_bf16(x), lo = RN_bf16(x - hi).
__device__ __forceinline__ void split8(const float (&x)[8], uint4 &hi, uint4 &lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    h[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
    const float h0 = __uint_as_float(h[e] << 16), h1 = __uint_as_float(h[e] & 0xFFFF0000u);
    l[e] = pack_bf16x2(x[2 * e] - h0, x[2 * e + 1] - h1);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Byte offset of 16-byte chunk c (0..7) of row r in a 128B-swizzled tile.
__device__ __forceinline__ uint32_t sw128(int r, int c) {
  return static_cast<uint32_t>(r) * 128u + (static_cast<uint32_t>(c ^ (r & 7)) << 4);
}

// The 8 fp32 means and 8 variances of one 8-dimension chunk.
struct Raw {
  float4 m0, m1, v0, v1;
};

template <int D, int NT>
__global__ void __launch_bounds__(kThreads, 1)
    select_tc_kernel(const float *__restrict__ q_mean, const float *__restrict__ q_var,
                     const float *__restrict__ k_mean, const float *__restrict__ k_var,
                     float *__restrict__ block_scores, int Hq, int Hkv, int N, int kblock, int nq, int nk,
                     float sm_scale, int var_product) {
  using TL = Tile<NT>;
  constexpr int GROUPS = D / 64;
  constexpr int TPT = TL::kTasksPerThread;
  constexpr int COLS_PER_WARP = NT / 4;
  extern __shared__ uint8_t dyn_smem[];
  __shared__ uint64_t mma_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_flag;
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nk_tiles = (nk + NT - 1) / NT;
  const int h = blockIdx.y, b = blockIdx.z, g_kv = h / (Hq / Hkv);
  const long long bh = static_cast<long long>(b) * Hq + h;
  const int i0 = static_cast<int>(blockIdx.x / nk_tiles) * kRows, j0 = static_cast<int>(blockIdx.x % nk_tiles) * NT;
  const float s = sm_scale, hs2 = 0.5f * sm_scale * sm_scale;
  const float *qm = q_mean + bh * nq * D;
  const float *qv = q_var + bh * nq * D;
  const float *km = k_mean + (static_cast<long long>(b) * Hkv + g_kv) * nk * D;
  const float *kv = k_var + (static_cast<long long>(b) * Hkv + g_kv) * nk * D;

  if (tid == 0) {
    mbar_init(smem_u32(&mma_bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc<NT>(smem_u32(&tmem_base_s));
    tmem_relinquish();
  }

  // task e = it * kThreads + tid: rows [0,128) are query blocks (A), the
  // next NT rows key blocks (B); chunk e % 8 covers 8 of the group's 64 dims
  auto load_group = [&](int grp, Raw (&raw)[TPT]) {
#pragma unroll
    for (int it = 0; it < TPT; ++it) {
      const int e = it * kThreads + tid;
      const int c = e & 7;
      const bool is_a = e < kRows * 8;
      const int r = is_a ? (e >> 3) : ((e - kRows * 8) >> 3);
      const int blk = (is_a ? i0 : j0) + r;
      raw[it].m0 = raw[it].m1 = raw[it].v0 = raw[it].v1 = make_float4(0.f, 0.f, 0.f, 0.f);
      if (blk < (is_a ? nq : nk)) {
        const long long off = static_cast<long long>(blk) * D + grp * 64 + c * 8;
        const float *pm = (is_a ? qm : km) + off;
        const float *pv = (is_a ? qv : kv) + off;
        raw[it].m0 = __ldg(reinterpret_cast<const float4 *>(pm));
        raw[it].m1 = __ldg(reinterpret_cast<const float4 *>(pm + 4));
        raw[it].v0 = __ldg(reinterpret_cast<const float4 *>(pv));
        raw[it].v1 = __ldg(reinterpret_cast<const float4 *>(pv + 4));
      }
    }
  };
  auto store_group = [&](const Raw (&raw)[TPT]) {
#pragma unroll
    for (int it = 0; it < TPT; ++it) {
      const int e = it * kThreads + tid;
      const bool is_a = e < kRows * 8;
      const int r = is_a ? (e >> 3) : ((e - kRows * 8) >> 3);
      const uint32_t o = sw128(r, e & 7);
      const float m[8] = {raw[it].m0.x, raw[it].m0.y, raw[it].m0.z, raw[it].m0.w,
                          raw[it].m1.x, raw[it].m1.y, raw[it].m1.z, raw[it].m1.w};
      const float v[8] = {raw[it].v0.x, raw[it].v0.y, raw[it].v0.z, raw[it].v0.w,
                          raw[it].v1.x, raw[it].v1.y, raw[it].v1.z, raw[it].v1.w};
#pragma unroll
      for (int p = 0; p < 3; ++p) {
        float x[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (is_a)
            x[q] = p == 0 ? s * m[q] : (p == 1 ? hs2 * v[q] : hs2 * m[q] * m[q]);
          else
            x[q] = p == 0 ? m[q] : (p == 1 ? (var_product ? fmaf(m[q], m[q], v[q]) : m[q] * m[q]) : v[q]);
        }
        uint4 hi, lo;
        split8(x, hi, lo);
        const uint32_t base = p * TL::kPart + (is_a ? 0u : 2u * kABytes);
        const uint32_t step = is_a ? kABytes : TL::kBBytes;
        *reinterpret_cast<uint4 *>(smem + base + o) = hi;
        *reinterpret_cast<uint4 *>(smem + base + step + o) = lo;
      }
    }
  };

  Raw raw[TPT];
  load_group(0, raw);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const uint32_t idesc = idesc_bf16_f32(128, NT, 0, 0);

  bool ok = true;
  for (int grp = 0; grp < GROUPS; ++grp) {
    if (grp > 0) {
      // the previous group's MMAs must be done reading the operand buffers
      const bool w = mbar_wait_bounded(smem_u32(&mma_bar), (grp - 1) & 1, &abort_flag);
      if (__syncthreads_or(!w)) {
        ok = false;
        break;
      }
    }
    store_group(raw);
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int p = 0; p < 3; ++p) {
        const uint32_t pa = sbase + p * TL::kPart;
        const uint32_t pb = pa + 2 * kABytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ah = smem_desc_sw128(pa + kk * 32, 16, 1024);
          const uint64_t al = smem_desc_sw128(pa + kABytes + kk * 32, 16, 1024);
          const uint64_t bhd = smem_desc_sw128(pb + kk * 32, 16, 1024);
          const uint64_t bld = smem_desc_sw128(pb + TL::kBBytes + kk * 32, 16, 1024);
          mma_ss(tmem, ah, bhd, idesc, (grp > 0 || p > 0 || kk > 0) ? 1u : 0u);
          mma_ss(tmem, ah, bld, idesc, 1u);
          mma_ss(tmem, al, bhd, idesc, 1u);
        }
      }
      mma_commit(smem_u32(&mma_bar));
    }
    if (grp + 1 < GROUPS) load_group(grp + 1, raw);
  }
  if (ok) {
    const bool w = mbar_wait_bounded(smem_u32(&mma_bar), (GROUPS - 1) & 1, &abort_flag);
    ok = !__syncthreads_or(!w);
  }
  tc_fence_after();

  // ---------------------------------------------------------------- scores out
  if (ok) {
    const int quad = warp & 3, cq = warp >> 2;
    const int i = i0 + quad * 32 + lane;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + cq * COLS_PER_WARP;
    const float ln_full = logf(static_cast<float>(kblock));
    const float ln_last = logf(static_cast<float>(N - (nk - 1) * kblock));
    const bool vec = (nk & 3) == 0;
#pragma unroll
    for (int c0 = 0; c0 < COLS_PER_WARP; c0 += 16) {
      uint32_t r[16];
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
          : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
            "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
          : "r"(taddr + c0));
      tmem_ld_wait();
      if (i < nq) {
        const int jb = j0 + cq * COLS_PER_WARP + c0;
        float *dst = block_scores + (bh * nq + i) * nk + jb;
        float val[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) val[c] = __uint_as_float(r[c]) + (jb + c == nk - 1 ? ln_last : ln_full);
        if (vec && jb + 16 <= nk) {
#pragma unroll
          for (int c = 0; c < 16; c += 4)
            *reinterpret_cast<float4 *>(dst + c) = make_float4(val[c], val[c + 1], val[c + 2], val[c + 3]);
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c)
            if (jb + c < nk) dst[c] = val[c];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc<NT>(tmem);
  }
}

}  // namespace seltc

// ---------------------------------------------------------------- feature-fed scores
// The same score map from augmented features that the statistics pass wrote
// once per block (FeatOut in stats.cuh: planes [part, hi/lo][rows][D] bf16),
// so no tile re-derives them. Persistent CTAs walk 128 x 128 tiles ordered
// (batch and head, query tile, key tile); roles (192 threads):
//   warp 4 lane 0  TMA producer: per (64-dim group, part) stage the A hi/lo
//                  and B hi/lo operand tiles (4 x 16 KB) into a 3-stage ring;
//                  warp 4 also allocates TMEM
//   warp 5 lane 0  MMA issuer: per stage, for each 16-dim step, hi*hi, hi*lo
//                  and lo*hi into one of two 128-column TMEM accumulators
//   warps 0-3      epilogue: drain an accumulator (lane = query block), add
//                  ln m_j and store the rows while the next tile accumulates
// The MMA sequence per tile is the one select_tc_kernel issues (groups, then
// parts, then 16-dim steps; hh, hl, lh), so the scores are bit-identical.
namespace selft {
constexpr int kThreads = 192;
constexpr int kStages = 3;
constexpr uint32_t kOp = 128 * 128;              // 128 rows x 64 bf16, one swizzle span
constexpr uint32_t kStageBytes = 4 * kOp;        // A hi, A lo, B hi, B lo
constexpr uint32_t kDynSmem = kStages * kStageBytes + 1024;
constexpr int kTile = 128;
enum Bar : int { FULL = 0, EMPTY = FULL + kStages, ACC_FULL = EMPTY + kStages, ACC_EMPTY = ACC_FULL + 2,
                 DRAIN = ACC_EMPTY + 2, NUM_BARS };

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    select_feat_kernel(const __grid_constant__ CUtensorMap tm_fq, const __grid_constant__ CUtensorMap tm_fk,
                       float *__restrict__ block_scores, int Hq, int Hkv, int N, int kblock, int nq, int nk,
                       long long n_tiles, int n_tq, int n_tk) {
  constexpr int GROUPS = D / 64;
  extern __shared__ uint8_t dyn_smem[];
  __shared__ uint64_t bars[NUM_BARS];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_flag;
  const uint32_t sbase = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int k) { return smem_u32(&bars[k]); };
  const int G = Hq / Hkv;
  // tile t -> (bh, query tile, key tile)
  auto decode = [&](long long t, long long &bh, int &tq, int &tk) {
    tk = static_cast<int>(t % n_tk);
    const long long r = t / n_tk;
    tq = static_cast<int>(r % n_tq);
    bh = r / n_tq;
  };
  if (threadIdx.x == 0) {
    for (int k = 0; k < NUM_BARS; ++k) mbar_init(bar(k), (k >= ACC_EMPTY && k < ACC_EMPTY + 2) ? 128u : 1u);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc<256>(smem_u32(&tmem_base_s));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  volatile int *abort = &abort_flag;
  // launched as a dependent of the statistics pass: its features (and the
  // score map's earlier readers) are settled only from here on
  pdl_wait();
  pdl_allow_dependents();

  if (warp == 4 && lane == 0) {
    // ------------------------------------------------------------ producer
    tma_prefetch_desc(&tm_fq);
    tma_prefetch_desc(&tm_fk);
    long long it = 0;
    bool stop = false;
    for (long long t = blockIdx.x; t < n_tiles && !stop; t += gridDim.x) {
      long long bh;
      int tq, tk;
      decode(t, bh, tq, tk);
      const int b = static_cast<int>(bh / Hq), h = static_cast<int>(bh % Hq);
      const int qrow = static_cast<int>(bh * nq) + tq * kTile;
      const int krow = (b * Hkv + h / G) * nk + tk * kTile;
      for (int g = 0; g < GROUPS && !stop; ++g) {
        for (int p = 0; p < 3; ++p, ++it) {
          const int st = static_cast<int>(it % kStages);
          const long long use = it / kStages;
          if (use > 0 && !mbar_wait_bounded(bar(EMPTY + st), static_cast<uint32_t>((use - 1) & 1), abort)) {
            stop = true;
            break;
          }
          const uint32_t dst = sbase + st * kStageBytes;
          mbar_arrive_expect_tx(bar(FULL + st), kStageBytes);
          tma_load_3d(&tm_fq, dst, bar(FULL + st), 64 * g, qrow, 2 * p);
          tma_load_3d(&tm_fq, dst + kOp, bar(FULL + st), 64 * g, qrow, 2 * p + 1);
          tma_load_3d(&tm_fk, dst + 2 * kOp, bar(FULL + st), 64 * g, krow, 2 * p);
          tma_load_3d(&tm_fk, dst + 3 * kOp, bar(FULL + st), 64 * g, krow, 2 * p + 1);
        }
      }
    }
    if (*abort) {
      // let the copies in flight land before the CTA's shared memory goes away
      for (long long u = it - 1; u >= 0 && u >= it - kStages; --u)
        mbar_wait_bounded(bar(FULL + static_cast<int>(u % kStages)), static_cast<uint32_t>((u / kStages) & 1), nullptr);
    }
  } else if (warp == 5 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(128, kTile, 0, 0);
    const uint64_t d0 = smem_desc_sw128(sbase, 16, 1024);
    long long it = 0;
    int tl = 0;
    bool ok = true;
    for (long long t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++tl) {
      const int acc = tl & 1, use = tl >> 1;
      if (use > 0 && !mbar_wait_bounded(bar(ACC_EMPTY + acc), static_cast<uint32_t>((use - 1) & 1), abort)) break;
      tc_fence_after();
      const uint32_t dt = tmem + acc * kTile;
      for (int sidx = 0; sidx < 3 * GROUPS; ++sidx, ++it) {
        const int st = static_cast<int>(it % kStages);
        if (!mbar_wait_bounded(bar(FULL + st), static_cast<uint32_t>((it / kStages) & 1), abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // start-address field in 16-byte units (no carry: shared addresses < 256 KB)
        const uint64_t ah = d0 + ((st * kStageBytes) >> 4), al = ah + (kOp >> 4);
        const uint64_t bhd = ah + ((2 * kOp) >> 4), bld = ah + ((3 * kOp) >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          mma_ss(dt, ah + 2 * kk, bhd + 2 * kk, idesc, (sidx > 0 || kk > 0) ? 1u : 0u);
          mma_ss(dt, ah + 2 * kk, bld + 2 * kk, idesc, 1u);
          mma_ss(dt, al + 2 * kk, bhd + 2 * kk, idesc, 1u);
        }
        mma_commit(bar(EMPTY + st));
      }
      if (!ok) break;
      mma_commit(bar(ACC_FULL + acc));
    }
    mma_commit(bar(DRAIN));
    mbar_wait_bounded(bar(DRAIN), 0, nullptr);
  } else if (warp < 4) {
    // ------------------------------------------------------------ epilogue
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float ln_full = logf(static_cast<float>(kblock));
    const float ln_last = logf(static_cast<float>(N - (nk - 1) * kblock));
    const bool vec = (nk & 3) == 0;
    int tl = 0;
    for (long long t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tl) {
      const int acc = tl & 1, use = tl >> 1;
      const bool w = mbar_wait_bounded(bar(ACC_FULL + acc), static_cast<uint32_t>(use & 1), abort);
      if (!__all_sync(0xFFFFFFFFu, w)) break;
      tc_fence_after();
      long long bh;
      int tq, tk;
      decode(t, bh, tq, tk);
      const int i = tq * kTile + warp * 32 + lane;
      const int j0 = tk * kTile;
#pragma unroll
      for (int c0 = 0; c0 < kTile; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + acc * kTile + c0, r);
        tmem_ld_wait();
        if (i < nq) {
          const int jb = j0 + c0;
          float *dst = block_scores + (bh * nq + i) * nk + jb;
          float val[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) val[c] = __uint_as_float(r[c]) + (jb + c == nk - 1 ? ln_last : ln_full);
          if (vec && jb + 32 <= nk) {
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              *reinterpret_cast<float4 *>(dst + c) = make_float4(val[c], val[c + 1], val[c + 2], val[c + 3]);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (jb + c < nk) dst[c] = val[c];
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(ACC_EMPTY + acc));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc<256>(tmem);
  }
}
}  // namespace selft

// Scores with the widest key tile that still gives at least half the SMs a
// CTA, then the top-k launch.
// flags: the ba_att_select_ex bits (BA_SELECT_*).
template <int D>
cudaError_t launch_select_tc(const float *qm, const float *qv, const float *km, const float *kv, int32_t *idx,
                             int32_t *cnt, float *scores, int B, int Hq, int Hkv, int N, int block, int kblock, int k,
                             int kmax, float sm_scale, uint32_t flags, float tau, int num_sms, cudaStream_t stream) {
  const int var_product = (flags & BA_SELECT_NO_VAR_PRODUCT) ? 0 : 1;
  const int nq = (N + block - 1) / block, nk = (N + kblock - 1) / kblock;
  const long long bhs = static_cast<long long>(B) * Hq;
  const int nq_tiles = (nq + seltc::kRows - 1) / seltc::kRows;
  const bool wide = static_cast<long long>(nq_tiles) * ((nk + 127) / 128) * bhs >= num_sms / 2;
  cudaError_t e;
  if (wide) {
    using TL = seltc::Tile<128>;
    e = cudaFuncSetAttribute(seltc::select_tc_kernel<D, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(TL::kDynSmem));
    if (e != cudaSuccess) return e;
    dim3 grid(((nk + 127) / 128) * nq_tiles, Hq, B);
    seltc::select_tc_kernel<D, 128><<<grid, seltc::kThreads, TL::kDynSmem, stream>>>(qm, qv, km, kv, scores, Hq, Hkv,
                                                                                      N, kblock, nq, nk, sm_scale,
                                                                                      var_product);
  } else {
    using TL = seltc::Tile<64>;
    e = cudaFuncSetAttribute(seltc::select_tc_kernel<D, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(TL::kDynSmem));
    if (e != cudaSuccess) return e;
    dim3 grid(((nk + 63) / 64) * nq_tiles, Hq, B);
    seltc::select_tc_kernel<D, 64><<<grid, seltc::kThreads, TL::kDynSmem, stream>>>(qm, qv, km, kv, scores, Hq, Hkv,
                                                                                     N, kblock, nq, nk, sm_scale,
                                                                                     var_product);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const bool shared = (flags & BA_SELECT_SHARED_GQA) != 0, diag = (flags & BA_SELECT_FORCE_DIAGONAL) != 0;
  const bool mass = (flags & BA_SELECT_BY_MASS) != 0;
  if (!shared && !diag && !mass) return launch_topk(scores, nk, k, idx, kmax, cnt, bhs * nq, num_sms, stream);
  const TopkVariant var{shared ? Hq / Hkv : 1, Hq, nq, diag, mass, tau};
  return launch_topk_variant(scores, nk, k, idx, kmax, cnt, static_cast<long long>(B) * (Hq / var.group) * nq, var,
                             num_sms, stream);
}

}  // namespace baatt
