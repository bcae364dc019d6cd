// select_tc.cuh — K7 on the tensor cores: covariance-compensated block
// scores as one tcgen05 GEMM, then an exact per-row top-k read from TMEM.
//
// Same operator as select.cuh ("Efficient Long-Context Modeling in DLMs via
// Block Approximate Sparse Attention": abstract; "Core claim"; Figure 2):
//   S~[i,j] = qt_i . kt_j + ln m_j,
//   qt_i = [ s qbar_i , (s^2/2) vq_i , (s^2/2) qbar_i^2 ],
//   kt_j = [ kbar_j , kbar_j^2 + vk_j , vk_j ]            (3d = 384 wide)
// ranked per query block, ties to the lower key block, top k kept ascending.
//
// One CTA = 128 query blocks of one (batch, head) x every key block (nk <=
// 512, so the fp32 score tile fits the 512 TMEM columns).
//  1. GEMM: the augmented rows are built from the fp32 statistics straight
//     into shared memory in the 128-byte-swizzled K-major layout, 64 of the
//     384 dimensions at a time. For fp32-level accuracy every operand is split
//     x = hi + lo (two bf16s, 16 significant bits) and S accumulates
//     hi*hi + hi*lo + lo*hi in fp32 (the dropped lo*lo is ~2^-16 relative).
//     One thread issues the tcgen05.mma (M=128, N<=256 per tile) and commits
//     to an mbarrier that gates the next slice.
//  2. The fp32 score rows are drained from TMEM through the (now free)
//     operand buffer into the score map; the top-k then runs as its own
//     launch with one warp per row over the whole GPU (topk_rows_kernel), as
//     one CTA's 128 rows per SM leave most SMs idle and each row's radix
//     select is latency-bound.
#pragma once

#include "common.cuh"
#include "select.cuh"

namespace baatt {
namespace seltc {

constexpr int kThreads = 256;
constexpr int kRows = 128;                       // query blocks per CTA (TMEM lanes)
constexpr int kMaxKeys = 512;                    // TMEM columns
constexpr uint32_t kSliceA = kRows * 128;        // 128 rows x 64 bf16 = 16 KB
constexpr uint32_t kSliceB = kMaxKeys * 128;     // 512 rows x 64 bf16 = 64 KB
constexpr uint32_t kOffAhi = 0, kOffAlo = kSliceA, kOffBhi = 2 * kSliceA, kOffBlo = 2 * kSliceA + kSliceB;
constexpr uint32_t kOperandBytes = 2 * kSliceA + 2 * kSliceB;             // 160 KB
constexpr uint32_t kScoreBytes = 152u * 1024u;                            // score rows (reuse the above)
constexpr uint32_t kDynSmem = kOperandBytes + 1024;

// 8 consecutive augmented values -> hi and lo bf16 vectors.
__device__ __forceinline__ void split8(const float (&x)[8], uint4 &hi, uint4 &lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat16 h0 = __float2bfloat16_rn(x[2 * e]), h1 = __float2bfloat16_rn(x[2 * e + 1]);
    const float r0 = x[2 * e] - __bfloat162float(h0), r1 = x[2 * e + 1] - __bfloat162float(h1);
    h[e] = pack_bf16x2(__bfloat162float(h0), __bfloat162float(h1));
    l[e] = pack_bf16x2(r0, r1);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Byte offset of 16-byte chunk c (0..7) of row r in a 128B-swizzled tile.
__device__ __forceinline__ uint32_t sw128(int r, int c) {
  return static_cast<uint32_t>(r) * 128u + (static_cast<uint32_t>(c ^ (r & 7)) << 4);
}

// 8 consecutive fp32 statistics (read-only path, so loads of several chunks
// can be in flight together).
struct Raw8 {
  float4 a, b;
};
__device__ __forceinline__ Raw8 ld8(const float *p) {
  return {__ldg(reinterpret_cast<const float4 *>(p)), __ldg(reinterpret_cast<const float4 *>(p + 4))};
}
__device__ __forceinline__ void unpack8(const Raw8 &r, float (&x)[8]) {
  x[0] = r.a.x; x[1] = r.a.y; x[2] = r.a.z; x[3] = r.a.w;
  x[4] = r.b.x; x[5] = r.b.y; x[6] = r.b.z; x[7] = r.b.w;
}

// Augmented query features, part 0/1/2: s*qbar, (s^2/2)*vq, (s^2/2)*qbar^2.
__device__ __forceinline__ void aug_q(const Raw8 &m, const Raw8 &v, int part, float s, float hs2, float (&x)[8]) {
  float mm[8], vv[8];
  unpack8(m, mm);
  unpack8(v, vv);
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = part == 0 ? s * mm[e] : (part == 1 ? hs2 * vv[e] : hs2 * mm[e] * mm[e]);
}
// Augmented key features, part 0/1/2: kbar, kbar^2 + vk, vk.
__device__ __forceinline__ void aug_k(const Raw8 &m, const Raw8 &v, int part, float (&x)[8]) {
  float mm[8], vv[8];
  unpack8(m, mm);
  unpack8(v, vv);
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = part == 0 ? mm[e] : (part == 1 ? fmaf(mm[e], mm[e], vv[e]) : vv[e]);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    select_tc_kernel(const float *__restrict__ q_mean, const float *__restrict__ q_var,
                     const float *__restrict__ k_mean, const float *__restrict__ k_var, int32_t *__restrict__ kv_idx,
                     int32_t *__restrict__ kv_cnt, float *__restrict__ block_scores, int Hq, int Hkv, int N,
                     int block, int nb, int k, int kmax, float sm_scale) {
  constexpr int SLICES = 3 * D / 64;
  constexpr int SL_PER_PART = D / 64;
  extern __shared__ uint8_t dyn_smem[];
  __shared__ uint64_t mma_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ float lnm[kMaxKeys];
  __shared__ int abort_flag;
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int b = blockIdx.z, h = blockIdx.y, g = h / (Hq / Hkv);
  const int i0 = blockIdx.x * kRows;
  const int nk_pad = (nb + 15) & ~15;
  const int n_tiles = nk_pad > 256 ? 2 : 1;
  const float s = sm_scale, hs2 = 0.5f * sm_scale * sm_scale;
  const float *qm = q_mean + (static_cast<long long>(b) * Hq + h) * nb * D;
  const float *qv = q_var + (static_cast<long long>(b) * Hq + h) * nb * D;
  const float *km = k_mean + (static_cast<long long>(b) * Hkv + g) * nb * D;
  const float *kv = k_var + (static_cast<long long>(b) * Hkv + g) * nb * D;

  for (int j = tid; j < kMaxKeys; j += kThreads)
    lnm[j] = j < nb ? logf(static_cast<float>(min(block, N - j * block))) : 0.f;
  if (tid == 0) {
    mbar_init(smem_u32(&mma_bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc<kMaxKeys>(smem_u32(&tmem_base_s));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;

  // ---------------------------------------------------------------- GEMM
  bool ok = true;
  for (int sl = 0; sl < SLICES && ok; ++sl) {
    const int part = sl / SL_PER_PART;
    const int d0 = (sl % SL_PER_PART) * 64;
    // A: 128 rows x 8 chunks, then B: nk_pad rows x 8 chunks, 4 chunks per
    // thread per batch with all their loads issued before any use.
    const Raw8 zero8 = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
    for (int e0 = 0; e0 < (kRows + nk_pad) * 8; e0 += 4 * kThreads) {
      Raw8 rm[4], rv[4];
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int e = e0 + it * kThreads + tid;
        rm[it] = zero8;
        rv[it] = zero8;
        if (e < kRows * 8) {
          const int i = i0 + (e >> 3);
          if (i < nb) {
            const long long off = static_cast<long long>(i) * D + d0 + 8 * (e & 7);
            if (part != 1) rm[it] = ld8(qm + off);
            if (part == 1) rv[it] = ld8(qv + off);
          }
        } else if (e < (kRows + nk_pad) * 8) {
          const int r = (e - kRows * 8) >> 3;
          if (r < nb) {
            const long long off = static_cast<long long>(r) * D + d0 + 8 * (e & 7);
            if (part != 2) rm[it] = ld8(km + off);
            if (part != 0) rv[it] = ld8(kv + off);
          }
        }
      }
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int e = e0 + it * kThreads + tid;
        if (e >= (kRows + nk_pad) * 8) break;
        float x[8];
        uint4 hi, lo;
        if (e < kRows * 8) {
          aug_q(rm[it], rv[it], part, s, hs2, x);
          split8(x, hi, lo);
          const uint32_t o = sw128(e >> 3, e & 7);
          *reinterpret_cast<uint4 *>(smem + kOffAhi + o) = hi;
          *reinterpret_cast<uint4 *>(smem + kOffAlo + o) = lo;
        } else {
          aug_k(rm[it], rv[it], part, x);
          split8(x, hi, lo);
          const uint32_t o = sw128((e - kRows * 8) >> 3, e & 7);
          *reinterpret_cast<uint4 *>(smem + kOffBhi + o) = hi;
          *reinterpret_cast<uint4 *>(smem + kOffBlo + o) = lo;
        }
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      for (int nt = 0; nt < n_tiles; ++nt) {
        const int n = (nt == 0) ? (nk_pad > 256 ? 256 : nk_pad) : nk_pad - 256;
        const uint32_t idesc = idesc_bf16_f32(128, n, 0, 0);
        const uint32_t d_tmem = tmem + nt * 256;
        const uint32_t boff = nt * 256 * 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ah = smem_desc_sw128(sbase + kOffAhi + kk * 32, 16, 1024);
          const uint64_t al = smem_desc_sw128(sbase + kOffAlo + kk * 32, 16, 1024);
          const uint64_t bh = smem_desc_sw128(sbase + kOffBhi + boff + kk * 32, 16, 1024);
          const uint64_t bl = smem_desc_sw128(sbase + kOffBlo + boff + kk * 32, 16, 1024);
          mma_ss(d_tmem, ah, bh, idesc, (sl > 0 || kk > 0) ? 1u : 0u);
          mma_ss(d_tmem, ah, bl, idesc, 1u);
          mma_ss(d_tmem, al, bh, idesc, 1u);
        }
      }
      mma_commit(smem_u32(&mma_bar));
    }
    // the operand buffers are rewritten by the next slice (and reused as
    // histograms after the last): wait for these MMAs to finish reading them
    const bool w = mbar_wait_bounded(smem_u32(&mma_bar), sl & 1, &abort_flag);
    ok = !__syncthreads_or(!w);
  }
  tc_fence_after();

  // ---------------------------------------------------------------- scores out
  // TMEM -> shared memory (row stride nk_pad + 1 keeps the per-row drain
  // conflict-free), 128 rows at once when they fit, else two halves of 64,
  // then coalesced row writes of S~ (ln m_j included) to the score map. Warps
  // w and w + 4 drain the same TMEM lane quadrant, each half of the columns.
  if (ok) {
    const int stride = nk_pad + 1;
    float *sc = reinterpret_cast<float *>(smem);
    const int rows_per_pass = (kRows * stride * 4 <= static_cast<int>(kScoreBytes)) ? kRows : kRows / 2;
    for (int r0 = 0; r0 < kRows; r0 += rows_per_pass) {
      const int quad = warp & 3;
      if (quad * 32 >= r0 && quad * 32 < r0 + rows_per_pass) {
        const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const int r = quad * 32 + (tid & 31) - r0;          // row within this pass
        const int half_cols = nk_pad / 2;                    // multiple of 8
        const int cbeg = (warp < 4) ? 0 : half_cols, cend = (warp < 4) ? half_cols : nk_pad;
        for (int c0 = cbeg; c0 < cend; c0 += 8) {
          uint32_t v[8];
          asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                       : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
                         "=r"(v[7])
                       : "r"(taddr + c0));
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 8; ++c) sc[r * stride + c0 + c] = __uint_as_float(v[c]) + lnm[c0 + c];
        }
      }
      __syncthreads();
      for (int rr = warp; rr < rows_per_pass; rr += kThreads / 32) {   // coalesced row write-out
        const int i = i0 + r0 + rr;
        if (i >= nb) break;
        const long long row = (static_cast<long long>(b) * Hq + h) * nb + i;
        const float *srow = sc + rr * stride;
        for (int j = tid & 31; j < nb; j += 32) block_scores[row * nb + j] = srow[j];
      }
      __syncthreads();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc<kMaxKeys>(tmem);
  }
}

}  // namespace seltc

template <int D>
cudaError_t launch_select_tc(const float *qm, const float *qv, const float *km, const float *kv, int32_t *idx,
                             int32_t *cnt, float *scores, int B, int Hq, int Hkv, int N, int block, int k, int kmax,
                             float sm_scale, cudaStream_t stream) {
  const int nb = (N + block - 1) / block;
  cudaError_t e = cudaFuncSetAttribute(seltc::select_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(seltc::kDynSmem));
  if (e != cudaSuccess) return e;
  dim3 grid((nb + seltc::kRows - 1) / seltc::kRows, Hq, B);
  seltc::select_tc_kernel<D><<<grid, seltc::kThreads, seltc::kDynSmem, stream>>>(qm, qv, km, kv, idx, cnt, scores, Hq,
                                                                                Hkv, N, block, nb, k, kmax, sm_scale);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_topk(scores, nb, k, idx, kmax, cnt, static_cast<long long>(B) * Hq * nb, stream);
}

}  // namespace baatt
