// select.cuh — K7: covariance-compensated block scores + norm sorting.
//
// "Efficient Long-Context Modeling in DLMs via Block Approximate Sparse
// Attention" (abstract; "Core claim"; Figure 2): key blocks are scored in
// the downsampled block space, the pooled score is corrected with diagonal
// Q/K variances, blocks are sorted and the top fraction is kept.
//
//   S~[i,j] = s qbar_i.kbar_j + (s^2/2) sum_m (vq kbar^2 + qbar^2 vk + vq vk) + ln m_j
//
// written as one 3d-long dot product of augmented rows
//   qt_i = [ s qbar_i , (s^2/2) vq_i , (s^2/2) qbar_i^2 ]
//   kt_j = [ kbar_j   , kbar_j^2 + vk_j , vk_j ]
// so that S~ = qt_i . kt_j + ln m_j (fp32 FMA accumulation).
//
// Two launches. select_kernel (SIMT; the tensor-core variant for nk <= 512
// lives in select_tc.cuh) writes the whole fp32 score map; topk_rows_kernel
// then gives one warp to each (batch, head, query block) row and selects its
// top k by an exact 4-pass radix select on order-preserving keys of the fp32
// scores (taken relative to the row minimum so that the high bytes carry
// information); equal scores go to the lower block index, and the kept
// indices are emitted ascending.
#pragma once

#include "common.cuh"

namespace baatt {

constexpr int kSelThreads = 256;
constexpr int kSelKeyChunk = 32;

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 0u;                       // NaN ranks last
  if (f == 0.f) f = 0.f;                       // -0 == +0
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exact top-k of one row held in shared memory; one warp.
__device__ void topk_row_warp(const float *__restrict__ srow, int nk, int k, int32_t *__restrict__ out_idx, int kmax,
                              int32_t *__restrict__ out_cnt, unsigned *__restrict__ hist, int lane) {
  constexpr int CH = 8;                                 // keys per lane held in registers at a time
  const uint32_t hist_s = smem_u32(hist);
  const unsigned full = 0xFFFFFFFFu;
  const unsigned lt_mask = (1u << lane) - 1u;
  if (k >= nk) {
    for (int j = lane; j < kmax; j += 32) out_idx[j] = j < nk ? j : -1;
    if (lane == 0) *out_cnt = nk;
    return;
  }
  // Block scores of a row sit in a narrow range, so the top bits of their
  // order keys are nearly all equal: select on u - umin instead, from its
  // highest differing bit, so that the first digit already spreads the keys.
  uint32_t umin = 0xFFFFFFFFu, umax = 0u;
  for (int j0 = 0; j0 < nk; j0 += 32 * CH) {
    uint32_t u[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int j = j0 + c * 32 + lane;
      u[c] = j < nk ? order_key(srow[j]) : 0u;
    }
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      if (j0 + c * 32 + lane < nk) {
        umin = min(umin, u[c]);
        umax = max(umax, u[c]);
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    umin = min(umin, __shfl_xor_sync(full, umin, off));
    umax = max(umax, __shfl_xor_sync(full, umax, off));
  }
  const uint32_t range = umax - umin;
  const int nbits = range == 0u ? 0 : ((32 - __clz(range) + 7) & ~7);    // 8, 16, 24 or 32
  uint32_t prefix = 0u, mask = 0u;
  int need = k;
  for (int shift = nbits - 8; shift >= 0; shift -= 8) {
    for (int t = lane; t < 256; t += 32) hist[t] = 0u;
    __syncwarp();
    for (int j0 = 0; j0 < nk; j0 += 32 * CH) {
      uint32_t v[CH];
#pragma unroll
      for (int c = 0; c < CH; ++c) {                   // all loads of the chunk first
        const int j = j0 + c * 32 + lane;
        v[c] = j < nk ? order_key(srow[j]) - umin : 0u;
      }
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        if (j0 + c * 32 + lane < nk && (v[c] & mask) == prefix)
          red_shared_add(hist_s + 4u * ((v[c] >> shift) & 255u), 1u);
      }
    }
    __syncwarp();
    int cnts[8];
    int local = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      cnts[t] = static_cast<int>(hist[255 - 8 * lane - t]);
      local += cnts[t];
    }
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(full, incl, off);
      if (lane >= off) incl += y;
    }
    const int excl = incl - local;
    const unsigned hit = __ballot_sync(full, incl >= need);
    const int src = __ffs(hit) - 1;
    int digit = 0, above = 0;
    if (lane == src) {
      int c = excl;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (c + cnts[t] >= need) {
          digit = 255 - 8 * lane - t;
          above = c;
          break;
        }
        c += cnts[t];
      }
    }
    digit = __shfl_sync(full, digit, src);
    above = __shfl_sync(full, above, src);
    prefix |= static_cast<uint32_t>(digit) << shift;
    mask |= 255u << shift;
    need -= above;
    __syncwarp();
  }
  // umin + prefix is the k-th largest key; take every larger key and the
  // first `need` equal keys in index order.
  prefix += umin;
  int pos = 0, eq_seen = 0;
  for (int j0 = 0; j0 < nk; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t u = j < nk ? order_key(srow[j]) : 0u;
    const bool gt = j < nk && u > prefix;
    const bool eq = j < nk && u == prefix;
    const unsigned eqb = __ballot_sync(full, eq);
    const int eq_rank = eq_seen + __popc(eqb & lt_mask);
    const bool kept = gt || (eq && eq_rank < need);
    const unsigned kb = __ballot_sync(full, kept);
    if (kept) out_idx[pos + __popc(kb & lt_mask)] = j;
    pos += __popc(kb);
    eq_seen += __popc(eqb);
  }
  for (int j = pos + lane; j < kmax; j += 32) out_idx[j] = -1;
  if (lane == 0) *out_cnt = pos;
}

// The same exact selection for a row held in registers: lane l holds the
// order keys of columns c*32 + l, c < KPL (so column order is chunk-major).
// Every radix pass reads registers only; the per-warp histogram lives in
// shared memory at hist_s.
template <int KPL>
__device__ __forceinline__ void topk_row_regs(const uint32_t (&u)[KPL], int nk, int k, int32_t *__restrict__ out_idx,
                                              int kmax, int32_t *__restrict__ out_cnt, uint32_t hist_s, int lane) {
  const unsigned full = 0xFFFFFFFFu;
  const unsigned lt_mask = (1u << lane) - 1u;
  if (k >= nk) {
    for (int j = lane; j < kmax; j += 32) out_idx[j] = j < nk ? j : -1;
    if (lane == 0) *out_cnt = nk;
    return;
  }
  uint32_t umin = 0xFFFFFFFFu, umax = 0u;
#pragma unroll
  for (int c = 0; c < KPL; ++c) {
    if (c * 32 + lane < nk) {
      umin = min(umin, u[c]);
      umax = max(umax, u[c]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    umin = min(umin, __shfl_xor_sync(full, umin, off));
    umax = max(umax, __shfl_xor_sync(full, umax, off));
  }
  const uint32_t range = umax - umin;
  const int nbits = range == 0u ? 0 : ((32 - __clz(range) + 7) & ~7);
  uint32_t prefix = 0u, mask = 0u;
  int need = k;
  for (int shift = nbits - 8; shift >= 0; shift -= 8) {
#pragma unroll
    for (int t = 0; t < 8; ++t) asm volatile("st.shared.u32 [%0], %1;" ::"r"(hist_s + 4u * (lane + 32 * t)), "r"(0u));
    __syncwarp();
#pragma unroll
    for (int c = 0; c < KPL; ++c) {
      const uint32_t v = u[c] - umin;
      if (c * 32 + lane < nk && (v & mask) == prefix) red_shared_add(hist_s + 4u * ((v >> shift) & 255u), 1u);
    }
    __syncwarp();
    int cnts[8];
    int local = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      uint32_t x;
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(x) : "r"(hist_s + 4u * (255 - 8 * lane - t)));
      cnts[t] = static_cast<int>(x);
      local += cnts[t];
    }
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(full, incl, off);
      if (lane >= off) incl += y;
    }
    const int excl = incl - local;
    const unsigned hit = __ballot_sync(full, incl >= need);
    const int src = __ffs(hit) - 1;
    int digit = 0, above = 0;
    if (lane == src) {
      int c = excl;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (c + cnts[t] >= need) {
          digit = 255 - 8 * lane - t;
          above = c;
          break;
        }
        c += cnts[t];
      }
    }
    digit = __shfl_sync(full, digit, src);
    above = __shfl_sync(full, above, src);
    prefix |= static_cast<uint32_t>(digit) << shift;
    mask |= 255u << shift;
    need -= above;
    __syncwarp();
  }
  const uint32_t thr = prefix + umin;                   // the k-th largest key
  int pos = 0, eq_seen = 0;
#pragma unroll
  for (int c = 0; c < KPL; ++c) {
    const int j = c * 32 + lane;
    const bool in = j < nk;
    const bool gt = in && u[c] > thr;
    const bool eq = in && u[c] == thr;
    const unsigned eqb = __ballot_sync(full, eq);
    const bool kept = gt || (eq && eq_seen + __popc(eqb & lt_mask) < need);
    const unsigned kb = __ballot_sync(full, kept);
    if (kept) out_idx[pos + __popc(kb & lt_mask)] = j;
    pos += __popc(kb);
    eq_seen += __popc(eqb);
  }
  for (int j = pos + lane; j < kmax; j += 32) out_idx[j] = -1;
  if (lane == 0) *out_cnt = pos;
}

// One warp per (batch, head, query block) row of the score map; rows up to
// 32*KPL keys are held in registers, longer rows are re-read per pass.
constexpr int kTopkWarps = 8;

template <int KPL>
__global__ void __launch_bounds__(kTopkWarps * 32) topk_rows_kernel(const float *__restrict__ scores, int nk, int k,
                                                                    int32_t *__restrict__ kv_idx, int kmax,
                                                                    int32_t *__restrict__ kv_cnt, long long rows) {
  __shared__ unsigned hist[kTopkWarps][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = blockIdx.x * static_cast<long long>(kTopkWarps) + warp;
  if (row >= rows) return;
  const float *srow = scores + row * nk;
  if constexpr (KPL > 0) {
    uint32_t u[KPL];
#pragma unroll
    for (int c = 0; c < KPL; ++c) {
      const int j = c * 32 + lane;
      u[c] = j < nk ? order_key(__ldg(srow + j)) : 0u;
    }
    topk_row_regs<KPL>(u, nk, k, kv_idx + row * kmax, kmax, kv_cnt + row, smem_u32(&hist[warp][0]), lane);
  } else {
    topk_row_warp(srow, nk, k, kv_idx + row * kmax, kmax, kv_cnt + row, &hist[warp][0], lane);
  }
}

inline cudaError_t launch_topk(const float *scores, int nk, int k, int32_t *idx, int kmax, int32_t *cnt,
                               long long rows, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>((rows + kTopkWarps - 1) / kTopkWarps);
  const int threads = kTopkWarps * 32;
  if (nk <= 256)
    topk_rows_kernel<8><<<grid, threads, 0, stream>>>(scores, nk, k, idx, kmax, cnt, rows);
  else if (nk <= 512)
    topk_rows_kernel<16><<<grid, threads, 0, stream>>>(scores, nk, k, idx, kmax, cnt, rows);
  else if (nk <= 1024)
    topk_rows_kernel<32><<<grid, threads, 0, stream>>>(scores, nk, k, idx, kmax, cnt, rows);
  else
    topk_rows_kernel<0><<<grid, threads, 0, stream>>>(scores, nk, k, idx, kmax, cnt, rows);
  return cudaGetLastError();
}

template <int D>
__global__ void __launch_bounds__(kSelThreads) select_kernel(
    const float *__restrict__ q_mean, const float *__restrict__ q_var, const float *__restrict__ k_mean,
    const float *__restrict__ k_var, int32_t *__restrict__ kv_idx, int32_t *__restrict__ kv_cnt,
    float *__restrict__ block_scores, int Hq, int Hkv, int N, int block, int nb, int R, int k, int kmax,
    float sm_scale) {
  constexpr int D3 = 3 * D;
  constexpr int KT_STRIDE = D3 + 4;                  // floats; keeps float4 rows conflict-free
  extern __shared__ __align__(16) float sel_smem[];
  float *qt = sel_smem;                              // [R][D3]
  float *kt = qt + R * D3;                           // [kSelKeyChunk][KT_STRIDE]
  float *sc = kt + kSelKeyChunk * KT_STRIDE;         // [R][nb]

  const int b = blockIdx.z, h = blockIdx.y;
  const int g = h / (Hq / Hkv);
  const int i0 = blockIdx.x * R;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float s = sm_scale, hs2 = 0.5f * sm_scale * sm_scale;

  const float *qm = q_mean + (static_cast<long long>(b) * Hq + h) * nb * D;
  const float *qv = q_var + (static_cast<long long>(b) * Hq + h) * nb * D;
  const float *km = k_mean + (static_cast<long long>(b) * Hkv + g) * nb * D;
  const float *kv = k_var + (static_cast<long long>(b) * Hkv + g) * nb * D;

  for (int e = tid; e < R * D; e += kSelThreads) {
    const int r = e / D, m = e % D;
    const int i = i0 + r;
    float a = 0.f, bq = 0.f, cq = 0.f;
    if (i < nb) {
      const float mu = __ldg(qm + static_cast<long long>(i) * D + m);
      const float va = __ldg(qv + static_cast<long long>(i) * D + m);
      a = s * mu;
      bq = hs2 * va;
      cq = hs2 * mu * mu;
    }
    qt[r * D3 + m] = a;
    qt[r * D3 + D + m] = bq;
    qt[r * D3 + 2 * D + m] = cq;
  }

  for (int j0 = 0; j0 < nb; j0 += kSelKeyChunk) {
    __syncthreads();
    for (int e = tid; e < kSelKeyChunk * D; e += kSelThreads) {
      const int c = e / D, m = e % D;
      const int j = j0 + c;
      float a = 0.f, bb = 0.f, cc = 0.f;
      if (j < nb) {
        const float mu = __ldg(km + static_cast<long long>(j) * D + m);
        const float va = __ldg(kv + static_cast<long long>(j) * D + m);
        a = mu;
        bb = mu * mu + va;
        cc = va;
      }
      kt[c * KT_STRIDE + m] = a;
      kt[c * KT_STRIDE + D + m] = bb;
      kt[c * KT_STRIDE + 2 * D + m] = cc;
    }
    __syncthreads();
    const int j = j0 + lane;
    const float4 *krow = reinterpret_cast<const float4 *>(kt + lane * KT_STRIDE);
    for (int r = warp; r < R; r += kSelThreads / 32) {
      const float4 *qrow = reinterpret_cast<const float4 *>(qt + r * D3);
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
      for (int m4 = 0; m4 < D3 / 4; ++m4) {
        const float4 qv4 = qrow[m4];
        const float4 kv4 = krow[m4];
        acc0 = fmaf(qv4.x, kv4.x, acc0);
        acc1 = fmaf(qv4.y, kv4.y, acc1);
        acc0 = fmaf(qv4.z, kv4.z, acc0);
        acc1 = fmaf(qv4.w, kv4.w, acc1);
      }
      if (j < nb) {
        const int mj = min(block, N - j * block);
        sc[r * nb + j] = (acc0 + acc1) + logf(static_cast<float>(mj));
      }
    }
  }
  __syncthreads();

  for (int e = tid; e < R * nb; e += kSelThreads) {     // coalesced rows of the score map
    const int r = e / nb, j = e % nb;
    const int i = i0 + r;
    if (i < nb) block_scores[((static_cast<long long>(b) * Hq + h) * nb + i) * nb + j] = sc[e];
  }
}

inline int select_rows_per_cta(int nb) {
  int R = 16384 / nb;
  if (R > 16) R = 16;
  if (R < 1) R = 1;
  return R;
}

inline size_t select_smem_bytes(int D, int nb) {
  const int R = select_rows_per_cta(nb);
  return sizeof(float) * (static_cast<size_t>(R) * 3 * D + static_cast<size_t>(kSelKeyChunk) * (3 * D + 4) +
                          static_cast<size_t>(R) * nb);
}

template <int D>
cudaError_t launch_select(const float *qm, const float *qv, const float *km, const float *kv, int32_t *idx,
                          int32_t *cnt, float *scores, int B, int Hq, int Hkv, int N, int block, int k, int kmax,
                          float sm_scale, cudaStream_t stream) {
  const int nb = (N + block - 1) / block;
  const int R = select_rows_per_cta(nb);
  const size_t smem = select_smem_bytes(D, nb);
  cudaError_t e = cudaFuncSetAttribute(select_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((nb + R - 1) / R, Hq, B);
  select_kernel<D><<<grid, kSelThreads, smem, stream>>>(qm, qv, km, kv, idx, cnt, scores, Hq, Hkv, N, block, nb, R,
                                                        k, kmax, sm_scale);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_topk(scores, nb, k, idx, kmax, cnt, static_cast<long long>(B) * Hq * nb, stream);
}

}  // namespace baatt
