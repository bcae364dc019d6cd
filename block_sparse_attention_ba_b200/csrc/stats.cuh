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

namespace baatt {

constexpr int kStatsThreads = 256;

template <typename T, int D, int RPT>
__global__ void __launch_bounds__(kStatsThreads) stats_kernel(const T *__restrict__ Q, const T *__restrict__ K,
                                                              float *__restrict__ q_mean, float *__restrict__ q_var,
                                                              float *__restrict__ k_mean, float *__restrict__ k_var,
                                                              int B, int Hq, int Hkv, int N, int N_alloc, int block,
                                                              int nb) {
  constexpr int VEC = Elem<T>::kVec;
  constexpr int COLS = D / VEC;                   // 16-byte vectors per row
  constexpr int RPP = kStatsThreads / COLS;       // rows covered per pass
  __shared__ float red[RPP][D];
  __shared__ float mean_s[D];

  const long long n_q_ctas = static_cast<long long>(B) * Hq * nb;
  long long cta = blockIdx.x;
  const bool is_q = cta < n_q_ctas;
  if (!is_q) cta -= n_q_ctas;
  const int blk = static_cast<int>(cta % nb);
  const long long bh = cta / nb;                 // b*H + h
  const T *X = is_q ? Q : K;
  float *out_mean = is_q ? q_mean : k_mean;
  float *out_var = is_q ? q_var : k_var;

  const int row0 = blk * block;
  const int n_rows = min(block, N - row0);
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
    const long long o = (bh * nb + blk) * static_cast<long long>(D) + tid;
    out_mean[o] = mean_s[tid];
    out_var[o] = s * inv_n;
  }
}

// Rows each thread holds for a given block size (power-of-two bucket).
template <typename T, int D>
inline int stats_rpt_needed(int block) {
  constexpr int RPP = kStatsThreads / (D / Elem<T>::kVec);
  return (block + RPP - 1) / RPP;
}

template <typename T, int D>
cudaError_t launch_stats(const T *Q, const T *K, float *qm, float *qv, float *km, float *kv, int B, int Hq, int Hkv,
                         int N, int N_alloc, int block, cudaStream_t stream) {
  const int nb = (N + block - 1) / block;
  const long long grid = static_cast<long long>(B) * (Hq + Hkv) * nb;
  const int need = stats_rpt_needed<T, D>(block);
  dim3 g(static_cast<unsigned>(grid));
  if (need <= 2) {
    stats_kernel<T, D, 2><<<g, kStatsThreads, 0, stream>>>(Q, K, qm, qv, km, kv, B, Hq, Hkv, N, N_alloc, block, nb);
  } else if (need <= 4) {
    stats_kernel<T, D, 4><<<g, kStatsThreads, 0, stream>>>(Q, K, qm, qv, km, kv, B, Hq, Hkv, N, N_alloc, block, nb);
  } else if (need <= 8) {
    stats_kernel<T, D, 8><<<g, kStatsThreads, 0, stream>>>(Q, K, qm, qv, km, kv, B, Hq, Hkv, N, N_alloc, block, nb);
  } else if (need <= 16) {
    stats_kernel<T, D, 16><<<g, kStatsThreads, 0, stream>>>(Q, K, qm, qv, km, kv, B, Hq, Hkv, N, N_alloc, block, nb);
  } else {
    stats_kernel<T, D, 32><<<g, kStatsThreads, 0, stream>>>(Q, K, qm, qv, km, kv, B, Hq, Hkv, N, N_alloc, block, nb);
  }
  return cudaGetLastError();
}

}  // namespace baatt
