// attn_simt.cuh — K8s: block-sparse attention forward on CUDA cores (fp32).
//
// Same operator as the tensor-core kernel ("Efficient Long-Context Modeling
// in DLMs via Block Approximate Sparse Attention": abstract, Figure 4 —
// attention over the kept blocks only, bidirectional), for the shapes that
// kernel does not take: fp32 inputs (exact fp32 arithmetic), d = 64, block
// sizes other than 128. Online softmax over the kept key blocks, fp32 state.
//
// One CTA of 4 warps handles 16 query rows of one query block; each warp owns
// 4 rows. Keys are staged 32 at a time in shared memory; lane c scores key c
// for a row, the warp updates that row's running max / sum / output, and the
// output dimensions are spread over the lanes (d/32 per lane).
#pragma once

#include "common.cuh"

namespace baatt {

constexpr int kSimtThreads = 128;
constexpr int kSimtRows = 16;     // keeps static shared memory under 48 KB at d = 128

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// MERGE: merge with an earlier fp32 partial (O_prev, L_prev) before storing,
// as in attn_tc.cuh (O, LSE may alias O_prev, L_prev when TO is float).
template <typename T, typename TO, int D, bool MERGE>
__global__ void __launch_bounds__(kSimtThreads) attn_simt_kernel(
    const T *__restrict__ Q, const T *__restrict__ K, const T *__restrict__ V, const int32_t *__restrict__ kv_idx,
    const int32_t *__restrict__ kv_cnt, int kmax, TO *O, float *LSE, const float *O_prev, const float *L_prev, int Hq,
    int Hkv, int N, int N_alloc, int Nq, int q_stride, int block, int nb, int kblock, int nk, int subs,
    float scale_log2) {
  constexpr int DPL = D / 32;
  constexpr int RPW = kSimtRows / (kSimtThreads / 32);      // rows per warp
  __shared__ float q_s[kSimtRows][D];
  __shared__ float k_s[32][D + 1];
  __shared__ float v_s[32][D];

  const int b = blockIdx.z, h = blockIdx.y;
  const int i = blockIdx.x / subs, sub = blockIdx.x % subs;
  const int g = h / (Hq / Hkv);
  const int row0 = i * block + sub * kSimtRows;
  const int row_end = min(min(i * block + block, Nq), row0 + kSimtRows);
  if (row0 >= row_end) return;
  const int nrows = row_end - row0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const long long qhead = (static_cast<long long>(b) * Hq + h) * q_stride;
  const long long khead = (static_cast<long long>(b) * Hkv + g) * N_alloc;
  for (int e = tid; e < kSimtRows * D; e += kSimtThreads) {
    const int r = e / D, m = e % D;
    q_s[r][m] = r < nrows ? Elem<T>::load(Q + (qhead + row0 + r) * D + m) : 0.f;
  }

  float o[RPW][DPL], mrow[RPW], lrow[RPW];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    mrow[rr] = -INFINITY;
    lrow[rr] = 0.f;
#pragma unroll
    for (int t = 0; t < DPL; ++t) o[rr][t] = 0.f;
  }

  const long long list_row = (static_cast<long long>(b) * Hq + h) * nb + i;
  int c = __ldg(kv_cnt + list_row);
  if (c < 0 || c > kmax) {
    if (tid == 0 && sub == 0) raise_error(BA_DEVERR_BAD_COUNT);
    c = c < 0 ? 0 : kmax;
  }
  const int32_t *list = kv_idx + list_row * kmax;

  for (int t = 0; t < c; ++t) {
    const int j = __ldg(list + t);
    if (j < 0 || j >= nk) {
      if (tid == 0 && sub == 0) raise_error(BA_DEVERR_BAD_INDEX);
      continue;
    }
    if (t > 0 && j <= __ldg(list + t - 1)) {
      if (tid == 0 && sub == 0) raise_error(BA_DEVERR_NOT_ASCENDING);
      continue;
    }
    const int key0 = j * kblock;
    const int mj = min(kblock, N - key0);
    for (int c0 = 0; c0 < mj; c0 += 32) {
      __syncthreads();
      for (int e = tid; e < 32 * D; e += kSimtThreads) {
        const int r = e / D, m = e % D;
        const bool ok = c0 + r < mj;
        const long long off = (khead + key0 + c0 + r) * D + m;
        k_s[r][m] = ok ? Elem<T>::load(K + off) : 0.f;
        v_s[r][m] = ok ? Elem<T>::load(V + off) : 0.f;
      }
      __syncthreads();
      const bool key_ok = c0 + lane < mj;
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
        const int r = warp * RPW + rr;
        if (r >= nrows) break;
        float s = 0.f;
#pragma unroll 16
        for (int m = 0; m < D; ++m) s = fmaf(q_s[r][m], k_s[lane][m], s);
        s = key_ok ? s * scale_log2 : -INFINITY;
        const float m_new = fmaxf(mrow[rr], warp_max(s));     // finite: key 0 of the chunk is valid
        const float p = exp2f(s - m_new);
        const float alpha = exp2f(mrow[rr] - m_new);
        lrow[rr] = lrow[rr] * alpha + warp_sum(p);
#pragma unroll
        for (int tt = 0; tt < DPL; ++tt) o[rr][tt] *= alpha;
#pragma unroll 8
        for (int cc = 0; cc < 32; ++cc) {
          const float pc = __shfl_sync(0xFFFFFFFFu, p, cc);
#pragma unroll
          for (int tt = 0; tt < DPL; ++tt) o[rr][tt] = fmaf(pc, v_s[cc][lane + 32 * tt], o[rr][tt]);
        }
        mrow[rr] = m_new;
      }
    }
  }

  constexpr float kLn2 = 0.6931471805599453f;
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int r = warp * RPW + rr;
    if (r >= nrows) break;
    const bool has = lrow[rr] > 0.f;
    const float inv = has ? 1.f / lrow[rr] : 0.f;
    const long long grow = qhead + row0 + r;
    const float lse_new = has ? (mrow[rr] + log2f(lrow[rr])) * kLn2 : -INFINITY;
    MergeWeights mw{0.f, 0.f, 0.f, lse_new};
    if constexpr (MERGE) mw = merge_weights(L_prev[grow], lse_new);
    __syncwarp();                                      // every lane has read L_prev before lane 0 writes LSE
    TO *orow = O + grow * D;
#pragma unroll
    for (int tt = 0; tt < DPL; ++tt) {
      float val = o[rr][tt] * inv;
      if constexpr (MERGE) val = merge_value(mw, O_prev[grow * D + lane + 32 * tt], val);
      store_out(orow + lane + 32 * tt, val);
    }
    if (lane == 0) LSE[grow] = mw.lse;
  }
}

// Nq query rows per head at a stride of q_stride rows (Nq = N, q_stride =
// N_alloc for a full call); keys: N valid rows at a stride of N_alloc.
template <typename T, typename TO, int D, bool MERGE = false>
cudaError_t launch_attn_simt(const T *Q, const T *K, const T *V, const int32_t *idx, const int32_t *cnt, int kmax, TO *O,
                             float *LSE, int B, int Hq, int Hkv, int N, int N_alloc, int Nq, int q_stride, int block,
                             int kblock, float sm_scale, cudaStream_t stream, const float *O_prev = nullptr,
                             const float *L_prev = nullptr) {
  const int nb = (Nq + block - 1) / block, nk = (N + kblock - 1) / kblock;
  const int subs = (block + kSimtRows - 1) / kSimtRows;
  dim3 grid(static_cast<unsigned>(nb * subs), Hq, B);
  const float scale_log2 = sm_scale * 1.4426950408889634f;
  attn_simt_kernel<T, TO, D, MERGE><<<grid, kSimtThreads, 0, stream>>>(Q, K, V, idx, cnt, kmax, O, LSE, O_prev, L_prev,
                                                                    Hq, Hkv, N, N_alloc, Nq, q_stride, block, nb,
                                                                    kblock, nk, subs, scale_log2);
  return cudaGetLastError();
}

}  // namespace baatt
