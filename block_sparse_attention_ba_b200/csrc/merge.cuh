// merge.cuh — K9: log-space merge of two partial attentions, and the list
// split that produces the two partial key sets.
//
// "FlashBlock: Attention Caching for Efficient Long-Context Block Diffusion",
// Eq. 5 (attention over a key set splits exactly into the contributions of
// two disjoint parts) and Eq. 9 (the parts are recombined from their outputs
// and log-normalisers after subtracting the larger normaliser).
#pragma once

#include "common.cuh"

namespace baatt {

constexpr int kMergeThreads = 256;

// VEC consecutive elements as floats, read with 16-byte loads.
template <typename T, int VEC>
__device__ __forceinline__ void load_vec(const T *p, float (&f)[VEC]) {
  constexpr int PER = Elem<T>::kVec;                  // elements per 16-byte load
  static_assert(VEC % PER == 0, "vector width");
#pragma unroll
  for (int k = 0; k < VEC / PER; ++k) {
    float g[PER];
    Elem<T>::unpack(*reinterpret_cast<const uint4 *>(p + k * PER), g);
#pragma unroll
    for (int e = 0; e < PER; ++e) f[k * PER + e] = g[e];
  }
}

// One 16-byte vector of a row per thread; rows are independent. HBM-bound:
// reads O1, O2, L1, L2 once and writes O, L once.
// Each thread handles VEC consecutive elements of one row, VEC = the number of
// output elements in 16 bytes; inputs are read as one or two 16-byte vectors.
template <typename TI, typename TO, int D>
__global__ void __launch_bounds__(kMergeThreads) merge_lse_kernel(const TI *O1, const float *L1, const TI *O2,
                                                                  const float *L2, TO *O, float *L,
                                                                  long long rows) {
  constexpr int VEC = Elem<TO>::kVec;
  constexpr int VPR = D / VEC;                         // vectors per row
  const long long total = rows * VPR;
  const int lane = threadIdx.x & 31;
  // A row's VPR threads sit in one warp (VPR divides 32), so a __syncwarp()
  // between the reads and the writes makes the in-place forms (O == O1,
  // L == L1, ...) safe. The loop bound is warp-uniform for that reason.
  for (long long base = blockIdx.x * static_cast<long long>(kMergeThreads) + (threadIdx.x & ~31); base < total;
       base += static_cast<long long>(gridDim.x) * kMergeThreads) {
    const long long v = base + lane;
    const bool act = v < total;
    const long long r = act ? v / VPR : 0;
    const int c = static_cast<int>(v % VPR);
    float out[VEC];
    float lse = 0.f;
    if (act) {
      const MergeWeights mw = merge_weights(L1[r], L2[r]);
      float fa[VEC], fb[VEC];
      load_vec<TI, VEC>(O1 + r * D + c * VEC, fa);
      load_vec<TI, VEC>(O2 + r * D + c * VEC, fb);
#pragma unroll
      for (int e = 0; e < VEC; ++e) out[e] = merge_value(mw, fa[e], fb[e]);
      lse = mw.lse;
    }
    __syncwarp();
    if (act) {
      uint4 res;
      if constexpr (VEC == 8) {
        res.x = pack_bf16x2(out[0], out[1]);
        res.y = pack_bf16x2(out[2], out[3]);
        res.z = pack_bf16x2(out[4], out[5]);
        res.w = pack_bf16x2(out[6], out[7]);
      } else {
        res.x = __float_as_uint(out[0]);
        res.y = __float_as_uint(out[1]);
        res.z = __float_as_uint(out[2]);
        res.w = __float_as_uint(out[3]);
      }
      reinterpret_cast<uint4 *>(O + r * D)[c] = res;
      if (c == 0) L[r] = lse;
    }
  }
}

template <typename TI, typename TO, int D>
cudaError_t launch_merge(const TI *O1, const float *L1, const TI *O2, const float *L2, TO *O, float *L, long long rows,
                         int num_sms, cudaStream_t stream) {
  constexpr int VPR = D / Elem<TO>::kVec;
  const long long total = rows * VPR;
  long long blocks = (total + kMergeThreads - 1) / kMergeThreads;
  const long long cap = static_cast<long long>(num_sms) * 8;     // 8 resident CTAs per SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  merge_lse_kernel<TI, TO, D><<<static_cast<unsigned>(blocks), kMergeThreads, 0, stream>>>(O1, L1, O2, L2, O, L, rows);
  return cudaGetLastError();
}

// One warp per list: entries below split_block go to the "lo" list, the rest
// to the "hi" list; both stay ascending. Out-of-range entries are dropped and
// flagged.
__global__ void split_lists_kernel(const int32_t *__restrict__ idx, const int32_t *__restrict__ cnt, int32_t *lo_idx,
                                   int32_t *lo_cnt, int32_t *hi_idx, int32_t *hi_cnt, long long n_lists, int kmax,
                                   int nk, int split) {
  const unsigned full = 0xFFFFFFFFu;
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  const long long warps_total = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  for (long long row = blockIdx.x * static_cast<long long>(blockDim.x / 32) + (threadIdx.x >> 5); row < n_lists;
       row += warps_total) {
    int c = __ldg(cnt + row);
    if (c < 0 || c > kmax) {
      if (lane == 0) raise_error(BA_DEVERR_BAD_COUNT);
      c = c < 0 ? 0 : kmax;
    }
    const int32_t *in = idx + row * kmax;
    int32_t *lo = lo_idx + row * kmax;
    int32_t *hi = hi_idx + row * kmax;
    int nlo = 0, nhi = 0;
    for (int t0 = 0; t0 < c; t0 += 32) {
      const int t = t0 + lane;
      const int j = t < c ? __ldg(in + t) : -1;
      const bool ok = t < c && j >= 0 && j < nk;
      if (t < c && !ok) raise_error(BA_DEVERR_BAD_INDEX);
      const bool is_lo = ok && j < split;
      const bool is_hi = ok && j >= split;
      const unsigned bl = __ballot_sync(full, is_lo);
      const unsigned bh = __ballot_sync(full, is_hi);
      if (is_lo) lo[nlo + __popc(bl & lt_mask)] = j;
      if (is_hi) hi[nhi + __popc(bh & lt_mask)] = j;
      nlo += __popc(bl);
      nhi += __popc(bh);
    }
    for (int t = nlo + lane; t < kmax; t += 32) lo[t] = -1;
    for (int t = nhi + lane; t < kmax; t += 32) hi[t] = -1;
    if (lane == 0) {
      lo_cnt[row] = nlo;
      hi_cnt[row] = nhi;
    }
  }
}

inline cudaError_t launch_split(const int32_t *idx, const int32_t *cnt, int32_t *lo_idx, int32_t *lo_cnt,
                                int32_t *hi_idx, int32_t *hi_cnt, long long n_lists, int kmax, int nk, int split,
                                int num_sms, cudaStream_t stream) {
  long long blocks = (n_lists + 7) / 8;
  const long long cap = static_cast<long long>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  split_lists_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(idx, cnt, lo_idx, lo_cnt, hi_idx, hi_cnt,
                                                                          n_lists, kmax, nk, split);
  return cudaGetLastError();
}

// The complement of each list: the key blocks of [0, nk) it does not hold,
// ascending, -1 padded to ckmax (attention over them, merged with attention
// over the kept blocks, is dense attention: FlashBlock Eq. 5 and Eq. 9). One
// warp per list marks its blocks in a shared-memory bitmap and emits the
// clear bits 32 words at a time with a warp prefix sum over the popcounts.
// Entries outside [0, nk) are ignored and flagged.
constexpr int kComplWarps = 8;
constexpr int kComplMaxWords = 4096 / 32;

__global__ void __launch_bounds__(kComplWarps * 32)
    complement_lists_kernel(const int32_t *__restrict__ idx, const int32_t *__restrict__ cnt,
                            int32_t *__restrict__ c_idx, int32_t *__restrict__ c_cnt, long long n_lists, int kmax,
                            int ckmax, int nk) {
  __shared__ unsigned bits[kComplWarps][kComplMaxWords];
  const unsigned full = 0xFFFFFFFFu;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int words = (nk + 31) >> 5;
  unsigned *bw = bits[warp];
  const long long warps_total = static_cast<long long>(gridDim.x) * kComplWarps;
  for (long long row = blockIdx.x * static_cast<long long>(kComplWarps) + warp; row < n_lists; row += warps_total) {
    for (int w = lane; w < words; w += 32) bw[w] = 0u;
    __syncwarp();
    int c = __ldg(cnt + row);
    if (c < 0 || c > kmax) {
      if (lane == 0) raise_error(BA_DEVERR_BAD_COUNT);
      c = c < 0 ? 0 : kmax;
    }
    const int32_t *in = idx + row * kmax;
    for (int t = lane; t < c; t += 32) {
      const int j = __ldg(in + t);
      if (j >= 0 && j < nk)
        atomicOr(&bw[j >> 5], 1u << (j & 31));
      else
        raise_error(BA_DEVERR_BAD_INDEX);
    }
    __syncwarp();
    int32_t *out = c_idx + row * ckmax;
    int pos = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {
      const int w = w0 + lane;
      unsigned rest = 0u;
      if (w < words) {
        rest = ~bw[w];
        const int valid = nk - (w << 5);                 // bits of this word inside [0, nk)
        if (valid < 32) rest &= (1u << valid) - 1u;
      }
      const int n = __popc(rest);
      int incl = n;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(full, incl, off);
        if (lane >= off) incl += y;
      }
      int at = pos + incl - n;
      while (rest) {                                     // this word's clear blocks, ascending
        const int bit = __ffs(rest) - 1;
        rest &= rest - 1u;
        if (at < ckmax) out[at] = (w << 5) + bit;
        ++at;
      }
      pos += __shfl_sync(full, incl, 31);
    }
    for (int t = pos + lane; t < ckmax; t += 32) out[t] = -1;
    if (lane == 0) c_cnt[row] = pos < ckmax ? pos : ckmax;
    __syncwarp();                                        // bitmap reused by the next list
  }
}

inline cudaError_t launch_complement(const int32_t *idx, const int32_t *cnt, int32_t *c_idx, int32_t *c_cnt,
                                     long long n_lists, int kmax, int ckmax, int nk, int num_sms,
                                     cudaStream_t stream) {
  long long blocks = (n_lists + kComplWarps - 1) / kComplWarps;
  const long long cap = static_cast<long long>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  complement_lists_kernel<<<static_cast<unsigned>(blocks), kComplWarps * 32, 0, stream>>>(idx, cnt, c_idx, c_cnt,
                                                                                         n_lists, kmax, ckmax, nk);
  return cudaGetLastError();
}

}  // namespace baatt
