// select.cuh — K7: norm sorting, the per-row exact top-k of the block scores.
//
// "Efficient Long-Context Modeling in DLMs via Block Approximate Sparse
// Attention" (abstract; "Core claim"; Figure 2): key blocks are scored in
// the downsampled block space, the pooled score is corrected with diagonal
// Q/K variances, blocks are sorted and the top fraction is kept.
//
// The scores S~[i,j] are written by the score kernels (select_tc.cuh, tensor
// cores); this file ranks each (batch, head, query block) row of that map.
// One warp per row selects the top k exactly on order-preserving 32-bit keys
// of the fp32 scores (topk_row_keys: a sampled key window, 8-bit radix
// passes, then direct ranking of at most 32 candidates); equal scores go to
// the lower block index, and the kept indices are emitted ascending. Rows of
// up to 1024 keys are held in registers lane-major (topk_rows_lm_kernel: each
// lane a contiguous run of columns, 16-byte loads, kept columns emitted from
// per-lane bit masks); longer rows are re-read from global memory
// (topk_rows_long_kernel, topk_row_warp). topk_variant_kernel serves the
// selection variants of ba_att_select_ex (shared per GQA group, forced
// diagonal, cumulative softmax share: topk_row_mass); it holds its rows
// chunk-major (lane l has columns c*32 + l).
#pragma once

#include "common.cuh"
#include "pdl.cuh"

namespace baatt {

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

// The same exact selection for a row of at most 32*KPL keys; key(c) is the
// order key of column c*32 + l for lane l (so column order is chunk-major),
// held in registers or in shared memory.
// The per-warp histogram (256 counters) lives in shared memory at hist_s.
//
//  1. Bracket: 32 keys sampled across the chunks are sorted across the warp
//     (bitonic), and the samples 8 ranks either side of the expected rank of
//     the k-th key give a key window [lo, hi]. One histogram pass over the
//     window at a bin width of 2^shift, (hi - lo) >> shift < 256, counts the
//     keys above the window separately. When the k-th key falls inside the
//     window its bin is the candidate range; otherwise (a poor sample) the
//     candidate range is the whole row [min, max].
//  2. While the candidate range holds more than 32 keys, 8-bit radix passes
//     narrow it from its top bit.
//  3. At most 32 candidates are ranked directly, one per lane, in the order
//     (key descending, column ascending); the rank-(need-1) candidate is the
//     exact cut. A range narrowed down to one key value instead keeps its
//     equal keys in column order.
// Scores of a row are concentrated in a narrow band with a long upper tail,
// so a window placed by the sample spreads the band over many bins where the
// row's full range would put most keys into one bin.
// Lane-major emission: lane l holds columns l*KPL .. l*KPL+KPL-1 and bit c of
// `mask` marks column l*KPL + c as kept. Writes every kept column in
// ascending order (lanes in order, each its set bits in order) and returns the
// total, identical in every lane.
template <int KPL>
__device__ __forceinline__ int emit_lane_runs(uint32_t mask, int lane, int32_t *__restrict__ out_idx) {
  const int n = __popc(mask);
  int incl = n;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += y;
  }
  int w = incl - n;
  for (uint32_t m = mask; m != 0u; m &= m - 1u) out_idx[w++] = lane * KPL + (__ffs(m) - 1);
  return __shfl_sync(0xFFFFFFFFu, incl, 31);
}

template <int KPL, bool LM = false, typename KeyAt>
__device__ __forceinline__ void topk_row_keys(const KeyAt &key, int nk, int k, int32_t *__restrict__ out_idx,
                                              int kmax, int32_t *__restrict__ out_cnt, uint32_t hist_s, int lane) {
  const unsigned full = 0xFFFFFFFFu;
  const unsigned lt_mask = (1u << lane) - 1u;
  // column of key c of this lane: chunk-major (c*32 + lane) or lane-major
  // (lane*KPL + c, each lane a contiguous run of columns)
  auto colof = [&](int c) { return LM ? lane * KPL + c : c * 32 + lane; };
  if (k >= nk) {
    for (int j = lane; j < kmax; j += 32) out_idx[j] = j < nk ? j : -1;
    if (lane == 0) *out_cnt = nk;
    return;
  }
  auto hist_zero = [&]() {
    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(hist_s + 32u * lane), "r"(0u) : "memory");
    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(hist_s + 32u * lane + 16u), "r"(0u) : "memory");
  };
  // Bins in descending order: lane l reads bins 255-8l .. 248-8l; the bin
  // where the running count first reaches `want` (0..255, or -1 if the bins
  // hold fewer keys), the count of keys above it and its own count.
  auto hist_find = [&](int want, int &digit, int &above, int &in_bin) {
    uint32_t h[8];
    const uint32_t a = hist_s + 4u * (248u - 8u * lane);
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(a));
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(h[4]), "=r"(h[5]), "=r"(h[6]), "=r"(h[7])
                 : "r"(a + 16u));
    int local = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) local += static_cast<int>(h[t]);
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(full, incl, off);
      if (lane >= off) incl += y;
    }
    const unsigned hit = __ballot_sync(full, incl >= want);
    digit = -1;
    if (hit == 0u) return;
    const int src = __ffs(hit) - 1;
    int dg = 0, ab = 0, ib = 0;
    if (lane == src) {
      int c = incl - local;
#pragma unroll
      for (int t = 7; t >= 0; --t) {                   // h[7] is the highest bin of this lane
        const int n = static_cast<int>(h[t]);
        if (dg == 0 && c + n >= want) {
          dg = 248 - 8 * lane + t + 1;                 // +1 so that 0 means "not yet"
          ab = c;
          ib = n;
        }
        c += n;
      }
    }
    digit = __shfl_sync(full, dg, src) - 1;
    above = __shfl_sync(full, ab, src);
    in_bin = __shfl_sync(full, ib, src);
  };

  // candidate range: keys in [base, base + 2^nbits) (nbits 32: every key >= base)
  uint32_t base = 0u;
  int nbits = 32, need = k, in_bin = nk;
  bool bracketed = false;
  if (KPL >= 2 && nk >= 64) {
    uint32_t smp = key(0);
    if constexpr (LM) {
      // the first key of every lane holding keys (evenly spaced columns);
      // lanes past the row's end take a copy of one of them
      const int nvl = (nk + KPL - 1) / KPL;
      smp = __shfl_sync(full, smp, lane < nvl ? lane : lane % nvl);
    } else {
      const int cs = lane % KPL;
#pragma unroll
      for (int c = 1; c < KPL; ++c)
        if (c == cs && c * 32 + lane < nk) smp = key(c);
    }
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {       // bitonic sort, descending across lanes
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const uint32_t o = __shfl_xor_sync(full, smp, stride);
        const bool take_max = ((lane & stride) == 0) == ((lane & size) == 0 || size == 32);
        smp = take_max ? max(smp, o) : min(smp, o);
      }
    }
    const int rq = min(31, static_cast<int>((static_cast<long long>(k) * 32) / nk));
    const uint32_t hi = __shfl_sync(full, smp, max(rq - 8, 0));
    const uint32_t lo = __shfl_sync(full, smp, min(rq + 8, 31));
    const int shift = max(0, 24 - static_cast<int>(__clz(hi - lo)));
    hist_zero();
    __syncwarp();
    int n_above = 0;
#pragma unroll
    for (int c = 0; c < KPL; ++c) {
      if (colof(c) < nk && key(c) >= lo) {
        const uint32_t bin = (key(c) - lo) >> shift;
        if (bin > 255u)
          ++n_above;
        else
          red_shared_add(hist_s + 4u * bin, 1u);
      }
    }
    n_above = __reduce_add_sync(full, n_above);
    __syncwarp();
    if (n_above < k) {
      int digit, ab, ib;
      hist_find(k - n_above, digit, ab, ib);
      if (digit >= 0) {
        bracketed = true;
        base = lo + (static_cast<uint32_t>(digit) << shift);
        nbits = shift;
        need = k - n_above - ab;
        in_bin = ib;
      }
    }
    __syncwarp();
  }
  if (!bracketed) {
    uint32_t umin = 0xFFFFFFFFu, umax = 0u;
#pragma unroll
    for (int c = 0; c < KPL; ++c) {
      if (colof(c) < nk) {
        umin = min(umin, key(c));
        umax = max(umax, key(c));
      }
    }
    umin = __reduce_min_sync(full, umin);
    umax = __reduce_max_sync(full, umax);
    base = umin;
    nbits = 32 - static_cast<int>(__clz(umax - umin));    // 0 when every key is equal
    need = k;
    in_bin = nk;
  }
  // in the range: nbits < 32 needs the offset below 2^nbits
  auto in_range = [&](uint32_t x, int j) {
    return j < nk && x >= base && (nbits >= 32 || ((x - base) >> nbits) == 0u);
  };

  uint32_t prefix = 0u, mask = 0u;                      // over the offset x - base
  for (int shift = ((nbits + 7) & ~7) - 8; shift >= 0 && in_bin > 32; shift -= 8) {
    hist_zero();
    __syncwarp();
#pragma unroll
    for (int c = 0; c < KPL; ++c) {
      const uint32_t v = key(c) - base;
      if (in_range(key(c), colof(c)) && (v & mask) == prefix)
        red_shared_add(hist_s + 4u * ((v >> shift) & 255u), 1u);
    }
    __syncwarp();
    int digit, ab, ib;
    hist_find(need, digit, ab, ib);                     // the range holds >= need keys: always found
    prefix |= static_cast<uint32_t>(digit) << shift;
    mask |= 255u << shift;
    need -= ab;
    in_bin = ib;
    __syncwarp();
  }

  int pos = 0;
  if (in_bin <= 32) {
    // gather the remaining candidates' (key, column) pairs, one per lane
    int cnt = 0;
#pragma unroll
    for (int c = 0; c < KPL; ++c) {
      const int j = colof(c);
      const bool cand = in_range(key(c), j) && ((key(c) - base) & mask) == prefix;
      const unsigned cb = __ballot_sync(full, cand);
      if (cand) {
        const uint32_t slot = hist_s + 8u * static_cast<uint32_t>(cnt + __popc(cb & lt_mask));
        asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(slot), "r"(key(c)), "r"(j) : "memory");
      }
      cnt += __popc(cb);
    }
    __syncwarp();
    uint32_t cv = 0u;
    int cj = 0x7FFFFFFF;
    if (lane < cnt)
      asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(cv), "=r"(cj) : "r"(hist_s + 8u * lane));
    int rank = 0;
    for (int t = 0; t < cnt; ++t) {
      const uint32_t tv = __shfl_sync(full, cv, t);
      const int tj = __shfl_sync(full, cj, t);
      rank += (tv > cv || (tv == cv && tj < cj)) ? 1 : 0;
    }
    const int cut = __ffs(__ballot_sync(full, lane < cnt && rank == need - 1)) - 1;
    const uint32_t thr_u = __shfl_sync(full, cv, cut);
    const int thr_j = __shfl_sync(full, cj, cut);
    if constexpr (LM) {
      uint32_t km = 0u;
#pragma unroll
      for (int c = 0; c < KPL; ++c) {
        const int j = colof(c);
        if (j < nk && (key(c) > thr_u || (key(c) == thr_u && j <= thr_j))) km |= 1u << c;
      }
      pos = emit_lane_runs<KPL>(km, lane, out_idx);
    } else {
#pragma unroll
      for (int c = 0; c < KPL; ++c) {
        const int j = c * 32 + lane;
        const bool kept = j < nk && (key(c) > thr_u || (key(c) == thr_u && j <= thr_j));
        const unsigned kb = __ballot_sync(full, kept);
        if (kept) out_idx[pos + __popc(kb & lt_mask)] = j;
        pos += __popc(kb);
      }
    }
  } else if constexpr (LM) {
    // the range is one key value (the k-th largest): every larger key and the
    // first `need` equal keys in column order (lanes hold ascending runs)
    const uint32_t thr = base + prefix;
    uint32_t gm = 0u, em = 0u;
#pragma unroll
    for (int c = 0; c < KPL; ++c) {
      if (colof(c) < nk) {
        if (key(c) > thr) gm |= 1u << c;
        if (key(c) == thr) em |= 1u << c;
      }
    }
    const int ne = __popc(em);
    int eincl = ne;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(full, eincl, off);
      if (lane >= off) eincl += y;
    }
    int room = need - (eincl - ne);                    // equal keys this lane may still take
    uint32_t take = 0u;
    for (uint32_t m = em; m != 0u && room > 0; m &= m - 1u, --room) take |= m & (0u - m);
    pos = emit_lane_runs<KPL>(gm | take, lane, out_idx);
  } else {
    const uint32_t thr = base + prefix;                 // the range is one key value: the k-th largest
    int eq_seen = 0;
#pragma unroll
    for (int c = 0; c < KPL; ++c) {
      const int j = c * 32 + lane;
      const bool in = j < nk;
      const bool gt = in && key(c) > thr;
      const bool eq = in && key(c) == thr;
      const unsigned eqb = __ballot_sync(full, eq);
      const bool kept = gt || (eq && eq_seen + __popc(eqb & lt_mask) < need);
      const unsigned kb = __ballot_sync(full, kept);
      if (kept) out_idx[pos + __popc(kb & lt_mask)] = j;
      pos += __popc(kb);
      eq_seen += __popc(eqb);
    }
  }
  for (int j = pos + lane; j < kmax; j += 32) out_idx[j] = -1;
  if (lane == 0) *out_cnt = pos;
}

// Row held in registers: lane l has the keys of columns c*32 + l in u[c].
template <int KPL>
__device__ __forceinline__ void topk_row_regs(const uint32_t (&u)[KPL], int nk, int k, int32_t *__restrict__ out_idx,
                                              int kmax, int32_t *__restrict__ out_cnt, uint32_t hist_s, int lane) {
  topk_row_keys<KPL>([&](int c) { return u[c]; }, nk, k, out_idx, kmax, out_cnt, hist_s, lane);
}

// One warp per (batch, head, query block) row of the score map; rows up to
// 32*KPL keys are held in registers, longer rows are re-read per pass.
constexpr int kTopkWarps = 8;

// Rows longer than 1024 keys: one warp per row, re-read from global memory
// on every pass (topk_row_warp).
__global__ void __launch_bounds__(kTopkWarps * 32) topk_rows_long_kernel(const float *__restrict__ scores, int nk,
                                                                         int k, int32_t *__restrict__ kv_idx, int kmax,
                                                                         int32_t *__restrict__ kv_cnt, long long rows) {
  __shared__ __align__(16) unsigned hist[kTopkWarps][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = blockIdx.x * static_cast<long long>(kTopkWarps) + warp;
  if (row >= rows) return;
  topk_row_warp(scores + row * nk, nk, k, kv_idx + row * kmax, kmax, kv_cnt + row, &hist[warp][0], lane);
}

// Lane-major rows of up to 32*KPL keys in registers: lane l holds the
// contiguous columns l*KPL .. l*KPL+KPL-1, fetched with 16-byte loads when the
// rows are 16-byte aligned; persistent warps prefetch the next row while the
// current one is selected. The selection is topk_row_keys in lane-major mode
// (same exact result as the chunk-major kernels).
template <int KPL>
__global__ void __launch_bounds__(kTopkWarps * 32) topk_rows_lm_kernel(const float *__restrict__ scores, int nk,
                                                                       int k, int32_t *__restrict__ kv_idx, int kmax,
                                                                       int32_t *__restrict__ kv_cnt, long long rows) {
  __shared__ __align__(16) unsigned hist[kTopkWarps][256];   // also holds (key, column) pairs
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  long long row = blockIdx.x * static_cast<long long>(kTopkWarps) + warp;
  const long long stride = static_cast<long long>(gridDim.x) * kTopkWarps;
  const bool vec = (nk & 3) == 0 && (lane + 1) * KPL <= nk;
  float nxt[KPL];
  auto fetch = [&](long long r) {
    const float *src = scores + r * nk + lane * KPL;
    if (r < rows && vec) {
#pragma unroll
      for (int q = 0; q < KPL / 4; ++q) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(src) + q);
        nxt[4 * q] = v.x;
        nxt[4 * q + 1] = v.y;
        nxt[4 * q + 2] = v.z;
        nxt[4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < KPL; ++c) nxt[c] = (r < rows && lane * KPL + c < nk) ? __ldg(src + c) : 0.f;
    }
  };
  pdl_wait();                                       // the score map is complete from here on
  fetch(row);
  for (; row < rows; row += stride) {
    uint32_t u[KPL];
#pragma unroll
    for (int c = 0; c < KPL; ++c) u[c] = order_key(nxt[c]);
    fetch(row + stride);
    topk_row_keys<KPL, true>([&](int c) { return u[c]; }, nk, k, kv_idx + row * kmax, kmax, kv_cnt + row,
                             smem_u32(&hist[warp][0]), lane);
  }
}

template <int KPL>
inline cudaError_t launch_topk_lm(const float *scores, int nk, int k, int32_t *idx, int kmax, int32_t *cnt,
                                  long long rows, int num_sms, cudaStream_t stream, bool dependent) {
  const int threads = kTopkWarps * 32;
  int per_sm = 0;
  const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_rows_lm_kernel<KPL>, threads, 0);
  if (e != cudaSuccess) return e;
  long long grid = (rows + kTopkWarps - 1) / kTopkWarps;
  const long long slots = static_cast<long long>(num_sms) * (per_sm > 0 ? per_sm : 1);
  grid = grid < slots ? grid : slots;
  if (dependent)
    return launch_dependent(topk_rows_lm_kernel<KPL>, dim3(static_cast<unsigned>(grid)), dim3(threads), 0, stream,
                            scores, nk, k, idx, kmax, cnt, rows);
  topk_rows_lm_kernel<KPL><<<static_cast<unsigned>(grid), threads, 0, stream>>>(scores, nk, k, idx, kmax, cnt, rows);
  return cudaGetLastError();
}

template <int KPL>
inline cudaError_t launch_topk_kpl(const float *scores, int nk, int k, int32_t *idx, int kmax, int32_t *cnt,
                                   long long rows, int num_sms, cudaStream_t stream, bool dependent = false) {
  if constexpr (KPL > 0) {
    return launch_topk_lm<KPL>(scores, nk, k, idx, kmax, cnt, rows, num_sms, stream, dependent);
  } else {
    const long long grid = (rows + kTopkWarps - 1) / kTopkWarps;
    topk_rows_long_kernel<<<static_cast<unsigned>(grid), kTopkWarps * 32, 0, stream>>>(scores, nk, k, idx, kmax, cnt,
                                                                                      rows);
    return cudaGetLastError();
  }
}

// Selection by cumulative share: keep the shortest prefix of the ranking
// (key descending, column ascending) whose softmax share
// exp(x_j - max) / sum_j exp(x_j - max) reaches tau (at least one block).
// e_j and their sum are fp32; the cut key t* is the largest key whose
// mass of keys >= t* still reaches tau*Z, found by bisection over the
// 32-bit key space with warp-wide sums; of the keys equal to t* (equal x,
// hence equal e) the first ones in column order are taken until the share
// is reached. All lanes hold identical sums (xor-butterfly), so every lane
// takes the same branch.
template <int KPL>
__device__ __forceinline__ void topk_row_mass(const float (&x)[KPL], const uint32_t (&u)[KPL], int nk, float tau,
                                              int32_t *__restrict__ out_idx, int kmax, int32_t *__restrict__ out_cnt,
                                              int lane) {
  const unsigned full = 0xFFFFFFFFu;
  const unsigned lt_mask = (1u << lane) - 1u;
  auto wsum = [&](float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(full, v, off);
    return v;
  };
  float mx = -INFINITY;
  uint32_t umin = 0xFFFFFFFFu, umax = 0u;
#pragma unroll
  for (int c = 0; c < KPL; ++c) {
    if (c * 32 + lane < nk) {
      mx = fmaxf(mx, x[c]);
      umin = min(umin, u[c]);
      umax = max(umax, u[c]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(full, mx, off));
  umin = __reduce_min_sync(full, umin);
  umax = __reduce_max_sync(full, umax);
  float e[KPL];
  float part = 0.f;
#pragma unroll
  for (int c = 0; c < KPL; ++c) {
    e[c] = (c * 32 + lane < nk) ? expf(x[c] - mx) : 0.f;
    part += e[c];
  }
  const float Z = wsum(part);
  const float target = tau * Z;
  // largest t with mass(keys >= t) >= target: invariant mass(>= lo) >= target > mass(>= hi)
  uint64_t lo = umin, hi = static_cast<uint64_t>(umax) + 1u;
  while (hi - lo > 1u) {
    const uint64_t mid = lo + ((hi - lo) >> 1);
    float m = 0.f;
#pragma unroll
    for (int c = 0; c < KPL; ++c) m += (c * 32 + lane < nk && u[c] >= mid) ? e[c] : 0.f;
    if (wsum(m) >= target) lo = mid; else hi = mid;
  }
  const uint32_t thr = static_cast<uint32_t>(lo);
  float above = 0.f, e_eq = 0.f;
  int n_eq = 0;
#pragma unroll
  for (int c = 0; c < KPL; ++c) {
    const bool in = c * 32 + lane < nk;
    if (in && u[c] > thr) above += e[c];
    if (in && u[c] == thr) {
      e_eq = e[c];
      ++n_eq;
    }
  }
  above = wsum(above);
  e_eq = __shfl_sync(full, e_eq, __ffs(__ballot_sync(full, e_eq > 0.f || n_eq > 0)) - 1);
  n_eq = __reduce_add_sync(full, n_eq);
  int take = n_eq;                                      // equal keys needed, in column order
  if (e_eq > 0.f) {
    const float need = target - above;
    take = static_cast<int>(ceilf(need / e_eq));
    take = take < 1 ? 1 : (take > n_eq ? n_eq : take);
  }
  int pos = 0, eq_seen = 0;
#pragma unroll
  for (int c = 0; c < KPL; ++c) {
    const int j = c * 32 + lane;
    const bool in = j < nk;
    const bool gt = in && u[c] > thr;
    const bool eq = in && u[c] == thr;
    const unsigned eqb = __ballot_sync(full, eq);
    const bool kept = gt || (eq && eq_seen + __popc(eqb & lt_mask) < take);
    const unsigned kb = __ballot_sync(full, kept);
    if (kept && pos + __popc(kb & lt_mask) < kmax) out_idx[pos + __popc(kb & lt_mask)] = j;
    pos += __popc(kb);
    eq_seen += __popc(eqb);
  }
  for (int j = pos + lane; j < kmax; j += 32) out_idx[j] = -1;
  if (lane == 0) *out_cnt = pos < kmax ? pos : kmax;
}

// Selection variants (the plain top-k above is the default):
//   group > 1       the `group` query heads of a KV group share one selection,
//                   ranked by the mean of their scores (one warp per
//                   (batch, KV head, query block); the list is written to
//                   every head of the group);
//   force_diagonal  key block i always ranks first for query block i;
//   by_mass         keep the shortest top-ranked prefix whose softmax share
//                   reaches tau (topk_row_mass) instead of k blocks.
// Rows of at most 1024 keys, held in registers.
struct TopkVariant {
  int group;            // query heads per selection (1: none shared)
  int heads;            // Hq
  int nq;               // query blocks per head
  bool force_diagonal;
  bool by_mass;         // keep the shortest prefix reaching the share tau (instead of k blocks)
  float tau;
};

template <int KPL>
__global__ void __launch_bounds__(kTopkWarps * 32) topk_variant_kernel(const float *__restrict__ scores, int nk, int k,
                                                                       int32_t *__restrict__ kv_idx, int kmax,
                                                                       int32_t *__restrict__ kv_cnt, long long sel_rows,
                                                                       TopkVariant var) {
  __shared__ __align__(16) unsigned hist[kTopkWarps][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long stride = static_cast<long long>(gridDim.x) * kTopkWarps;
  const int kv_heads = var.heads / var.group;
  const float inv_group = 1.f / static_cast<float>(var.group);
  for (long long r = blockIdx.x * static_cast<long long>(kTopkWarps) + warp; r < sel_rows; r += stride) {
    const int i = static_cast<int>(r % var.nq);
    const long long bg = r / var.nq;                   // b*Hkv + g (shared) or b*Hq + h
    const long long first_row = var.group > 1
                                    ? ((bg / kv_heads) * var.heads + (bg % kv_heads) * var.group) * var.nq + i
                                    : r;
    float acc[KPL];
#pragma unroll
    for (int c = 0; c < KPL; ++c) acc[c] = 0.f;
    for (int hh = 0; hh < var.group; ++hh) {           // heads of the group are consecutive score rows nq apart
      const float *srow = scores + (first_row + static_cast<long long>(hh) * var.nq) * nk;
#pragma unroll
      for (int c = 0; c < KPL; ++c) {
        const int j = c * 32 + lane;
        if (j < nk) acc[c] += __ldg(srow + j);
      }
    }
    uint32_t u[KPL];
#pragma unroll
    for (int c = 0; c < KPL; ++c) {
      const int j = c * 32 + lane;
      if (var.group > 1) acc[c] *= inv_group;
      u[c] = order_key(acc[c]);
      if (var.force_diagonal && j == i) u[c] = 0xFFFFFFFFu;
    }
    int32_t *out = kv_idx + first_row * kmax;
    if (var.by_mass)
      topk_row_mass<KPL>(acc, u, nk, var.tau, out, kmax, kv_cnt + first_row, lane);
    else
      topk_row_regs<KPL>(u, nk, k, out, kmax, kv_cnt + first_row, smem_u32(&hist[warp][0]), lane);
    __syncwarp();
    for (int hh = 1; hh < var.group; ++hh) {           // the same list for the other heads of the group
      const long long orow = first_row + static_cast<long long>(hh) * var.nq;
      for (int t = lane; t < kmax; t += 32) kv_idx[orow * kmax + t] = out[t];
      if (lane == 0) kv_cnt[orow] = kv_cnt[first_row];
    }
  }
}

template <int KPL>
inline cudaError_t launch_topk_variant_kpl(const float *scores, int nk, int k, int32_t *idx, int kmax, int32_t *cnt,
                                           long long sel_rows, const TopkVariant &var, int num_sms,
                                           cudaStream_t stream) {
  const int threads = kTopkWarps * 32;
  int per_sm = 0;
  const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_variant_kernel<KPL>, threads, 0);
  if (e != cudaSuccess) return e;
  long long grid = (sel_rows + kTopkWarps - 1) / kTopkWarps;
  const long long slots = static_cast<long long>(num_sms) * (per_sm > 0 ? per_sm : 1);
  grid = grid < slots ? grid : slots;
  topk_variant_kernel<KPL><<<static_cast<unsigned>(grid), threads, 0, stream>>>(scores, nk, k, idx, kmax, cnt,
                                                                                sel_rows, var);
  return cudaGetLastError();
}

// sel_rows = B * (Hq / group) * nq
inline cudaError_t launch_topk_variant(const float *scores, int nk, int k, int32_t *idx, int kmax, int32_t *cnt,
                                       long long sel_rows, const TopkVariant &var, int num_sms, cudaStream_t stream) {
  if (nk <= 256) return launch_topk_variant_kpl<8>(scores, nk, k, idx, kmax, cnt, sel_rows, var, num_sms, stream);
  if (nk <= 512) return launch_topk_variant_kpl<16>(scores, nk, k, idx, kmax, cnt, sel_rows, var, num_sms, stream);
  return launch_topk_variant_kpl<32>(scores, nk, k, idx, kmax, cnt, sel_rows, var, num_sms, stream);
}

// dependent: launch the lane-major kernel as a programmatic dependent of the
// kernel before it on the stream (which must be the one writing `scores`).
inline cudaError_t launch_topk(const float *scores, int nk, int k, int32_t *idx, int kmax, int32_t *cnt,
                               long long rows, int num_sms, cudaStream_t stream, bool dependent = false) {
  if (nk <= 256) return launch_topk_kpl<8>(scores, nk, k, idx, kmax, cnt, rows, num_sms, stream, dependent);
  if (nk <= 512) return launch_topk_kpl<16>(scores, nk, k, idx, kmax, cnt, rows, num_sms, stream, dependent);
  if (nk <= 1024) return launch_topk_kpl<32>(scores, nk, k, idx, kmax, cnt, rows, num_sms, stream, dependent);
  return launch_topk_kpl<0>(scores, nk, k, idx, kmax, cnt, rows, num_sms, stream);
}

}  // namespace baatt
