// attn_tc.cuh — K8: block-sparse attention forward on the 5th-generation
// tensor cores (tcgen05 + TMEM), bf16 inputs, d = 128, block = 128.
//
// Operator: "Efficient Long-Context Modeling in DLMs via Block Approximate
// Sparse Attention" (abstract; Figure 4) — bidirectional attention over the
// kept key blocks only, emitting O and the per-row log-sum-exp; the online
// softmax over blocks is the FlashAttention recurrence the pages compare to.
//
// One CTA = one 128-row query block of one (batch, head) = one tile. Two CTAs
// share an SM (96 KB shared memory and 256 TMEM columns each), so one CTA's
// softmax overlaps the other CTA's MMAs. Roles (192 threads):
//   warps 0-3  softmax + correction + epilogue; thread t owns query row t,
//              i.e. TMEM lane t (a warp may only touch its own 32 lanes)
//   warp 4     TMA producer (lane 0) and TMEM allocator (whole warp)
//   warp 5     MMA issuer (lane 0)
// Per kept block j (list order):
//   TMA:  K_j, V_j  -> shared memory, 128B-swizzled, one 2-D box per 64 dims
//   MMA:  S = Q K_j^T               (SS form, fp32 accumulator in TMEM cols 0-127)
//   SM :  P = exp2(s*log2e*S - m) as bf16, written back over S (cols 0-63);
//         running max m only moves when it grows by more than 2^8, and only
//         then is O (TMEM cols 128-255) rescaled
//   MMA:  O += P V_j                (TS form: A = P from TMEM, B = V MN-major)
// Because the key blocks are whole 128-row slabs of K and V, the "gather" of
// the selected blocks is one tile load per block at the block's coordinate.
// Every barrier wait is bounded; a stuck pipeline sets an error bit and the
// CTA drains its copies and MMAs, frees TMEM and exits.
#pragma once

#include "common.cuh"

namespace baatt {
namespace tc {

constexpr int kThreads = 192;
constexpr int kTileRows = 128;
constexpr int kHeadDim = 128;
constexpr uint32_t kHalfBytes = 128 * 64 * 2;        // 128 rows x 64 bf16 (one 128-byte swizzle span)
constexpr uint32_t kTileBytes = 2 * kHalfBytes;      // 128 x 128 bf16
constexpr uint32_t kSmemQ = 0, kSmemK = kTileBytes, kSmemV = 2 * kTileBytes;
constexpr uint32_t kDynSmem = 3 * kTileBytes + 1024; // + alignment slack
constexpr int kTmemCols = 256;
constexpr uint32_t kColS = 0, kColO = 128;
constexpr float kRescaleLog2 = 8.0f;

enum Bar { Q_FULL = 0, K_FULL, K_EMPTY, V_FULL, V_EMPTY, S_FULL, P_FULL, O_FINAL, DRAIN, NUM_BARS };

struct Ctl {
  uint64_t bar[NUM_BARS];
  uint32_t tmem_base;
  int abort;
};

// Validity of list entry t, computed identically by every role from the raw
// list: inside [0, nb) and strictly above the previous raw entry.
__device__ __forceinline__ bool entry_ok(const int32_t *list, int t, int nb, int &j) {
  j = __ldg(list + t);
  if (j < 0 || j >= nb) return false;
  if (t > 0 && j <= __ldg(list + t - 1)) return false;
  return true;
}

// P = 2^(s*scale_log2 - m) for one row: packed to bf16 pairs and stored
// over the S columns 64 keys at a time; the fp32 values are summed into 8
// independent partial sums. (Evaluating a share of the exponentials on the
// FMA pipe instead of MUFU was measured slower here: issue slots, not MUFU
// throughput, bound this loop.)
__device__ __forceinline__ void exp_pack_store(const uint32_t (&sr)[4][32], float scale_log2, float negm,
                                               float (&acc)[8], uint32_t tS) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint32_t pk[32];
#pragma unroll
    for (int qq = 0; qq < 2; ++qq) {
      const int q = 2 * half + qq;
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float x0 = fmaf(__uint_as_float(sr[q][c]), scale_log2, negm);
        const float x1 = fmaf(__uint_as_float(sr[q][c + 1]), scale_log2, negm);
        const float p0 = ex2_approx(x0);
        const float p1 = ex2_approx(x1);
        acc[c & 7] += p0;
        acc[(c & 7) + 1] += p1;
        pk[qq * 16 + (c >> 1)] = pack_bf16x2(p0, p1);
      }
    }
    tmem_st32(tS + half * 32, pk);
  }
}

// TO: output element type, bf16 (final output) or float (a partial that is
// merged later, so the merged result is rounded only once).
template <typename TO>
__global__ void __launch_bounds__(kThreads, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const int32_t *__restrict__ kv_idx,
                   const int32_t *__restrict__ kv_cnt, int kmax, TO *__restrict__ O,
                   float *__restrict__ LSE, int Hq, int Hkv, int N, int N_alloc, int nb, float scale_log2) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ Ctl ctl;
  const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  const uint32_t sQ = smem_base + kSmemQ, sK = smem_base + kSmemK, sV = smem_base + kSmemV;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // tile -> (b, kv head, query block, head within group): consecutive CTAs
  // share a KV head, so its K/V stay hot in L2.
  const int G = Hq / Hkv;
  long long tile = blockIdx.x;
  const int hg = static_cast<int>(tile % G);
  tile /= G;
  const int i = static_cast<int>(tile % nb);
  tile /= nb;
  const int g = static_cast<int>(tile % Hkv);
  const int b = static_cast<int>(tile / Hkv);
  const int h = g * G + hg;
  const long long list_row = (static_cast<long long>(b) * Hq + h) * nb + i;
  const int32_t *list = kv_idx + list_row * kmax;
  int cnt = __ldg(kv_cnt + list_row);
  if (cnt < 0 || cnt > kmax) {
    if (threadIdx.x == 0) raise_error(BA_DEVERR_BAD_COUNT);
    cnt = cnt < 0 ? 0 : kmax;
  }

  if (threadIdx.x == 0) {
    for (int k = 0; k < NUM_BARS; ++k) mbar_init(smem_u32(&ctl.bar[k]), k == P_FULL ? 128u : 1u);
    ctl.abort = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc<kTmemCols>(smem_u32(&ctl.tmem_base));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;
  volatile int *abort = &ctl.abort;
  auto bar = [&](int k) { return smem_u32(&ctl.bar[k]); };

  const int qz = b * Hq + h;          // row of the [B*H] head axis in the tensor maps
  const int kz = b * Hkv + g;

  if (cnt > 0 && warp == 4 && lane == 0) {
    // ------------------------------------------------------------ producer
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    mbar_arrive_expect_tx(bar(Q_FULL), kTileBytes);
    tma_load_3d(&tm_q, sQ, bar(Q_FULL), 0, i * kTileRows, qz);
    tma_load_3d(&tm_q, sQ + kHalfBytes, bar(Q_FULL), 64, i * kTileRows, qz);
    int k_issued = -1, v_issued = -1;
    bool bad_index = false, bad_order = false;
    for (int t = 0; t < cnt; ++t) {
      int j;
      if (!entry_ok(list, t, nb, j)) {
        const int raw = __ldg(list + t);
        if (raw < 0 || raw >= nb) bad_index = true; else bad_order = true;
        j = 0;                            // load a valid block; softmax masks it out
      }
      if (t > 0 && !mbar_wait_bounded(bar(K_EMPTY), (t - 1) & 1, abort)) break;
      mbar_arrive_expect_tx(bar(K_FULL), kTileBytes);
      tma_load_3d(&tm_k, sK, bar(K_FULL), 0, j * kTileRows, kz);
      tma_load_3d(&tm_k, sK + kHalfBytes, bar(K_FULL), 64, j * kTileRows, kz);
      k_issued = t;
      if (t > 0 && !mbar_wait_bounded(bar(V_EMPTY), (t - 1) & 1, abort)) break;
      mbar_arrive_expect_tx(bar(V_FULL), kTileBytes);
      tma_load_3d(&tm_v, sV, bar(V_FULL), 0, j * kTileRows, kz);
      tma_load_3d(&tm_v, sV + kHalfBytes, bar(V_FULL), 64, j * kTileRows, kz);
      v_issued = t;
    }
    if (bad_index) raise_error(BA_DEVERR_BAD_INDEX);
    if (bad_order) raise_error(BA_DEVERR_NOT_ASCENDING);
    if (*abort) {
      // let copies in flight land before the CTA's shared memory goes away
      if (k_issued >= 0) mbar_wait_bounded(bar(K_FULL), k_issued & 1, nullptr);
      if (v_issued >= 0) mbar_wait_bounded(bar(V_FULL), v_issued & 1, nullptr);
      mbar_wait_bounded(bar(Q_FULL), 0, nullptr);
    }
  } else if (cnt > 0 && warp == 5 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
    bool ok = mbar_wait_bounded(bar(Q_FULL), 0, abort);
    for (int t = 0; ok && t < cnt; ++t) {
      if (!mbar_wait_bounded(bar(K_FULL), t & 1, abort)) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {            // K = 128 = 8 x 16
        const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
        mma_ss(tmem + kColS, smem_desc_sw128(sQ + off, 16, 1024), smem_desc_sw128(sK + off, 16, 1024), idesc_qk,
               kk > 0 ? 1u : 0u);
      }
      mma_commit(bar(S_FULL));
      mma_commit(bar(K_EMPTY));
      if (!mbar_wait_bounded(bar(V_FULL), t & 1, abort)) break;
      if (!mbar_wait_bounded(bar(P_FULL), t & 1, abort)) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {            // 128 keys = 8 x 16; P packs 2 keys per column
        mma_ts(tmem + kColO, tmem + kColS + kk * 8, smem_desc_sw128(sV + kk * 2048, kHalfBytes, 1024), idesc_pv,
               (t > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(bar(V_EMPTY));
    }
    mma_commit(bar(O_FINAL));
    mma_commit(bar(DRAIN));
    mbar_wait_bounded(bar(DRAIN), 0, nullptr);
  } else if (warp < 4) {
    // ------------------------------------------------------------ softmax
    const int row = threadIdx.x;                       // TMEM lane = query row in tile
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_off + kColS, tO = tmem + lane_off + kColO;
    const int qrow = i * kTileRows + row;
    const long long orow = static_cast<long long>(qz) * N_alloc + qrow;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < cnt; ++t) {
      int j;
      const bool valid = entry_ok(list, t, nb, j);
      const int n_keys = valid ? min(kTileRows, N - j * kTileRows) : 0;
      bool w = mbar_wait_bounded(bar(S_FULL), t & 1, abort);
      if (!__all_sync(0xFFFFFFFFu, w)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld32(tS + q * 32, sr[q]);
      tmem_ld_wait();
      if (n_keys < kTileRows) {                        // ragged last block or a skipped entry (rare)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (q * 32 + c >= n_keys) sr[q][c] = __float_as_uint(-INFINITY);
        }
      }
      // Row max of the raw scores: 4 independent chains of 3-input max.
      float mxp[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        mxp[q] = fmaxf(__uint_as_float(sr[q][0]), __uint_as_float(sr[q][31]));
#pragma unroll
        for (int c = 1; c < 31; c += 2)
          mxp[q] = fmax3(mxp[q], __uint_as_float(sr[q][c]), __uint_as_float(sr[q][c + 1]));
      }
      const float mx = fmaxf(fmax3(mxp[0], mxp[1], mxp[2]), mxp[3]) * scale_log2;   // scale > 0 keeps the order
      float alpha = 1.f;
      bool rescale = false;
      if (mx - m_used > kRescaleLog2) {                // false when both are -inf
        alpha = ex2_approx(m_used - mx);               // 0 when m_used = -inf
        m_used = mx;
        rescale = true;
      }
      const float m_ref = (m_used == -INFINITY) ? 0.f : m_used;
      // p = 2^(s*scale_log2 - m): one packed FMA per pair, 8 independent
      // packed partial sums.
      const float negm = -m_ref;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      exp_pack_store(sr, scale_log2, negm, acc, tS);
      l = l * alpha + (((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7])));
      if (t > 0 && __any_sync(0xFFFFFFFFu, rescale)) {
        // O holds blocks 0..t-1 (their MMAs completed before S_t did)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t orr[32];
          tmem_ld32(tO + q * 32, orr);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
          tmem_st32(tO + q * 32, orr);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(P_FULL));
    }
    if (cnt == 0) {
      if (qrow < N) {
        uint4 *dst = reinterpret_cast<uint4 *>(O + orow * kHeadDim);
#pragma unroll
        for (int v = 0; v < kHeadDim * static_cast<int>(sizeof(TO)) / 16; ++v) dst[v] = make_uint4(0, 0, 0, 0);
        LSE[orow] = -INFINITY;
      }
    } else if (ok) {
      const bool w = mbar_wait_bounded(bar(O_FINAL), 0, abort);
      if (__all_sync(0xFFFFFFFFu, w)) {
        tc_fence_after();
        const bool has = l > 0.f;
        const float inv = has ? 1.f / l : 0.f;
        uint4 *dst = reinterpret_cast<uint4 *>(O + orow * kHeadDim);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t orr[32];
          tmem_ld32(tO + q * 32, orr);
          tmem_ld_wait();
          if (qrow < N) {
            if constexpr (sizeof(TO) == 2) {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                uint4 pkt;
                pkt.x = pack_bf16x2(__uint_as_float(orr[8 * v + 0]) * inv, __uint_as_float(orr[8 * v + 1]) * inv);
                pkt.y = pack_bf16x2(__uint_as_float(orr[8 * v + 2]) * inv, __uint_as_float(orr[8 * v + 3]) * inv);
                pkt.z = pack_bf16x2(__uint_as_float(orr[8 * v + 4]) * inv, __uint_as_float(orr[8 * v + 5]) * inv);
                pkt.w = pack_bf16x2(__uint_as_float(orr[8 * v + 6]) * inv, __uint_as_float(orr[8 * v + 7]) * inv);
                dst[q * 4 + v] = pkt;
              }
            } else {
#pragma unroll
              for (int v = 0; v < 8; ++v) {
                uint4 pkt;
                pkt.x = __float_as_uint(__uint_as_float(orr[4 * v + 0]) * inv);
                pkt.y = __float_as_uint(__uint_as_float(orr[4 * v + 1]) * inv);
                pkt.z = __float_as_uint(__uint_as_float(orr[4 * v + 2]) * inv);
                pkt.w = __float_as_uint(__uint_as_float(orr[4 * v + 3]) * inv);
                dst[q * 8 + v] = pkt;
              }
            }
          }
        }
        if (qrow < N) LSE[orow] = has ? (m_used + __log2f(l)) * 0.6931471805599453f : -INFINITY;
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc<kTmemCols>(tmem);
  }
}

}  // namespace tc
}  // namespace baatt
