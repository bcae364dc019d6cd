// attn_tc2.cuh — K8 for 256-row query blocks on a CTA pair: the two 128-row
// halves of a query block run as the two CTAs of a cluster whose MMAs are
// issued once, for M = 256, by tcgen05.mma.cta_group::2.
//
// Operator: the same as attn_tc.cuh ("Efficient Long-Context Modeling in DLMs
// via Block Approximate Sparse Attention": abstract; Figure 4), bf16, d = 128.
//
// With one CTA per 128-row tile, each CTA reads every K and V tile of its
// list into its own shared memory, and every S MMA (M = 128, N = 64) reads
// its whole B operand (64 keys) from there. In a pair the B operand of one
// M = 256 MMA is split between the two CTAs: each holds 32 of the 64 keys of
// a K half block and 64 of the 128 dimensions of a V half block, so each
// SM's shared memory holds and serves half of the K/V bytes.
//   - Both CTAs load their own operand halves with 2-SM TMA loads (no
//     multicast) whose bytes complete on the leader's (rank 0) barriers; the
//     leader's producer arms those barriers with the bytes of both.
//   - The leader's MMA thread issues S = Q K^T (M 256, N 64) and
//     O += P V (M 256, N 128, P from TMEM) for the pair; its commits are
//     multicast to the same barrier in both CTAs (S ready, K/V slot free,
//     PV done, O final).
//   - Each CTA's softmax warps work on its own 128 rows in its own TMEM, as
//     in attn_tc.cuh, and arrive on the leader's P barrier (one arrival per
//     warp, eight in all).
//   - A cluster barrier after the barrier set-up and before teardown keeps
//     either CTA from signalling, or writing into, a CTA that is not there.
// TMEM: S (128 columns) and O (128 columns) in each CTA, allocated for the
// pair (cta_group::2). Every mbarrier wait is bounded, as in attn_tc.cuh.
#pragma once

#include "attn_tc.cuh"

namespace baatt {
namespace tc2 {

using tc::kColO;
using tc::kColS;
using tc::kHalfKeys;
using tc::kRescaleLog2;
using tc::kThreads;
using tc::kTileRows;
using tc::kTmemCols;

constexpr int D = 128;
constexpr uint32_t kQBytes = 2 * 128 * 128;                 // 128 rows x 128 dims bf16, two 64-dim spans
constexpr uint32_t kQSpan = 128 * 128;                      // one span of the Q tile
constexpr int kKRows = kHalfKeys / 2;                       // keys of a K half held by one CTA
constexpr uint32_t kKSpan = 2 * kKRows * 128;               // one 64-dim span of both K halves (8 KB)
constexpr uint32_t kKHalfOff = kKRows * 128;                // half h within a span (4 KB)
constexpr uint32_t kKLoadBytes = kKRows * 128;              // one TMA load of K: 32 rows x 64 dims
constexpr uint32_t kVHalf = kHalfKeys * 128;                // a V half: 64 keys x this CTA's 64 dims (8 KB)
constexpr uint32_t kSmemQ = 0, kSmemK = kQBytes, kSmemV = kQBytes + 2 * kKSpan;
constexpr uint32_t kDynSmem = kSmemV + 2 * kVHalf + 1024;    // + alignment slack
constexpr uint16_t kPairMask = 0x3;

enum Bar {
  Q_FULL = 0,
  K_FULL0, K_FULL1, K_EMPTY0, K_EMPTY1,
  V_FULL0, V_FULL1, V_EMPTY0, V_EMPTY1,
  S_FULL0, S_FULL1, P_FULL0, P_FULL1, PV_DONE0, PV_DONE1,
  O_FINAL, DRAIN, NUM_BARS
};

struct Ctl {
  uint64_t bar[NUM_BARS];
  uint32_t tmem_base;
  int abort;
  int peer_abort;          // (leader) the peer's abort flag at teardown
  int peer_issued[2];      // (leader) the last K / V half the peer's producers loaded
};
constexpr unsigned long long kTeardownWaitNs = 20ull * 1000ull * 1000ull;   // loads land in microseconds

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The shared::cluster address of the same shared-memory location in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on a barrier of either CTA of the pair. What the arrival publishes
// is TMEM written by tcgen05.st, ordered by tcgen05.wait::st and
// tcgen05.fence::before_thread_sync, not generic memory, so CTA-scope release
// suffices; a cluster-scope release would add a memory fence to every arrival.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cta.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// 3-D tiled load into this CTA's shared memory whose bytes complete on the
// barrier at `bar_cluster` (the leader's), for a pair MMA.
__device__ __forceinline__ void tma_load_3d_pair(const CUtensorMap *map, uint32_t dst, uint32_t bar_cluster, int c0,
                                                 int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
      "%5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void mma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the barrier at this offset in both CTAs of the pair when the
// pair's tcgen05 operations issued so far have completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(kPairMask)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "n"(kTmemCols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "n"(kTmemCols) : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// One cluster = one 256-row query block of one (batch, head); CTA rank r
// holds query rows 128r .. 128r+127 of it. Query rows, O, LSE and the merge
// follow attn_tc_kernel (Nq valid rows per head at a stride of q_stride
// rows; nq blocks of 256 rows); key blocks of `kblock` rows (64, 128, 256)
// are one, two or four 64-key halves. The K tensor map has 32-row boxes, the
// Q and V maps 128- and 64-row boxes, all 64 dims wide.
template <typename TO, bool MERGE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 2)
    attn_tc2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const int32_t *__restrict__ kv_idx,
                    const int32_t *__restrict__ kv_cnt, int kmax, TO *O, float *LSE, const float *O_prev,
                    const float *L_prev, int Hq, int Hkv, int N, int Nq, int q_stride, int nq, int nk, int kblock,
                    float scale_log2) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ Ctl ctl;
  // the same offsets in both CTAs: every descriptor the leader issues names
  // the operand halves of both
  const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  const uint32_t sQ = smem_base + kSmemQ, sK = smem_base + kSmemK, sV = smem_base + kSmemV;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  // cluster -> (b, kv head, query block, head within group), the head within
  // the group innermost so consecutive clusters share K/V in L2
  const int G = Hq / Hkv;
  long long pr = blockIdx.x >> 1;
  const int hg = static_cast<int>(pr % G);
  pr /= G;
  const int iq = static_cast<int>(pr % nq);
  pr /= nq;
  const int g = static_cast<int>(pr % Hkv);
  const int b = static_cast<int>(pr / Hkv);
  const int h = g * G + hg;
  const int tile_row0 = iq * 256 + static_cast<int>(rank) * kTileRows;
  const int hpe_log2 = kblock == 256 ? 2 : (kblock == 128 ? 1 : 0), hpe = 1 << hpe_log2;
  const long long list_row = (static_cast<long long>(b) * Hq + h) * nq + iq;
  const int32_t *list = kv_idx + list_row * kmax;
  int cnt = __ldg(kv_cnt + list_row);
  if (cnt < 0 || cnt > kmax) {
    if (threadIdx.x == 0 && leader) raise_error(BA_DEVERR_BAD_COUNT);
    cnt = cnt < 0 ? 0 : kmax;
  }
  const bool has_work = cnt > 0;                     // the same in both CTAs

  if (threadIdx.x == 0) {
    // P_FULL: one arrival per softmax warp of both CTAs
    for (int k = 0; k < NUM_BARS; ++k) mbar_init(smem_u32(&ctl.bar[k]), (k == P_FULL0 || k == P_FULL1) ? 8u : 1u);
    ctl.abort = 0;
    ctl.peer_abort = 0;
    ctl.peer_issued[0] = ctl.peer_issued[1] = -1;
    fence_mbar_init();
  }
  if (warp == 4) {                                   // the same warp in both CTAs
    tmem_alloc_pair(smem_u32(&ctl.tmem_base));
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();                                    // barriers and TMEM of both CTAs exist from here on
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;
  volatile int *abort = &ctl.abort;
  auto bar = [&](int k) { return smem_u32(&ctl.bar[k]); };
  auto lead_bar = [&](int k) { return mapa_rank(smem_u32(&ctl.bar[k]), 0); };

  const int qz = b * Hq + h;
  const int kz = b * Hkv + g;
  int issued = -1;                                   // (producers) last half-block index u loaded

  if (has_work && warp == 4 && lane < 2) {
    // ------------------------------------------------------------ producers
    // lane 0: Q, then this CTA's 32 keys of every K half; lane 1: this CTA's
    // 64 dims of every V half. The leader arms the full barriers with the
    // bytes of both CTAs.
    const bool is_k = lane == 0;
    const int full0 = is_k ? K_FULL0 : V_FULL0, empty0 = is_k ? K_EMPTY0 : V_EMPTY0;
    const uint32_t per_cta = is_k ? 2 * kKLoadBytes : kVHalf;
    tma_prefetch_desc(is_k ? &tm_k : &tm_v);
    if (is_k) {
      tma_prefetch_desc(&tm_q);
      if (leader) mbar_arrive_expect_tx(bar(Q_FULL), 2 * kQBytes);
      for (int sp = 0; sp < 2; ++sp) tma_load_3d_pair(&tm_q, sQ + sp * kQSpan, lead_bar(Q_FULL), 64 * sp, tile_row0, qz);
    }
    bool bad_index = false, bad_order = false;
    tc::UnionCursor cur(list, cnt, nullptr, 0, nk);
    for (int t = 0; !cur.done(); ++t) {
      int j;
      bool in_a, in_b;
      cur.step(j, in_a, in_b, bad_index, bad_order);   // j = 0 when invalid: loaded, then masked
      bool stop = false;
      for (int hh = 0; hh < hpe; ++hh) {
        const int u = t * hpe + hh, hs = u & 1;
        if (u >= 2 && !mbar_wait_bounded(bar(empty0 + hs), ((u >> 1) - 1) & 1, abort)) {
          stop = true;
          break;
        }
        if (leader) mbar_arrive_expect_tx(bar(full0 + hs), 2 * per_cta);
        const int row = j * kblock + hh * kHalfKeys;
        if (is_k) {
          for (int sp = 0; sp < 2; ++sp)
            tma_load_3d_pair(&tm_k, sK + sp * kKSpan + hs * kKHalfOff, lead_bar(full0 + hs), 64 * sp,
                             row + static_cast<int>(rank) * kKRows, kz);
        } else {
          tma_load_3d_pair(&tm_v, sV + hs * kVHalf, lead_bar(full0 + hs), 64 * static_cast<int>(rank), row, kz);
        }
        issued = u;
      }
      if (stop) break;
    }
    if (leader && is_k && bad_index) raise_error(BA_DEVERR_BAD_INDEX);
    if (leader && is_k && bad_order) raise_error(BA_DEVERR_NOT_ASCENDING);
    if (!leader) st_cluster_u32(mapa_rank(smem_u32(&ctl.peer_issued[lane]), 0), static_cast<uint32_t>(issued));
  } else if (has_work && leader && warp == 5 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer (the pair's)
    constexpr uint32_t idesc_qk = idesc_bf16_f32(256, kHalfKeys, 0, 0);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(256, D, 0, 1);
    tc::UnionCursor mc(list, cnt, nullptr, 0, nk);
    int steps_seen = 0;
    auto half_exists = [&](int u) -> bool {
      const int st = u >> hpe_log2;
      while (steps_seen <= st && !mc.done()) {
        int j;
        bool in_a, in_b, bi = false, bo = false;
        mc.step(j, in_a, in_b, bi, bo);
        ++steps_seen;
      }
      return st < steps_seen;
    };
    // S_u = Q K_u^T for all 256 rows: A = each CTA's Q rows, B = each CTA's 32 keys
    auto issue_s = [&](int u) -> bool {
      const int hs = u & 1;
      if (!mbar_wait_bounded(bar(K_FULL0 + hs), (u >> 1) & 1, abort)) return false;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t qoff = (kk >> 2) * kQSpan + (kk & 3) * 32;
        const uint32_t koff = (kk >> 2) * kKSpan + hs * kKHalfOff + (kk & 3) * 32;
        mma_ss_pair(tmem + kColS + hs * kHalfKeys, smem_desc_sw128(sQ + qoff, 16, 1024),
                    smem_desc_sw128(sK + koff, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
      }
      mma_commit_pair(bar(S_FULL0 + hs));
      mma_commit_pair(bar(K_EMPTY0 + hs));
      return true;
    };
    bool ok = mbar_wait_bounded(bar(Q_FULL), 0, abort);
    if (ok) ok = issue_s(0);
    if (ok && half_exists(1)) ok = issue_s(1);
    for (int u = 0; ok && half_exists(u); ++u) {
      const int hs = u & 1;
      if (!mbar_wait_bounded(bar(V_FULL0 + hs), (u >> 1) & 1, abort)) break;
      if (!mbar_wait_bounded(bar(P_FULL0 + hs), (u >> 1) & 1, abort)) break;
      tc_fence_after();
      // O += P_u V_u: A = P from each CTA's TMEM, B = each CTA's 64 dims of V
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        mma_ts_pair(tmem + kColO, tmem + kColS + hs * kHalfKeys + kk * 8,
                    smem_desc_sw128(sV + hs * kVHalf + kk * 2048, 2 * kVHalf, 1024), idesc_pv,
                    (u > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit_pair(bar(V_EMPTY0 + hs));
      mma_commit_pair(bar(PV_DONE0 + hs));
      if (half_exists(u + 2) && !issue_s(u + 2)) break;   // after PV_u: S_{u+2} overwrites P_u
    }
    mma_commit_pair(bar(O_FINAL));
    mma_commit_pair(bar(DRAIN));
    mbar_wait_bounded(bar(DRAIN), 0, nullptr);
  } else if (has_work && !leader && warp == 5 && lane == 0) {
    // the leader's last commit arrives here too: no MMA of the pair is in
    // flight once it has
    mbar_wait_bounded(bar(DRAIN), 0, nullptr);
  } else if (warp < 4) {
    // ------------------------------------------------------------ softmax (this CTA's 128 rows)
    const int row = threadIdx.x;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_off + kColS, tO = tmem + lane_off + kColO;
    const int qrow = tile_row0 + row;
    const bool owned = qrow < Nq;
    const long long orow = static_cast<long long>(qz) * q_stride + qrow;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    int n_keys = 0;
    tc::UnionCursor cur(list, cnt, nullptr, 0, nk);
    for (int u = 0;; ++u) {
      const int hs = u & 1, hh = u & (hpe - 1);
      if (hh == 0) {
        if (cur.done()) break;
        int j;
        bool in_a, in_b, bi = false, bo = false;
        cur.step(j, in_a, in_b, bi, bo);
        n_keys = in_a ? min(kblock, N - j * kblock) : 0;
      }
      const int n_half = min(max(n_keys - hh * kHalfKeys, 0), kHalfKeys);
      bool w = mbar_wait_bounded(bar(S_FULL0 + hs), (u >> 1) & 1, abort);
      if (!__all_sync(0xFFFFFFFFu, w)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tSu = tS + hs * kHalfKeys;
      uint32_t sr[2][32];
      tmem_ld32(tSu, sr[0]);
      tmem_ld32(tSu + 32, sr[1]);
      tmem_ld_wait();
      if (n_half < kHalfKeys) {                        // ragged last block or a skipped entry
#pragma unroll
        for (int q = 0; q < 2; ++q) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (q * 32 + c >= n_half) sr[q][c] = __float_as_uint(-INFINITY);
        }
      }
      const float mx = tc::row_max64(sr) * scale_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (mx - m_used > kRescaleLog2) {
        alpha = ex2_approx(m_used - mx);
        m_used = mx;
        rescale = true;
      }
      const float m_ref = (m_used == -INFINITY) ? 0.f : m_used;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      tc::exp_pack_store(sr, scale_log2, -m_ref, acc, tSu);
      l = l * alpha + (((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7])));
      if (u > 0 && __any_sync(0xFFFFFFFFu, rescale)) {
        const int v = u - 1;
        w = mbar_wait_bounded(bar(PV_DONE0 + (v & 1)), (v >> 1) & 1, abort);
        if (!__all_sync(0xFFFFFFFFu, w)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
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
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(lead_bar(P_FULL0 + hs));
    }
    // ------------------------------------------------------------ epilogue
    bool go = !has_work;
    if (has_work && ok) {
      const bool w = mbar_wait_bounded(bar(O_FINAL), 0, abort);
      go = __all_sync(0xFFFFFFFFu, w);
      if (go) tc_fence_after();
    }
    if (go) {
      const bool has = l > 0.f;
      const float inv = has ? 1.f / l : 0.f;
      const float lse_new = has ? (m_used + __log2f(l)) * 0.6931471805599453f : -INFINITY;
      MergeWeights mw{0.f, 0.f, 0.f, lse_new};
      if constexpr (MERGE) mw = merge_weights(owned ? L_prev[orow] : -INFINITY, lse_new);
      const float *prev = MERGE ? O_prev + orow * D : nullptr;
      uint4 *dst = reinterpret_cast<uint4 *>(O + orow * D);
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        uint32_t orr[32];
        if (has_work) {
          tmem_ld32(tO + q * 32, orr);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) orr[c] = 0u;
        }
        if (owned) {
          float o[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __uint_as_float(orr[c]) * inv;
          if constexpr (MERGE) {
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const float4 pv = *reinterpret_cast<const float4 *>(prev + q * 32 + 4 * v);
              o[4 * v + 0] = merge_value(mw, pv.x, o[4 * v + 0]);
              o[4 * v + 1] = merge_value(mw, pv.y, o[4 * v + 1]);
              o[4 * v + 2] = merge_value(mw, pv.z, o[4 * v + 2]);
              o[4 * v + 3] = merge_value(mw, pv.w, o[4 * v + 3]);
            }
          }
          if constexpr (sizeof(TO) == 2) {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[q * 4 + v] = make_uint4(pack_bf16x2(o[8 * v + 0], o[8 * v + 1]), pack_bf16x2(o[8 * v + 2], o[8 * v + 3]),
                                          pack_bf16x2(o[8 * v + 4], o[8 * v + 5]), pack_bf16x2(o[8 * v + 6], o[8 * v + 7]));
          } else {
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[q * 8 + v] = make_uint4(__float_as_uint(o[4 * v + 0]), __float_as_uint(o[4 * v + 1]),
                                          __float_as_uint(o[4 * v + 2]), __float_as_uint(o[4 * v + 3]));
          }
        }
      }
      if (owned) LSE[orow] = mw.lse;
    }
    tc_fence_before();
  }

  // ------------------------------------------------------------ teardown
  // The peer's loads complete on the leader's barriers. After a timeout the
  // two producers may have stopped at different halves: the leader arms the
  // halves only the peer loaded, then waits (briefly) for the newest loads
  // of both, so no copy is in flight when either CTA exits.
  if (threadIdx.x == 0 && !leader) st_cluster_u32(mapa_rank(smem_u32(&ctl.peer_abort), 0), static_cast<uint32_t>(*abort));
  cluster_sync();
  if (has_work && leader && warp == 4 && lane < 2) {
    const bool is_k = lane == 0;
    const int full0 = is_k ? K_FULL0 : V_FULL0;
    const int pi = ctl.peer_issued[lane];
    for (int u = issued + 1; u <= pi; ++u) mbar_arrive_expect_tx(bar(full0 + (u & 1)), is_k ? 2 * kKLoadBytes : kVHalf);
    if (*abort || ctl.peer_abort || pi != issued) {
      const int top = max(issued, pi);
      for (int u = top; u >= 0 && u > top - 2; --u)
        mbar_wait_bounded(bar(full0 + (u & 1)), (u >> 1) & 1, nullptr, kTeardownWaitNs);
      if (is_k) mbar_wait_bounded(bar(Q_FULL), 0, nullptr, kTeardownWaitNs);
    }
  }
  cluster_sync();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc_pair(tmem);
  }
}

}  // namespace tc2
}  // namespace baatt
