// attn_tc.cuh — K8: block-sparse attention forward on the 5th-generation
// tensor cores (tcgen05 + TMEM), bf16 inputs, d = 64 or 128, query blocks of
// 64, 128 or 256 rows, key blocks of 64, 128 or 256 rows.
//
// Operator: "Efficient Long-Context Modeling in DLMs via Block Approximate
// Sparse Attention" (abstract; Figure 4) — bidirectional attention over the
// kept key blocks only, emitting O and the per-row log-sum-exp; the online
// softmax over blocks is the FlashAttention recurrence the pages compare to.
//
// One CTA = one 128-row query tile of one (batch, head): a 128-row query
// block, half of a 256-row one, or two 64-row ones whose tile attends the
// union of their two lists, each row masking the key blocks its own list
// leaves out (UnionCursor). Two CTAs
// share an SM (up to 96 KB shared memory and 256 TMEM columns each), so one CTA's
// softmax overlaps the other CTA's MMAs. Roles (192 threads):
//   warps 0-3  softmax + correction + epilogue; thread t owns query row t,
//              i.e. TMEM lane t (a warp may only touch its own 32 lanes)
//   warp 4     TMA producers (lane 0: Q and K, lane 1: V), TMEM allocator
//   warp 5     MMA issuer (lane 0)
// Each kept block j (list order) is taken as two 64-key halves, u = 2j + h,
// with their own S columns (h*64 .. h*64+63), so the tensor cores compute
// the next half's scores while the softmax warps work on this half:
//   MMA:  S_u = Q K_u^T             (SS form, N = 64, fp32 in TMEM)
//   SM :  P_u = exp2(s*log2e*S_u - m) as bf16, written back over S_u's first
//         32 columns; the running max m only moves when it grows by more than
//         2^8, and only then is O (TMEM cols 128-255) rescaled, after the
//         MMA that last wrote O has completed
//   MMA:  O += P_u V_u              (TS form: A = P from TMEM, B = V MN-major)
// in the order S_0 S_1 PV_0 S_2 PV_1 S_3 ...: S_{u+2} reuses P_u's columns,
// so it is issued after PV_u. K and V halves are loaded as separate 64-row
// boxes with their own full/empty barriers. Because the key blocks are whole
// 128-row slabs of K and V, the "gather" of the selected blocks is one tile
// load per half block at the block's coordinate.
// Every barrier wait is bounded; a stuck pipeline sets an error bit and the
// CTA drains its copies and MMAs, frees TMEM and exits.
#pragma once

#include "common.cuh"

namespace baatt {
namespace tc {

constexpr int kThreads = 192;
constexpr int kTileRows = 128;
constexpr uint32_t kHalfBytes = 128 * 64 * 2;        // 128 rows x 64 bf16 (one 128-byte swizzle span)
// Per head dimension D (64 or 128): D/64 swizzle spans per 128-row tile.
template <int D>
struct Dims {
  static_assert(D == 64 || D == 128, "head dimension");
  static constexpr int kSpans = D / 64;
  static constexpr uint32_t kTileBytes = kSpans * kHalfBytes;    // 128 x D bf16
  static constexpr uint32_t kSmemQ = 0, kSmemK = kTileBytes, kSmemV = 2 * kTileBytes;
  static constexpr uint32_t kDynSmem = 3 * kTileBytes + 1024;   // + alignment slack
};
constexpr uint32_t dyn_smem_bytes(int d) { return d == 64 ? Dims<64>::kDynSmem : Dims<128>::kDynSmem; }
constexpr int kTmemCols = 256;                       // S (128) + O (D <= 128), a power of two
constexpr uint32_t kColS = 0, kColO = 128;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kHalfKeys = 64;                        // keys per half block
constexpr int kKvBoxRows = kHalfKeys;                // K/V tensor-map box: 64 dims x 64 rows
constexpr uint32_t kHalfRowsBytes = kHalfKeys * 128; // 64 rows of one 64-dim span

// Barriers with a [2] suffix come in two, one per key half h.
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
};

// The key blocks a tile attends, walked in ascending order by every role
// alike: the kept list of its query block, or, for a 128-row tile that holds
// two 64-row query blocks, the union of their two lists. An entry of a list
// is valid when it lies in [0, nb) and above the previous raw entry of that
// list. Each step is one key block: raw entries of equal value in both lists
// make one step; a step valid in neither list is block 0, which the softmax
// masks for every row. Next entries are loaded one step ahead.
struct UnionCursor {
  const int32_t *la, *lb;
  int ca, cb, nb, ta, tb, pa, pb, va, vb;
  __device__ __forceinline__ UnionCursor(const int32_t *a, int na, const int32_t *b, int nbl, int n)
      : la(a), lb(b), ca(na), cb(nbl), nb(n), ta(0), tb(0), pa(-1), pb(-1) {
    va = ca > 0 ? __ldg(la) : 0;
    vb = cb > 0 ? __ldg(lb) : 0;
  }
  __device__ __forceinline__ bool done() const { return ta >= ca && tb >= cb; }
  // the next step's block j and whether it is a valid entry of list A / B;
  // a taken entry out of range or out of order sets bad_index / bad_order
  __device__ __forceinline__ void step(int &j, bool &in_a, bool &in_b, bool &bad_index, bool &bad_order) {
    const bool take_a = ta < ca && (tb >= cb || va <= vb);
    const bool take_b = tb < cb && (ta >= ca || vb <= va);
    int v = 0;
    in_a = in_b = false;
    if (take_a) {
      v = va;
      const bool range = va >= 0 && va < nb, order = ta == 0 || va > pa;
      in_a = range && order;
      bad_index |= !range;
      bad_order |= range && !order;
      pa = va;
      if (++ta < ca) va = __ldg(la + ta);
    }
    if (take_b) {
      v = vb;                                        // equal to A's entry when both are taken
      const bool range = vb >= 0 && vb < nb, order = tb == 0 || vb > pb;
      in_b = range && order;
      bad_index |= !range;
      bad_order |= range && !order;
      pb = vb;
      if (++tb < cb) vb = __ldg(lb + tb);
    }
    j = (in_a || in_b) ? v : 0;
  }
};

// Row max of 64 raw scores held as two 32-column halves: four independent
// chains of 3-input max.
__device__ __forceinline__ float row_max64(const uint32_t (&sr)[2][32]) {
  float m4[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t *v = &sr[k >> 1][(k & 1) * 16];
    float m = fmaxf(__uint_as_float(v[0]), __uint_as_float(v[1]));
#pragma unroll
    for (int c = 2; c < 16; c += 2) m = fmax3(m, __uint_as_float(v[c]), __uint_as_float(v[c + 1]));
    m4[k] = m;
  }
  return fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]);
}

// P = 2^(s*scale_log2 - m) for one row's 64 keys of a half block: packed to
// bf16 pairs and stored over the first 32 of its S columns. The scale and
// shift and the running sums use the packed .f32x2 instructions (two keys per
// instruction, four packed partial sums); the exponentials run on MUFU.
// (Evaluating a share of them on the FMA pipe instead was measured slower
// here: issue slots, not MUFU throughput, bound this loop.)
__device__ __forceinline__ void exp_pack_store(const uint32_t (&sr)[2][32], float scale_log2, float negm,
                                               float (&acc)[8], uint32_t tS) {
  uint32_t pk[32];
  const uint64_t sc2 = pack_f32x2(scale_log2, scale_log2), nm2 = pack_f32x2(negm, negm);
  uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int q = 0; q < 2; ++q) {
#pragma unroll
    for (int c = 0; c < 32; c += 2) {
      const uint64_t x2 = fma_f32x2(pack_u32x2(sr[q][c], sr[q][c + 1]), sc2, nm2);
      const float p0 = ex2_approx(lo_f32(x2));
      const float p1 = ex2_approx(hi_f32(x2));
      acc2[(c >> 1) & 3] = add_f32x2(acc2[(c >> 1) & 3], pack_f32x2(p0, p1));
      pk[q * 16 + (c >> 1)] = pack_bf16x2(p0, p1);
    }
  }
  tmem_st32(tS, pk);
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    acc[2 * a] += lo_f32(acc2[a]);
    acc[2 * a + 1] += hi_f32(acc2[a]);
  }
}

// Query rows: Nq valid rows per head at a stride of q_stride rows (Q, O, LSE,
// O_prev, L_prev), in nq blocks of `block`; keys: N valid rows per KV head
// (the K/V tensor maps). A full call has Nq = N; a call for one range of
// query rows (ba_att_sparse_fwd_rows) has its own Nq and stride.
// TO: output element type, bf16 (final output) or float (a partial that is
// merged later, so the merged result is rounded only once).
// MERGE: the epilogue merges this span's result with an earlier fp32 partial
// (O_prev, L_prev) over a disjoint key set before storing (O and LSE may
// alias O_prev and L_prev when TO is float: each row is read before it is
// written, by the same thread).
template <typename TO, bool MERGE, int D>
__global__ void __launch_bounds__(kThreads, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const int32_t *__restrict__ kv_idx,
                   const int32_t *__restrict__ kv_cnt, int kmax, TO *O, float *LSE, const float *O_prev,
                   const float *L_prev, int Hq, int Hkv, int N, int Nq, int q_stride, int nq, int block,
                   int nk, int kblock, float scale_log2) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ Ctl ctl;
  const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  using DM = Dims<D>;
  const uint32_t sQ = smem_base + DM::kSmemQ, sK = smem_base + DM::kSmemK, sV = smem_base + DM::kSmemV;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // tile -> (b, kv head, 128-row query tile, head within group): consecutive
  // CTAs share a KV head, so its K/V stay hot in L2. A query block of `block`
  // rows (128 or 256) is block/128 query tiles, which share its list; two
  // 64-row query blocks 2t and 2t+1 share one tile, which attends the union
  // of their lists (each row masks the blocks its own list leaves out). A key
  // block of `kblock` rows (64, 128 or 256) is kblock/64 key halves.
  const int G = Hq / Hkv;
  const bool pair = block < kTileRows;               // 64-row blocks, two per tile
  const int qpb = pair ? 1 : block >> 7;
  const long long tiles_per_head = pair ? (nq + 1) / 2 : static_cast<long long>(nq) * qpb;
  const int hpe_log2 = kblock == 256 ? 2 : (kblock == 128 ? 1 : 0), hpe = 1 << hpe_log2;
  long long tile = blockIdx.x;
  const int hg = static_cast<int>(tile % G);
  tile /= G;
  const int it = static_cast<int>(tile % tiles_per_head);                        // query tile within the head
  const int ia = pair ? 2 * it : it / qpb;                                       // its (first) query block
  const int tile_row0 = pair ? it * kTileRows : ia * block + (it % qpb) * kTileRows;
  tile /= tiles_per_head;
  const int g = static_cast<int>(tile % Hkv);
  const int b = static_cast<int>(tile / Hkv);
  const int h = g * G + hg;
  auto list_of = [&](int i, const int32_t *&list) -> int {
    const long long list_row = (static_cast<long long>(b) * Hq + h) * nq + i;
    list = kv_idx + list_row * kmax;
    int c = __ldg(kv_cnt + list_row);
    if (c < 0 || c > kmax) {
      if (threadIdx.x == 0) raise_error(BA_DEVERR_BAD_COUNT);
      c = c < 0 ? 0 : kmax;
    }
    return c;
  };
  const int32_t *list_a = nullptr, *list_b = nullptr;
  const int cnt_a = list_of(ia, list_a);
  const int cnt_b = (pair && ia + 1 < nq) ? list_of(ia + 1, list_b) : 0;
  const bool has_work = cnt_a + cnt_b > 0;

  if (threadIdx.x == 0) {
    for (int k = 0; k < NUM_BARS; ++k) mbar_init(smem_u32(&ctl.bar[k]), (k == P_FULL0 || k == P_FULL1) ? 128u : 1u);
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

  if (has_work && warp == 4 && lane < 2) {
    // ------------------------------------------------------------ producers
    // lane 0: Q, then the K halves; lane 1: the V halves. Half h of block t
    // reuses the slot rows of half h of block t-1 once its MMAs are done.
    const bool is_k = lane == 0;
    const CUtensorMap *tm = is_k ? &tm_k : &tm_v;
    const uint32_t slot = is_k ? sK : sV;
    const int full0 = is_k ? K_FULL0 : V_FULL0, empty0 = is_k ? K_EMPTY0 : V_EMPTY0;
    tma_prefetch_desc(tm);
    if (is_k) {
      tma_prefetch_desc(&tm_q);
      mbar_arrive_expect_tx(bar(Q_FULL), DM::kTileBytes);
#pragma unroll
      for (int sp = 0; sp < DM::kSpans; ++sp) tma_load_3d(&tm_q, sQ + sp * kHalfBytes, bar(Q_FULL), 64 * sp, tile_row0, qz);
    }
    int issued = -1;                    // last half-block index u loaded
    bool bad_index = false, bad_order = false;
    UnionCursor cur(list_a, cnt_a, list_b, cnt_b, nk);
    for (int t = 0; !cur.done(); ++t) {
      int j;
      bool in_a, in_b;
      cur.step(j, in_a, in_b, bad_index, bad_order);   // j = 0 when invalid: loaded, then masked
      bool stop = false;
      for (int hh = 0; hh < hpe; ++hh) {
        const int u = t * hpe + hh, h = u & 1;          // half index; halves alternate the two slots
        if (u >= 2 && !mbar_wait_bounded(bar(empty0 + h), ((u >> 1) - 1) & 1, abort)) {
          stop = true;
          break;
        }
        mbar_arrive_expect_tx(bar(full0 + h), DM::kSpans * kHalfRowsBytes);
        const int row = j * kblock + hh * kHalfKeys;
#pragma unroll
        for (int sp = 0; sp < DM::kSpans; ++sp)
          tma_load_3d(tm, slot + sp * kHalfBytes + h * kHalfRowsBytes, bar(full0 + h), 64 * sp, row, kz);
        issued = u;
      }
      if (stop) break;
    }
    if (is_k && bad_index) raise_error(BA_DEVERR_BAD_INDEX);
    if (is_k && bad_order) raise_error(BA_DEVERR_NOT_ASCENDING);
    if (*abort) {
      // let copies in flight land before the CTA's shared memory goes away
      // (the newest load of each half)
      for (int u = issued; u >= 0 && u > issued - 2; --u) mbar_wait_bounded(bar(full0 + (u & 1)), (u >> 1) & 1, nullptr);
      if (is_k) mbar_wait_bounded(bar(Q_FULL), 0, nullptr);
    }
  } else if (has_work && warp == 5 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kHalfKeys, 0, 0);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
    // whether half u exists: the steps are counted from the same walk
    UnionCursor mc(list_a, cnt_a, list_b, cnt_b, nk);
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
    // S_u = Q K_u^T into S columns h*64..h*64+63
    auto issue_s = [&](int u) -> bool {
      const int h = u & 1;
      if (!mbar_wait_bounded(bar(K_FULL0 + h), (u >> 1) & 1, abort)) return false;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {       // K = D in steps of 16
        const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
        mma_ss(tmem + kColS + h * kHalfKeys, smem_desc_sw128(sQ + off, 16, 1024),
               smem_desc_sw128(sK + off + h * kHalfRowsBytes, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
      }
      mma_commit(bar(S_FULL0 + h));
      mma_commit(bar(K_EMPTY0 + h));
      return true;
    };
    bool ok = mbar_wait_bounded(bar(Q_FULL), 0, abort);
    if (ok) ok = issue_s(0);                           // a tile with work has at least one step
    if (ok && half_exists(1)) ok = issue_s(1);
    for (int u = 0; ok && half_exists(u); ++u) {
      const int h = u & 1;
      if (!mbar_wait_bounded(bar(V_FULL0 + h), (u >> 1) & 1, abort)) break;
      if (!mbar_wait_bounded(bar(P_FULL0 + h), (u >> 1) & 1, abort)) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {            // 64 keys = 4 x 16; P packs 2 keys per column
        mma_ts(tmem + kColO, tmem + kColS + h * kHalfKeys + kk * 8,
               smem_desc_sw128(sV + (4 * h + kk) * 2048, kHalfBytes, 1024), idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(bar(V_EMPTY0 + h));
      mma_commit(bar(PV_DONE0 + h));
      if (half_exists(u + 2) && !issue_s(u + 2)) break;   // after PV_u: S_{u+2} overwrites P_u
    }
    mma_commit(bar(O_FINAL));
    mma_commit(bar(DRAIN));
    mbar_wait_bounded(bar(DRAIN), 0, nullptr);
  } else if (warp < 4) {
    // ------------------------------------------------------------ softmax
    const int row = threadIdx.x;                       // TMEM lane = query row in tile
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_off + kColS, tO = tmem + lane_off + kColO;
    const int qrow = tile_row0 + row;
    const bool owned = qrow < Nq;                      // a token (rows past the range are not written)
    const bool row_in_b = pair && row >= 64;           // this row's block is the tile's second one
    const long long orow = static_cast<long long>(qz) * q_stride + qrow;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    int n_keys = 0;
    UnionCursor cur(list_a, cnt_a, list_b, cnt_b, nk);
    for (int u = 0;; ++u) {
      const int h = u & 1, hh = u & (hpe - 1);          // S slot; half within the key block
      if (hh == 0) {
        if (cur.done()) break;
        int j;
        bool in_a, in_b, bi = false, bo = false;
        cur.step(j, in_a, in_b, bi, bo);
        n_keys = (row_in_b ? in_b : in_a) ? min(kblock, N - j * kblock) : 0;
      }
      const int n_half = min(max(n_keys - hh * kHalfKeys, 0), kHalfKeys);
      bool w = mbar_wait_bounded(bar(S_FULL0 + h), (u >> 1) & 1, abort);
      if (!__all_sync(0xFFFFFFFFu, w)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tSu = tS + h * kHalfKeys;
      uint32_t sr[2][32];
      tmem_ld32(tSu, sr[0]);
      tmem_ld32(tSu + 32, sr[1]);
      tmem_ld_wait();
      if (n_half < kHalfKeys) {                        // ragged last block, a block of the other list, a skipped entry
#pragma unroll
        for (int q = 0; q < 2; ++q) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (q * 32 + c >= n_half) sr[q][c] = __float_as_uint(-INFINITY);
        }
      }
      const float mx = row_max64(sr) * scale_log2;   // scale > 0 keeps the order
      float alpha = 1.f;
      bool rescale = false;
      if (mx - m_used > kRescaleLog2) {                // false when both are -inf
        alpha = ex2_approx(m_used - mx);               // 0 when m_used = -inf
        m_used = mx;
        rescale = true;
      }
      const float m_ref = (m_used == -INFINITY) ? 0.f : m_used;
      const float negm = -m_ref;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      exp_pack_store(sr, scale_log2, negm, acc, tSu);
      l = l * alpha + (((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7])));
      if (u > 0 && __any_sync(0xFFFFFFFFu, rescale)) {
        // O holds halves 0..u-1 once PV_{u-1} has completed (PV_{u-2} did
        // before S_u was issued)
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
      mbar_arrive(bar(P_FULL0 + h));
    }
    // ------------------------------------------------------------ epilogue
    // (no listed block: nothing was accumulated; this span contributes O = 0,
    // LSE = -inf, and a merge passes the earlier partial through)
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

  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc<kTmemCols>(tmem);
  }
}


}  // namespace tc
}  // namespace baatt
