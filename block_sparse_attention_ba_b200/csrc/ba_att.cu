// ba_att.cu — host side of the C ABI declared in include/ba_att.h.
//
// Every entry point validates its arguments on the host first and launches
// nothing on a bad argument. Launches are asynchronous on the caller's
// stream; no call synchronises except ba_att_get_device_error. No call
// allocates device memory: the global state is the device error word (a
// __device__ variable), a cache of per-device SM counts, per device the two
// copy streams and events of the host-buffer pipeline, and the static
// scratch of ba_att_forward_host_noalloc, a __device__ array that the module
// reserves on every device where it loads, whichever entry points are used.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "stats.cuh"
#include "select.cuh"
#include "select_tc.cuh"
#include "merge.cuh"
#include "attn_simt.cuh"
#include "attn_tc.cuh"
#include "attn_tc2.cuh"

using namespace baatt;

namespace {

constexpr int kMaxDevices = 64;

int num_sms_of_current_device() {
  static int cache[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ba_status check_shape(const ba_att_shape *s) {
  if (s == nullptr) return BA_ERR_INVALID_ARG;
  if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->N < 1 || s->N_alloc < s->N) return BA_ERR_INVALID_ARG;
  if (s->Hq % s->Hkv != 0) return BA_ERR_INVALID_ARG;
  if (s->B > 65535 || s->Hq > 65535) return BA_ERR_UNSUPPORTED;
  if (s->dtype != BA_DTYPE_F32 && s->dtype != BA_DTYPE_BF16) return BA_ERR_INVALID_ARG;
  if (s->d != 64 && s->d != 128) return BA_ERR_UNSUPPORTED;
  if (s->block < 16 || s->block > 256 || s->block % 16 != 0) return BA_ERR_UNSUPPORTED;
  if (s->block_k != 0 && (s->block_k < 16 || s->block_k > 256 || s->block_k % 16 != 0)) return BA_ERR_UNSUPPORTED;
  if (std::isnan(s->sm_scale) || std::isinf(s->sm_scale)) return BA_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(s->B) * (s->Hq > s->Hkv ? s->Hq : s->Hkv) * s->N_alloc;
  if (rows > (1LL << 36)) return BA_ERR_UNSUPPORTED;
  return BA_OK;
}

// query blocks (block rows) and key blocks (kblock rows)
int nblocks(const ba_att_shape *s) { return (s->N + s->block - 1) / s->block; }
int kblock(const ba_att_shape *s) { return s->block_k > 0 ? s->block_k : s->block; }
int nkblocks(const ba_att_shape *s) { return (s->N + kblock(s) - 1) / kblock(s); }

float effective_scale(const ba_att_shape *s) {
  return s->sm_scale > 0.f ? s->sm_scale : 1.0f / std::sqrt(static_cast<float>(s->d));
}

ba_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BA_OK : BA_ERR_CUDA; }

// ---- tensor maps (driver entry point fetched through the runtime, so the
// library links no libcuda stub)
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [BH, rows, d] bf16 head-major tensor read in boxes of 64 dims x box_rows
// rows; rows >= N_valid read as zeros.
bool make_head_map(CUtensorMap *map, const void *ptr, int d, int N_valid, int N_alloc, long long BH, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N_valid), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2u, static_cast<cuuint64_t>(N_alloc) * d * 2u};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool use_tensor_core_path(const ba_att_shape *s) {
  const int kb = s->block_k > 0 ? s->block_k : s->block;
  return s->dtype == BA_DTYPE_BF16 && (s->d == 128 || s->d == 64) &&
         (s->block == 64 || s->block == 128 || s->block == 256) && (kb == 64 || kb == 128 || kb == 256);
}

__global__ void bounded_wait_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_bounded(smem_u32(&bar), 0, nullptr, limit_ns);
}

}  // namespace

extern "C" {

const char *ba_att_version(void) { return "0.1.0 sm_100a"; }

const char *ba_att_status_string(ba_status st) {
  switch (st) {
    case BA_OK: return "BA_OK";
    case BA_ERR_INVALID_ARG: return "BA_ERR_INVALID_ARG";
    case BA_ERR_UNSUPPORTED: return "BA_ERR_UNSUPPORTED";
    case BA_ERR_MISALIGNED: return "BA_ERR_MISALIGNED";
    case BA_ERR_CUDA: return "BA_ERR_CUDA";
    case BA_ERR_DEVICE: return "BA_ERR_DEVICE";
    case BA_ERR_TIMEOUT: return "BA_ERR_TIMEOUT";
  }
  return "BA_ERR_UNKNOWN";
}

int32_t ba_att_num_blocks(const ba_att_shape *shape) {
  if (check_shape(shape) != BA_OK) return -1;
  return nblocks(shape);
}

int32_t ba_att_num_key_blocks(const ba_att_shape *shape) {
  if (check_shape(shape) != BA_OK) return -1;
  return nkblocks(shape);
}

int32_t ba_att_keep_count(const ba_att_shape *shape, double keep) {
  if (check_shape(shape) != BA_OK) return -1;
  if (!(keep > 0.f && keep <= 1.f)) return -1;
  const int nk = nkblocks(shape);
  const double kk = std::ceil(static_cast<double>(keep) * nk - 1e-9);
  int k = static_cast<int>(kk);
  if (k < 1) k = 1;
  if (k > nk) k = nk;
  return k;
}

ba_status ba_att_stats(const ba_att_shape *s, const void *Q, const void *K, float *q_mean, float *q_var,
                       float *k_mean, float *k_var, ba_stream_t stream) {
  ba_status st = check_shape(s);
  if (st != BA_OK) return st;
  if (!Q || !K || !q_mean || !q_var || !k_mean || !k_var) return BA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(q_mean) || !aligned16(q_var) || !aligned16(k_mean) ||
      !aligned16(k_var))
    return BA_ERR_MISALIGNED;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const int sms = num_sms_of_current_device();
  cudaError_t e;
  if (s->dtype == BA_DTYPE_BF16) {
    auto q = static_cast<const __nv_bfloat16 *>(Q);
    auto k = static_cast<const __nv_bfloat16 *>(K);
    e = s->d == 128 ? launch_stats<__nv_bfloat16, 128>(q, k, q_mean, q_var, k_mean, k_var, s->B, s->Hq, s->Hkv, s->N,
                                                       s->N_alloc, s->block, kblock(s), sms, cs)
                    : launch_stats<__nv_bfloat16, 64>(q, k, q_mean, q_var, k_mean, k_var, s->B, s->Hq, s->Hkv, s->N,
                                                      s->N_alloc, s->block, kblock(s), sms, cs);
  } else {
    auto q = static_cast<const float *>(Q);
    auto k = static_cast<const float *>(K);
    e = s->d == 128 ? launch_stats<float, 128>(q, k, q_mean, q_var, k_mean, k_var, s->B, s->Hq, s->Hkv, s->N,
                                               s->N_alloc, s->block, kblock(s), sms, cs)
                    : launch_stats<float, 64>(q, k, q_mean, q_var, k_mean, k_var, s->B, s->Hq, s->Hkv, s->N,
                                              s->N_alloc, s->block, kblock(s), sms, cs);
  }
  return from_cuda(e);
}

ba_status ba_att_select_ex(const ba_att_shape *s, double keep, uint32_t flags, const float *q_mean,
                           const float *q_var, const float *k_mean, const float *k_var, int32_t *kv_idx,
                           int32_t *kv_cnt, int32_t kmax, float *block_scores, ba_stream_t stream) {
  ba_status st = check_shape(s);
  if (st != BA_OK) return st;
  constexpr uint32_t kKnown =
      BA_SELECT_NO_VAR_PRODUCT | BA_SELECT_FORCE_DIAGONAL | BA_SELECT_SHARED_GQA | BA_SELECT_BY_MASS;
  if (flags & ~kKnown) return BA_ERR_INVALID_ARG;
  if (!q_mean || !q_var || !k_mean || !k_var || !kv_idx || !kv_cnt || !block_scores) return BA_ERR_INVALID_ARG;
  if (!aligned16(q_mean) || !aligned16(q_var) || !aligned16(k_mean) || !aligned16(k_var) || !aligned16(kv_idx) ||
      !aligned16(kv_cnt) || !aligned16(block_scores))
    return BA_ERR_MISALIGNED;
  const int k = ba_att_keep_count(s, keep);
  if (k < 1) return BA_ERR_INVALID_ARG;
  if (kmax < k) return BA_ERR_INVALID_ARG;
  const int nb = nkblocks(s);                     // score row length
  if (nb > 4096 || nblocks(s) > 1048576) return BA_ERR_UNSUPPORTED;
  // the forced diagonal pairs query block i with key block i: equal block sizes only
  if ((flags & BA_SELECT_FORCE_DIAGONAL) && kblock(s) != s->block) return BA_ERR_UNSUPPORTED;
  if ((flags & (BA_SELECT_FORCE_DIAGONAL | BA_SELECT_SHARED_GQA | BA_SELECT_BY_MASS)) && nb > 1024)
    return BA_ERR_UNSUPPORTED;
  if (flags & BA_SELECT_BY_MASS) {
    if (flags & BA_SELECT_FORCE_DIAGONAL) return BA_ERR_UNSUPPORTED;
    if (kmax < nb) return BA_ERR_INVALID_ARG;
  }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const float scale = effective_scale(s);
  const int sms = num_sms_of_current_device();
  const float tau = static_cast<float>(keep);
  cudaError_t e = s->d == 128 ? launch_select_tc<128>(q_mean, q_var, k_mean, k_var, kv_idx, kv_cnt, block_scores, s->B,
                                                      s->Hq, s->Hkv, s->N, s->block, kblock(s), k, kmax, scale, flags, tau, sms,
                                                      cs)
                              : launch_select_tc<64>(q_mean, q_var, k_mean, k_var, kv_idx, kv_cnt, block_scores, s->B,
                                                     s->Hq, s->Hkv, s->N, s->block, kblock(s), k, kmax, scale, flags, tau, sms,
                                                     cs);
  return from_cuda(e);
}

ba_status ba_att_select(const ba_att_shape *s, double keep, const float *q_mean, const float *q_var,
                        const float *k_mean, const float *k_var, int32_t *kv_idx, int32_t *kv_cnt, int32_t kmax,
                        float *block_scores, ba_stream_t stream) {
  return ba_att_select_ex(s, keep, 0u, q_mean, q_var, k_mean, k_var, kv_idx, kv_cnt, kmax, block_scores, stream);
}

}  // extern "C"

// ---------------------------------------------------------------- one-call selector

namespace {
// [6 planes][rows][d] bf16 feature array read in boxes of 64 dims x box_rows rows.
bool make_feat_map(CUtensorMap *map, const void *ptr, int d, long long rows, int box_rows = selft::kTile) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), 6u};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2u, static_cast<cuuint64_t>(rows) * d * 2u};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

long long feat_rows_q(const ba_att_shape *s) { return static_cast<long long>(s->B) * s->Hq * nblocks(s); }
long long feat_rows_k(const ba_att_shape *s) { return static_cast<long long>(s->B) * s->Hkv * nkblocks(s); }

// Whether the shape takes the feature path (else the selector is the plain
// ba_att_stats + ba_att_select sequence).
bool selector_feature_path(const ba_att_shape *s) {
  return feat_rows_q(s) + selft::kTile < 0x7FFFFFFFLL;
}

// Workspace of ba_att_selector: the score features, then room for the score
// map when the caller passes none; each part 256-byte aligned.
size_t ws_align(long long x) { return static_cast<size_t>((x + 255) & ~255LL); }
long long feat_bytes(const ba_att_shape *s) { return 6LL * (feat_rows_q(s) + feat_rows_k(s)) * s->d * 2; }
long long score_map_bytes(const ba_att_shape *s) {
  return static_cast<long long>(s->B) * s->Hq * nblocks(s) * nkblocks(s) * 4;
}
size_t ws_scores_offset(const ba_att_shape *s) { return ws_align(feat_bytes(s)); }

template <int D>
cudaError_t launch_select_feat(const CUtensorMap &mq, const CUtensorMap &mk, float *scores, const ba_att_shape *s,
                               int nq, int nk, int sms, cudaStream_t cs) {
  const int n_tq = (nq + selft::kTile - 1) / selft::kTile, n_tk = (nk + selft::kTile - 1) / selft::kTile;
  const long long n_tiles = static_cast<long long>(s->B) * s->Hq * n_tq * n_tk;
  cudaError_t e = cudaFuncSetAttribute(selft::select_feat_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(selft::kDynSmem));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(n_tiles < sms ? n_tiles : sms);
  // a programmatic dependent of the statistics pass that writes its features
  return launch_dependent(selft::select_feat_kernel<D>, dim3(grid), dim3(selft::kThreads), selft::kDynSmem, cs, mq, mk,
                          scores, s->Hq, s->Hkv, s->N, kblock(s), nq, nk, n_tiles, n_tq, n_tk);
}
}  // namespace

extern "C" {

int64_t ba_att_selector_workspace(const ba_att_shape *s) {
  if (check_shape(s) != BA_OK) return -1;
  return static_cast<int64_t>(ws_scores_offset(s) + ws_align(score_map_bytes(s)));
}

ba_status ba_att_selector(const ba_att_shape *s, double keep, const void *Q, const void *K, float *q_mean,
                          float *q_var, float *k_mean, float *k_var, void *workspace, float *block_scores,
                          int32_t *kv_idx, int32_t *kv_cnt, int32_t kmax, ba_stream_t stream) {
  ba_status st = check_shape(s);
  if (st != BA_OK) return st;
  if (!Q || !K || !q_mean || !q_var || !k_mean || !k_var || !workspace || !kv_idx || !kv_cnt)
    return BA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(q_mean) || !aligned16(q_var) || !aligned16(k_mean) ||
      !aligned16(k_var) || !aligned16(workspace) || !aligned16(block_scores) || !aligned16(kv_idx) ||
      !aligned16(kv_cnt))
    return BA_ERR_MISALIGNED;
  const int k = ba_att_keep_count(s, keep);
  if (k < 1 || kmax < k) return BA_ERR_INVALID_ARG;
  const int nq = nblocks(s), nk = nkblocks(s);
  if (nk > 4096 || nq > 1048576) return BA_ERR_UNSUPPORTED;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  // without a caller map the scores live in the workspace (read back by the top-k, never returned)
  float *scores = block_scores != nullptr ? block_scores : reinterpret_cast<float *>(ws + ws_scores_offset(s));
  if (!selector_feature_path(s)) {
    st = ba_att_stats(s, Q, K, q_mean, q_var, k_mean, k_var, stream);
    return st == BA_OK ? ba_att_select(s, keep, q_mean, q_var, k_mean, k_var, kv_idx, kv_cnt, kmax, scores, stream)
                       : st;
  }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const int sms = num_sms_of_current_device();
  const float scale = effective_scale(s);
  auto *fq = reinterpret_cast<__nv_bfloat16 *>(ws);
  auto *fk = fq + 6 * feat_rows_q(s) * s->d;
  const FeatOut feat{fq, fk, scale, 0.5f * scale * scale, feat_rows_q(s), feat_rows_k(s)};
  cudaError_t e;
  if (s->dtype == BA_DTYPE_BF16) {
    auto q = static_cast<const __nv_bfloat16 *>(Q);
    auto kk = static_cast<const __nv_bfloat16 *>(K);
    e = s->d == 128 ? launch_stats<__nv_bfloat16, 128>(q, kk, q_mean, q_var, k_mean, k_var, s->B, s->Hq, s->Hkv, s->N,
                                                       s->N_alloc, s->block, kblock(s), sms, cs, feat)
                    : launch_stats<__nv_bfloat16, 64>(q, kk, q_mean, q_var, k_mean, k_var, s->B, s->Hq, s->Hkv, s->N,
                                                      s->N_alloc, s->block, kblock(s), sms, cs, feat);
  } else {
    auto q = static_cast<const float *>(Q);
    auto kk = static_cast<const float *>(K);
    e = s->d == 128 ? launch_stats<float, 128>(q, kk, q_mean, q_var, k_mean, k_var, s->B, s->Hq, s->Hkv, s->N,
                                               s->N_alloc, s->block, kblock(s), sms, cs, feat)
                    : launch_stats<float, 64>(q, kk, q_mean, q_var, k_mean, k_var, s->B, s->Hq, s->Hkv, s->N,
                                              s->N_alloc, s->block, kblock(s), sms, cs, feat);
  }
  if (e != cudaSuccess) return from_cuda(e);
  CUtensorMap mq, mk;
  if (!make_feat_map(&mq, fq, s->d, feat_rows_q(s)) || !make_feat_map(&mk, fk, s->d, feat_rows_k(s)))
    return BA_ERR_CUDA;
  e = s->d == 128 ? launch_select_feat<128>(mq, mk, scores, s, nq, nk, sms, cs)
                  : launch_select_feat<64>(mq, mk, scores, s, nq, nk, sms, cs);
  if (e != cudaSuccess) return from_cuda(e);
  return from_cuda(launch_topk(scores, nk, k, kv_idx, kmax, kv_cnt, static_cast<long long>(s->B) * s->Hq * nq,
                               sms, cs, /*dependent=*/true));
}

ba_status ba_att_topk(const float *block_scores, int64_t rows, int32_t nk, int32_t k, int32_t *kv_idx,
                      int32_t *kv_cnt, int32_t kmax, ba_stream_t stream) {
  if (!block_scores || !kv_idx || !kv_cnt) return BA_ERR_INVALID_ARG;
  if (!aligned16(block_scores) || !aligned16(kv_idx) || !aligned16(kv_cnt)) return BA_ERR_MISALIGNED;
  if (rows < 1 || nk < 1 || k < 1 || kmax < k) return BA_ERR_INVALID_ARG;
  if (nk > 4096) return BA_ERR_UNSUPPORTED;
  return from_cuda(launch_topk(block_scores, nk, k, kv_idx, kmax, kv_cnt, rows, num_sms_of_current_device(),
                               reinterpret_cast<cudaStream_t>(stream)));
}

ba_status ba_att_complement_lists(const ba_att_shape *s, const int32_t *kv_idx, const int32_t *kv_cnt, int32_t kmax,
                                  int32_t *c_idx, int32_t *c_cnt, int32_t c_kmax, ba_stream_t stream) {
  ba_status st = check_shape(s);
  if (st != BA_OK) return st;
  if (!kv_idx || !kv_cnt || !c_idx || !c_cnt) return BA_ERR_INVALID_ARG;
  if (!aligned16(kv_idx) || !aligned16(kv_cnt) || !aligned16(c_idx) || !aligned16(c_cnt)) return BA_ERR_MISALIGNED;
  const int nb = nkblocks(s);
  if (nb > kComplMaxWords * 32) return BA_ERR_UNSUPPORTED;
  if (kmax < 1 || c_kmax < nb) return BA_ERR_INVALID_ARG;
  const long long n_lists = static_cast<long long>(s->B) * s->Hq * nblocks(s);
  return from_cuda(launch_complement(kv_idx, kv_cnt, c_idx, c_cnt, n_lists, kmax, c_kmax, nb,
                                     num_sms_of_current_device(), reinterpret_cast<cudaStream_t>(stream)));
}

ba_status ba_att_split_lists(const ba_att_shape *s, int32_t split_block, const int32_t *kv_idx, const int32_t *kv_cnt,
                             int32_t kmax, int32_t *lo_idx, int32_t *lo_cnt, int32_t *hi_idx, int32_t *hi_cnt,
                             ba_stream_t stream) {
  ba_status st = check_shape(s);
  if (st != BA_OK) return st;
  if (!kv_idx || !kv_cnt || !lo_idx || !lo_cnt || !hi_idx || !hi_cnt) return BA_ERR_INVALID_ARG;
  if (!aligned16(kv_idx) || !aligned16(kv_cnt) || !aligned16(lo_idx) || !aligned16(lo_cnt) || !aligned16(hi_idx) ||
      !aligned16(hi_cnt))
    return BA_ERR_MISALIGNED;
  const int nb = nkblocks(s);                     // split_block counts key blocks
  if (kmax < 1 || split_block < 0 || split_block > nb) return BA_ERR_INVALID_ARG;
  const long long n_lists = static_cast<long long>(s->B) * s->Hq * nblocks(s);
  return from_cuda(launch_split(kv_idx, kv_cnt, lo_idx, lo_cnt, hi_idx, hi_cnt, n_lists, kmax, nb, split_block,
                                num_sms_of_current_device(), reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// Attention over the listed blocks; with O_prev/L_prev (both non-null) the
// epilogue merges the result with that earlier fp32 partial. Query side: Nq
// rows per head at a stride of q_stride rows (Nq = N, q_stride = N_alloc for
// the whole sequence).
ba_status sparse_fwd_impl(const ba_att_shape *s, const void *Q, const void *K, const void *V, const int32_t *kv_idx,
                          const int32_t *kv_cnt, int32_t kmax, void *O, int32_t o_dtype, float *LSE,
                          const float *O_prev, const float *L_prev, int Nq, int q_stride, ba_stream_t stream) {
  ba_status st = check_shape(s);
  if (st != BA_OK) return st;
  if (Nq < 1 || q_stride < Nq) return BA_ERR_INVALID_ARG;
  if (static_cast<long long>(s->B) * s->Hq * q_stride > (1LL << 36)) return BA_ERR_UNSUPPORTED;
  if (!Q || !K || !V || !kv_idx || !kv_cnt || !O || !LSE) return BA_ERR_INVALID_ARG;
  if (o_dtype != s->dtype && o_dtype != BA_DTYPE_F32) return BA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(kv_idx) || !aligned16(kv_cnt) || !aligned16(O) ||
      !aligned16(LSE))
    return BA_ERR_MISALIGNED;
  const bool merge = O_prev != nullptr;
  if (merge && (!aligned16(O_prev) || (reinterpret_cast<uintptr_t>(L_prev) & 3u))) return BA_ERR_MISALIGNED;
  if (kmax < 1) return BA_ERR_INVALID_ARG;
  const int nb = (Nq + s->block - 1) / s->block;        // query blocks of this call
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const float scale = effective_scale(s);
  const bool out_f32 = (o_dtype == BA_DTYPE_F32);
  if (use_tensor_core_path(s) && s->block == 256 && s->d == 128) {
    // a 256-row query block on a CTA pair (cta_group::2): each CTA holds 32
    // keys of every K half, so the K map has 32-row boxes
    CUtensorMap mq, mk, mv;
    if (!make_head_map(&mq, Q, s->d, Nq, q_stride, static_cast<long long>(s->B) * s->Hq, tc::kTileRows) ||
        !make_head_map(&mk, K, s->d, s->N, s->N_alloc, static_cast<long long>(s->B) * s->Hkv, tc2::kKRows) ||
        !make_head_map(&mv, V, s->d, s->N, s->N_alloc, static_cast<long long>(s->B) * s->Hkv, tc::kKvBoxRows))
      return BA_ERR_CUDA;
    const long long ctas = 2LL * s->B * s->Hq * nb;
    if (ctas > 0x7FFFFFFFLL) return BA_ERR_UNSUPPORTED;
    const float sl2 = scale * 1.4426950408889634f;
    const uint32_t smem = tc2::kDynSmem;
    auto run = [&](auto kernel, auto *out) -> ba_status {
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return BA_ERR_CUDA;
      kernel<<<static_cast<unsigned>(ctas), tc::kThreads, smem, cs>>>(mq, mk, mv, kv_idx, kv_cnt, kmax, out, LSE, O_prev,
                                                                   L_prev, s->Hq, s->Hkv, s->N, Nq, q_stride, nb,
                                                                   nkblocks(s), kblock(s), sl2);
      return from_cuda(cudaGetLastError());
    };
    if (out_f32) {
      float *of = static_cast<float *>(O);
      return merge ? run(tc2::attn_tc2_kernel<float, true>, of) : run(tc2::attn_tc2_kernel<float, false>, of);
    }
    __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(O);
    return merge ? run(tc2::attn_tc2_kernel<__nv_bfloat16, true>, ob)
                 : run(tc2::attn_tc2_kernel<__nv_bfloat16, false>, ob);
  }
  if (use_tensor_core_path(s)) {
    CUtensorMap mq, mk, mv;
    if (!make_head_map(&mq, Q, s->d, Nq, q_stride, static_cast<long long>(s->B) * s->Hq, tc::kTileRows) ||
        !make_head_map(&mk, K, s->d, s->N, s->N_alloc, static_cast<long long>(s->B) * s->Hkv, tc::kKvBoxRows) ||
        !make_head_map(&mv, V, s->d, s->N, s->N_alloc, static_cast<long long>(s->B) * s->Hkv, tc::kKvBoxRows))
      return BA_ERR_CUDA;
    // one CTA per 128-row query tile (a 256-row block at d = 64 is two tiles
    // sharing its list; two 64-row blocks share one tile, which attends both
    // lists)
    const long long tiles = static_cast<long long>(s->B) * s->Hq *
                            (s->block >= tc::kTileRows ? static_cast<long long>(nb) * (s->block / tc::kTileRows)
                                                       : (nb + 1) / 2);
    if (tiles > 0x7FFFFFFFLL) return BA_ERR_UNSUPPORTED;
    const float sl2 = scale * 1.4426950408889634f;
    const uint32_t smem = tc::dyn_smem_bytes(s->d);
    auto run = [&](auto kernel, auto *out) -> ba_status {
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return BA_ERR_CUDA;
      kernel<<<static_cast<unsigned>(tiles), tc::kThreads, smem, cs>>>(
          mq, mk, mv, kv_idx, kv_cnt, kmax, out, LSE, O_prev, L_prev, s->Hq, s->Hkv, s->N, Nq, q_stride, nb,
          s->block, nkblocks(s), kblock(s), sl2);
      return from_cuda(cudaGetLastError());
    };
    float *of = static_cast<float *>(O);
    __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(O);
    if (s->d == 128) {
      if (out_f32)
        return merge ? run(tc::attn_tc_kernel<float, true, 128>, of) : run(tc::attn_tc_kernel<float, false, 128>, of);
      return merge ? run(tc::attn_tc_kernel<__nv_bfloat16, true, 128>, ob)
                   : run(tc::attn_tc_kernel<__nv_bfloat16, false, 128>, ob);
    }
    if (out_f32)
      return merge ? run(tc::attn_tc_kernel<float, true, 64>, of) : run(tc::attn_tc_kernel<float, false, 64>, of);
    return merge ? run(tc::attn_tc_kernel<__nv_bfloat16, true, 64>, ob)
                 : run(tc::attn_tc_kernel<__nv_bfloat16, false, 64>, ob);
  }
  cudaError_t e;
#define BA_SIMT(T, TO, DD)                                                                                           \
  (merge ? launch_attn_simt<T, TO, DD, true>(static_cast<const T *>(Q), static_cast<const T *>(K),                   \
                                             static_cast<const T *>(V), kv_idx, kv_cnt, kmax, static_cast<TO *>(O), \
                                             LSE, s->B, s->Hq, s->Hkv, s->N, s->N_alloc, Nq, q_stride, s->block,   \
                                             kblock(s), scale, cs, O_prev, L_prev)                                   \
         : launch_attn_simt<T, TO, DD, false>(static_cast<const T *>(Q), static_cast<const T *>(K),                  \
                                              static_cast<const T *>(V), kv_idx, kv_cnt, kmax, static_cast<TO *>(O), \
                                              LSE, s->B, s->Hq, s->Hkv, s->N, s->N_alloc, Nq, q_stride, s->block,  \
                                              kblock(s), scale, cs))
  if (s->dtype == BA_DTYPE_BF16) {
    if (out_f32)
      e = s->d == 128 ? BA_SIMT(__nv_bfloat16, float, 128) : BA_SIMT(__nv_bfloat16, float, 64);
    else
      e = s->d == 128 ? BA_SIMT(__nv_bfloat16, __nv_bfloat16, 128) : BA_SIMT(__nv_bfloat16, __nv_bfloat16, 64);
  } else {
    e = s->d == 128 ? BA_SIMT(float, float, 128) : BA_SIMT(float, float, 64);
  }
#undef BA_SIMT
  return from_cuda(e);
}

}  // namespace

extern "C" {

ba_status ba_att_sparse_fwd(const ba_att_shape *s, const void *Q, const void *K, const void *V, const int32_t *kv_idx,
                            const int32_t *kv_cnt, int32_t kmax, void *O, int32_t o_dtype, float *LSE,
                            ba_stream_t stream) {
  if (s == nullptr) return BA_ERR_INVALID_ARG;
  return sparse_fwd_impl(s, Q, K, V, kv_idx, kv_cnt, kmax, O, o_dtype, LSE, nullptr, nullptr, s->N, s->N_alloc,
                         stream);
}

ba_status ba_att_sparse_fwd_merge(const ba_att_shape *s, const void *Q, const void *K, const void *V,
                                  const int32_t *kv_idx, const int32_t *kv_cnt, int32_t kmax, const float *O_prev,
                                  const float *LSE_prev, void *O, int32_t o_dtype, float *LSE, ba_stream_t stream) {
  if (s == nullptr || !O_prev || !LSE_prev) return BA_ERR_INVALID_ARG;
  return sparse_fwd_impl(s, Q, K, V, kv_idx, kv_cnt, kmax, O, o_dtype, LSE, O_prev, LSE_prev, s->N, s->N_alloc,
                         stream);
}

ba_status ba_att_sparse_fwd_rows(const ba_att_shape *s, int32_t q_rows, int32_t q_stride, const void *Q,
                                 const void *K, const void *V, const int32_t *kv_idx, const int32_t *kv_cnt,
                                 int32_t kmax, const float *O_prev, const float *LSE_prev, void *O, int32_t o_dtype,
                                 float *LSE, ba_stream_t stream) {
  if (s == nullptr || (O_prev == nullptr) != (LSE_prev == nullptr)) return BA_ERR_INVALID_ARG;
  return sparse_fwd_impl(s, Q, K, V, kv_idx, kv_cnt, kmax, O, o_dtype, LSE, O_prev, LSE_prev, q_rows, q_stride,
                         stream);
}

ba_status ba_att_merge_lse(int64_t rows, int32_t d, int32_t in_dtype, int32_t out_dtype, const void *O1,
                           const float *L1, const void *O2, const float *L2, void *O, float *L, ba_stream_t stream) {
  if (rows < 0) return BA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BA_ERR_UNSUPPORTED;
  if ((in_dtype != BA_DTYPE_F32 && in_dtype != BA_DTYPE_BF16) ||
      (out_dtype != BA_DTYPE_F32 && out_dtype != BA_DTYPE_BF16))
    return BA_ERR_INVALID_ARG;
  if (in_dtype == BA_DTYPE_BF16 && out_dtype == BA_DTYPE_F32) return BA_ERR_UNSUPPORTED;
  if (!O1 || !L1 || !O2 || !L2 || !O || !L) return BA_ERR_INVALID_ARG;
  if (!aligned16(O1) || !aligned16(O2) || !aligned16(O) || (reinterpret_cast<uintptr_t>(L1) & 3u) ||
      (reinterpret_cast<uintptr_t>(L2) & 3u) || (reinterpret_cast<uintptr_t>(L) & 3u))
    return BA_ERR_MISALIGNED;
  if (rows == 0) return BA_OK;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const int sms = num_sms_of_current_device();
  cudaError_t e;
#define BA_MERGE(TI, TO, DD)                                                                                      \
  launch_merge<TI, TO, DD>(static_cast<const TI *>(O1), L1, static_cast<const TI *>(O2), L2, static_cast<TO *>(O), \
                           L, rows, sms, cs)
  if (in_dtype == BA_DTYPE_BF16)
    e = d == 128 ? BA_MERGE(__nv_bfloat16, __nv_bfloat16, 128) : BA_MERGE(__nv_bfloat16, __nv_bfloat16, 64);
  else if (out_dtype == BA_DTYPE_BF16)
    e = d == 128 ? BA_MERGE(float, __nv_bfloat16, 128) : BA_MERGE(float, __nv_bfloat16, 64);
  else
    e = d == 128 ? BA_MERGE(float, float, 128) : BA_MERGE(float, float, 64);
#undef BA_MERGE
  return from_cuda(e);
}

ba_status ba_att_get_device_error(ba_stream_t stream, uint32_t *word_out) {
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(cs) != cudaSuccess) return BA_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return BA_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return BA_ERR_CUDA;
  if (word_out) *word_out = word;
  if (word == 0) return BA_OK;
  if (word & BA_DEVERR_WAIT_TIMEOUT) return BA_ERR_TIMEOUT;
  return BA_ERR_DEVICE;
}

ba_status ba_att_selftest_bounded_wait(uint32_t timeout_us, ba_stream_t stream) {
  if (timeout_us < 1 || timeout_us > 2000000u) return BA_ERR_INVALID_ARG;
  bounded_wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(timeout_us) * 1000ull);
  return from_cuda(cudaGetLastError());
}

}  // extern "C"

// ---------------------------------------------------------------- host-buffer pipeline
namespace {

constexpr size_t kWsAlign = 256;
size_t round_up(size_t x) { return (x + kWsAlign - 1) / kWsAlign * kWsAlign; }

// Workspace layout of ba_att_forward_host for chunks of C KV heads.
struct PipeLayout {
  int C = 0, G = 0, nb = 0, k = 0;
  size_t q[2], kk[2], v[2], o[2], l[2];                 // double-buffered chunk inputs and outputs
  size_t qm, qv, km, kv, idx, cnt, feat;                // selector buffers of one chunk
  size_t lo_idx, lo_cnt, hi_idx, hi_cnt, o1, l1;         // split buffers and the first span's fp32 partial
  size_t total = 0;
};

// Fewest KV heads per chunk that still give the attention kernel about 1024
// (query head, query block) tiles, a few waves of the GPU's CTA slots.
int auto_chunk(const ba_att_shape *s) {
  const long long tiles_per_kv_head = static_cast<long long>(s->Hq / s->Hkv) * nblocks(s);   // query blocks
  const long long c = (1024 + tiles_per_kv_head - 1) / tiles_per_kv_head;
  return static_cast<int>(c < 1 ? 1 : (c > s->Hkv ? s->Hkv : c));
}

bool pipe_layout(const ba_att_shape *s, double keep, int32_t split_block, int32_t chunk, PipeLayout *L) {
  if (check_shape(s) != BA_OK) return false;
  const int k = ba_att_keep_count(s, keep);
  if (k < 1) return false;
  const int nb = nblocks(s), nk = nkblocks(s);
  if (split_block > nk) return false;
  L->C = chunk > 0 ? (chunk < s->Hkv ? chunk : s->Hkv) : auto_chunk(s);
  L->G = s->Hq / s->Hkv;
  L->nb = nb;
  L->k = k;
  const size_t e = s->dtype == BA_DTYPE_BF16 ? 2 : 4;
  const size_t hq = static_cast<size_t>(L->C) * L->G, hk = static_cast<size_t>(L->C);
  const size_t rows_q = hq * s->N_alloc, rows_k = hk * s->N_alloc;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += round_up(bytes);
    return at;
  };
  for (int b = 0; b < 2; ++b) {
    L->q[b] = take(rows_q * s->d * e);
    L->kk[b] = take(rows_k * s->d * e);
    L->v[b] = take(rows_k * s->d * e);
    L->o[b] = take(rows_q * s->d * e);
    L->l[b] = take(rows_q * 4);
  }
  L->qm = take(hq * nb * s->d * 4);
  L->qv = take(hq * nb * s->d * 4);
  L->km = take(hk * nk * s->d * 4);
  L->kv = take(hk * nk * s->d * 4);
  L->idx = take(hq * nb * k * 4);
  L->cnt = take(hq * nb * 4);
  ba_att_shape cs = *s;                                     // one chunk of C KV heads of one batch entry
  cs.B = 1;
  cs.Hq = static_cast<int32_t>(hq);
  cs.Hkv = static_cast<int32_t>(hk);
  L->feat = take(static_cast<size_t>(ba_att_selector_workspace(&cs)));   // features, counters, score map
  if (split_block >= 0) {
    L->lo_idx = take(hq * nb * k * 4);
    L->lo_cnt = take(hq * nb * 4);
    L->hi_idx = take(hq * nb * k * 4);
    L->hi_cnt = take(hq * nb * 4);
    L->o1 = take(rows_q * s->d * 4);
    L->l1 = take(rows_q * 4);
  }
  L->total = off;
  return true;
}

// Per-device copy streams and events, created on first use and kept for the
// life of the process; `lock` serialises enqueueing calls on one device.
struct PipeResources {
  std::mutex lock;
  bool ready = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t entry = nullptr, tail = nullptr;
  cudaEvent_t in_ready[2] = {nullptr, nullptr}, in_free[2] = {nullptr, nullptr};
  cudaEvent_t out_ready[2] = {nullptr, nullptr}, out_free[2] = {nullptr, nullptr};
  cudaEvent_t scratch_free = nullptr;     // end of the last call on the static scratch
  bool scratch_used = false;
};

PipeResources *pipe_resources(int dev) {
  static PipeResources res[kMaxDevices];
  return (dev >= 0 && dev < kMaxDevices) ? &res[dev] : nullptr;
}

cudaError_t pipe_init(PipeResources *r) {
  if (r->ready) return cudaSuccess;
  cudaError_t e = cudaStreamCreateWithFlags(&r->h2d, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&r->d2h, cudaStreamNonBlocking);
  cudaEvent_t *evs[] = {&r->entry, &r->tail, &r->in_ready[0], &r->in_ready[1], &r->in_free[0], &r->in_free[1],
                        &r->out_ready[0], &r->out_ready[1], &r->out_free[0], &r->out_free[1], &r->scratch_free};
  for (cudaEvent_t *ev : evs)
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  if (e == cudaSuccess) r->ready = true;
  return e;
}

}  // namespace

extern "C" {

int64_t ba_att_forward_host_workspace(const ba_att_shape *s, double keep, int32_t split_block,
                                      int32_t kv_heads_per_chunk) {
  PipeLayout L;
  if (!pipe_layout(s, keep, split_block, kv_heads_per_chunk, &L)) return -1;
  return static_cast<int64_t>(L.total);
}

}  // extern "C"

namespace {

// The pipeline proper; arguments already validated, r->lock held.
ba_status forward_host_impl(PipeResources *r, const ba_att_shape *s, double keep, int32_t split_block,
                            const PipeLayout &L, const void *Q, const void *K, const void *V, void *O, float *LSE,
                            void *workspace, ba_stream_t stream) {
  ba_status st = BA_OK;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const size_t e = s->dtype == BA_DTYPE_BF16 ? 2 : 4;
  const size_t head_elems = static_cast<size_t>(s->N_alloc) * s->d;
  const int chunks_per_b = (s->Hkv + L.C - 1) / L.C;
  const int n_chunks = s->B * chunks_per_b;

  // the copy streams start after whatever `stream` holds (e.g. an earlier
  // call that used the same workspace)
  cudaError_t ce = cudaEventRecord(r->entry, cs);
  if (ce == cudaSuccess) ce = cudaStreamWaitEvent(r->h2d, r->entry, 0);
  if (ce == cudaSuccess) ce = cudaStreamWaitEvent(r->d2h, r->entry, 0);
  if (ce != cudaSuccess) return BA_ERR_CUDA;

  for (int c = 0; c < n_chunks && st == BA_OK; ++c) {
    const int sl = c & 1;
    const int b = c / chunks_per_b, g0 = (c % chunks_per_b) * L.C;
    const int gc = (s->Hkv - g0) < L.C ? (s->Hkv - g0) : L.C;
    const int hq0 = g0 * L.G, hqc = gc * L.G;
    const size_t q_off = (static_cast<size_t>(b) * s->Hq + hq0) * head_elems;
    const size_t k_off = (static_cast<size_t>(b) * s->Hkv + g0) * head_elems;
    void *Qc = ws + L.q[sl], *Kc = ws + L.kk[sl], *Vc = ws + L.v[sl], *Oc = ws + L.o[sl];
    float *Lc = reinterpret_cast<float *>(ws + L.l[sl]);

    // inputs of chunk c into slot sl, once chunk c-2 has finished reading it
    if (c >= 2) ce = cudaStreamWaitEvent(r->h2d, r->in_free[sl], 0);
    if (ce == cudaSuccess)
      ce = cudaMemcpyAsync(Qc, static_cast<const uint8_t *>(Q) + q_off * e, hqc * head_elems * e,
                           cudaMemcpyHostToDevice, r->h2d);
    if (ce == cudaSuccess)
      ce = cudaMemcpyAsync(Kc, static_cast<const uint8_t *>(K) + k_off * e, gc * head_elems * e,
                           cudaMemcpyHostToDevice, r->h2d);
    if (ce == cudaSuccess)
      ce = cudaMemcpyAsync(Vc, static_cast<const uint8_t *>(V) + k_off * e, gc * head_elems * e,
                           cudaMemcpyHostToDevice, r->h2d);
    if (ce == cudaSuccess) ce = cudaEventRecord(r->in_ready[sl], r->h2d);
    // compute on `stream`, into output slot sl once chunk c-2's outputs are out
    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(cs, r->in_ready[sl], 0);
    if (ce == cudaSuccess && c >= 2) ce = cudaStreamWaitEvent(cs, r->out_free[sl], 0);
    if (ce != cudaSuccess) {
      st = BA_ERR_CUDA;
      break;
    }
    ba_att_shape sc = *s;
    sc.B = 1;
    sc.Hq = hqc;
    sc.Hkv = gc;
    float *qm = reinterpret_cast<float *>(ws + L.qm), *qv = reinterpret_cast<float *>(ws + L.qv);
    float *km = reinterpret_cast<float *>(ws + L.km), *kv = reinterpret_cast<float *>(ws + L.kv);
    int32_t *idx = reinterpret_cast<int32_t *>(ws + L.idx), *cnt = reinterpret_cast<int32_t *>(ws + L.cnt);
    st = ba_att_selector(&sc, keep, Qc, Kc, qm, qv, km, kv, ws + L.feat, nullptr, idx, cnt, L.k, stream);
    if (st == BA_OK && split_block >= 0) {
      int32_t *lo_idx = reinterpret_cast<int32_t *>(ws + L.lo_idx), *lo_cnt = reinterpret_cast<int32_t *>(ws + L.lo_cnt);
      int32_t *hi_idx = reinterpret_cast<int32_t *>(ws + L.hi_idx), *hi_cnt = reinterpret_cast<int32_t *>(ws + L.hi_cnt);
      float *l1 = reinterpret_cast<float *>(ws + L.l1);
      st = ba_att_split_lists(&sc, split_block, idx, cnt, L.k, lo_idx, lo_cnt, hi_idx, hi_cnt, stream);
      if (st == BA_OK)
        st = ba_att_sparse_fwd(&sc, Qc, Kc, Vc, lo_idx, lo_cnt, L.k, ws + L.o1, BA_DTYPE_F32, l1, stream);
      if (st == BA_OK)   // the second span merges with the first in its epilogue
        st = ba_att_sparse_fwd_merge(&sc, Qc, Kc, Vc, hi_idx, hi_cnt, L.k, reinterpret_cast<const float *>(ws + L.o1),
                                     l1, Oc, s->dtype, Lc, stream);
      if (st == BA_OK && cudaEventRecord(r->in_free[sl], cs) != cudaSuccess) st = BA_ERR_CUDA;
    } else if (st == BA_OK) {
      st = ba_att_sparse_fwd(&sc, Qc, Kc, Vc, idx, cnt, L.k, Oc, s->dtype, Lc, stream);
      if (st == BA_OK && cudaEventRecord(r->in_free[sl], cs) != cudaSuccess) st = BA_ERR_CUDA;
    }
    if (st == BA_OK && cudaEventRecord(r->out_ready[sl], cs) != cudaSuccess) st = BA_ERR_CUDA;
    if (st != BA_OK) break;
    // outputs of chunk c: the N valid rows of each head
    ce = cudaStreamWaitEvent(r->d2h, r->out_ready[sl], 0);
    const size_t pitch_o = head_elems * e, row_o = static_cast<size_t>(s->N) * s->d * e;
    if (ce == cudaSuccess)
      ce = cudaMemcpy2DAsync(static_cast<uint8_t *>(O) + q_off * e, pitch_o, Oc, pitch_o, row_o, hqc,
                             cudaMemcpyDeviceToHost, r->d2h);
    const size_t pitch_l = static_cast<size_t>(s->N_alloc) * 4, row_l = static_cast<size_t>(s->N) * 4;
    if (ce == cudaSuccess)
      ce = cudaMemcpy2DAsync(LSE + (static_cast<size_t>(b) * s->Hq + hq0) * s->N_alloc, pitch_l, Lc, pitch_l, row_l,
                             hqc, cudaMemcpyDeviceToHost, r->d2h);
    if (ce == cudaSuccess) ce = cudaEventRecord(r->out_free[sl], r->d2h);
    if (ce != cudaSuccess) st = BA_ERR_CUDA;
  }
  // `stream` passes this call only after both copy streams have drained
  ce = cudaEventRecord(r->tail, r->h2d);
  if (ce == cudaSuccess) ce = cudaStreamWaitEvent(cs, r->tail, 0);
  if (ce == cudaSuccess) ce = cudaEventRecord(r->tail, r->d2h);
  if (ce == cudaSuccess) ce = cudaStreamWaitEvent(cs, r->tail, 0);
  if (st == BA_OK && ce != cudaSuccess) st = BA_ERR_CUDA;
  return st;
}

ba_status validate_host_call(const ba_att_shape *s, double keep, int32_t split_block, int32_t chunk, const void *Q,
                             const void *K, const void *V, const void *O, const float *LSE, PipeLayout *L) {
  ba_status st = check_shape(s);
  if (st != BA_OK) return st;
  if (!pipe_layout(s, keep, split_block, chunk, L)) return BA_ERR_INVALID_ARG;
  if (!Q || !K || !V || !O || !LSE) return BA_ERR_INVALID_ARG;
  return BA_OK;
}

PipeResources *lock_pipe(std::unique_lock<std::mutex> &guard, ba_status *st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    *st = BA_ERR_CUDA;
    return nullptr;
  }
  PipeResources *r = pipe_resources(dev);
  if (r == nullptr) {
    *st = BA_ERR_UNSUPPORTED;
    return nullptr;
  }
  guard = std::unique_lock<std::mutex>(r->lock);
  if (pipe_init(r) != cudaSuccess) {
    *st = BA_ERR_CUDA;
    return nullptr;
  }
  return r;
}

// Scratch of ba_att_forward_host_noalloc: static device memory of the
// module, reserved when the module loads; nothing is allocated per call.
__device__ __align__(256) uint8_t g_static_scratch[BA_ATT_STATIC_SCRATCH_BYTES];

}  // namespace

extern "C" {

ba_status ba_att_forward_host(const ba_att_shape *s, double keep, int32_t split_block, int32_t kv_heads_per_chunk,
                              const void *Q, const void *K, const void *V, void *O, float *LSE, void *workspace,
                              int64_t workspace_bytes, ba_stream_t stream) {
  PipeLayout L;
  ba_status st = validate_host_call(s, keep, split_block, kv_heads_per_chunk, Q, K, V, O, LSE, &L);
  if (st != BA_OK) return st;
  if (!workspace || workspace_bytes < static_cast<int64_t>(L.total)) return BA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) % kWsAlign != 0) return BA_ERR_MISALIGNED;
  std::unique_lock<std::mutex> guard;
  PipeResources *r = lock_pipe(guard, &st);
  if (r == nullptr) return st;
  return forward_host_impl(r, s, keep, split_block, L, Q, K, V, O, LSE, workspace, stream);
}

ba_status ba_att_forward_host_noalloc(const ba_att_shape *s, double keep, int32_t split_block, const void *Q,
                                      const void *K, const void *V, void *O, float *LSE, ba_stream_t stream) {
  PipeLayout L;
  ba_status st = validate_host_call(s, keep, split_block, 0, Q, K, V, O, LSE, &L);
  if (st != BA_OK) return st;
  // the chunk ba_att_forward_host would pick (about 1024 query tiles, so that
  // copies and compute overlap), narrowed until its workspace fits the scratch
  int chunk = auto_chunk(s);
  for (; chunk >= 1; --chunk) {
    if (!pipe_layout(s, keep, split_block, chunk, &L)) return BA_ERR_INVALID_ARG;
    if (L.total <= static_cast<size_t>(BA_ATT_STATIC_SCRATCH_BYTES)) break;
  }
  if (chunk < 1) return BA_ERR_UNSUPPORTED;
  std::unique_lock<std::mutex> guard;
  PipeResources *r = lock_pipe(guard, &st);
  if (r == nullptr) return st;
  void *scratch = nullptr;
  if (cudaGetSymbolAddress(&scratch, g_static_scratch) != cudaSuccess) return BA_ERR_CUDA;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  // one scratch per device: a call starts after the previous call on it ended,
  // whatever stream that call used
  if (r->scratch_used && cudaStreamWaitEvent(cs, r->scratch_free, 0) != cudaSuccess) return BA_ERR_CUDA;
  st = forward_host_impl(r, s, keep, split_block, L, Q, K, V, O, LSE, scratch, stream);
  if (cudaEventRecord(r->scratch_free, cs) != cudaSuccess && st == BA_OK) st = BA_ERR_CUDA;
  r->scratch_used = true;
  return st;
}

}  // extern "C"
