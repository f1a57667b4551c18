// dsa.cu - C ABI of the gated Indexer + Top-K sparse-attention layer (include/dsa.h):
// argument validation, launch configuration, TMA tensor maps, the fused prefill and
// decode drivers, per-stage timing and the device status word.  All kernels live in
// the headers included here, so the library is one translation unit.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "dsa.h"
#include "common.cuh"
#include "idx_cand.cuh"
#include "idx_scores.cuh"
#include "sparse_attn.cuh"
#include "topk.cuh"

namespace dsa {

// Device status word: kernels record DSA_ERR_TIMEOUT here when a bounded wait ends.
__device__ int g_status;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxTopK = 16384;

thread_local int64_t t_launches = 0;
thread_local int64_t t_fused_rows = 0;  // query rows whose steps 1-2 ran fused

// ---------------------------------------------------------------- stage timing
struct StageRec {
  int stage;
  cudaEvent_t start, stop;
};
thread_local bool t_timing = false;
thread_local std::vector<StageRec> t_pending;
thread_local std::vector<cudaEvent_t> t_free_events;
thread_local double t_stage_ms[3] = {0, 0, 0};
thread_local int64_t t_stage_launches[3] = {0, 0, 0};

cudaEvent_t take_event() {
  if (!t_free_events.empty()) {
    cudaEvent_t e = t_free_events.back();
    t_free_events.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

struct StageScope {
  int stage;
  cudaStream_t stream;
  cudaEvent_t start = nullptr, stop = nullptr;
  StageScope(int s, cudaStream_t st) : stage(s), stream(st) {
    if (t_timing) {
      start = take_event();
      stop = take_event();
      if (start) cudaEventRecord(start, stream);
    }
  }
  ~StageScope() {
    if (start && stop) {
      cudaEventRecord(stop, stream);
      t_pending.push_back({stage, start, stop});
    }
    ++t_stage_launches[stage];
  }
};

// ---------------------------------------------------------------- per-device setup
//
// What the setup caches (the device address of the status word, the kernels' shared-memory
// limits) belongs to the device's CUDA context: a context created anew (after
// cudaDeviceReset, for instance) reloads the library's module at possibly other addresses.
// The cache is therefore keyed by the context's unique id and redone when it changes.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;
std::once_flag g_ctx_fns_once;

// Unique id of the calling thread's current context, 0 if there is none (or it cannot be
// read; callers then redo their setup, which is correct, only slower).
uint64_t current_context_id() {
  std::call_once(g_ctx_fns_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(fn);
  });
  if (!g_ctx_get_current || !g_ctx_get_id) return 0;
  CUcontext c = nullptr;
  if (g_ctx_get_current(&c) != CUDA_SUCCESS || !c) return 0;
  unsigned long long id = 0;
  if (g_ctx_get_id(c, &id) != CUDA_SUCCESS) return 0;
  return (uint64_t)id;
}

struct DeviceState {
  bool ready = false;
  uint64_t ctx = 0;       // id of the context the cached setup belongs to
  int* status = nullptr;  // device address of g_status
  int num_sms = 148;
  size_t max_smem = 0;
  // copy streams of dsa_prefill_from_host (created on first use) and its events
  cudaStream_t s_in = nullptr, s_out = nullptr;
  std::vector<cudaEvent_t> events;
  std::mutex enqueue_mu;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

dsa_status device_setup(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceState& d = g_dev[dev];
  const uint64_t ctx = current_context_id();
  if (!d.ready || ctx == 0 || ctx != d.ctx) {
    d.ready = false;
    // (this call also creates and binds the primary context if there is none yet)
    if (cudaGetSymbolAddress((void**)&d.status, g_status) != cudaSuccess) return DSA_ERR_CUDA;
    cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
    int smem_optin = 0;
    cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    d.max_smem = (size_t)smem_optin;
    const size_t idx_max = idx_smem_bytes(4, 64, false);
    cudaError_t e = cudaSuccess;
    e = e ? e : allow_smem(idx_scores_kernel<64, false, kIdxScores>, idx_max);
    e = e ? e : allow_smem(idx_scores_kernel<16, false, kIdxScores>, idx_max);
    e = e ? e : allow_smem(idx_scores_kernel<64, true, kIdxScores>, idx_max);
    e = e ? e : allow_smem(idx_scores_kernel<16, true, kIdxScores>, idx_max);
    e = e ? e : allow_smem(idx_scores_kernel<64, false, kIdxSamples>, idx_max);
    e = e ? e : allow_smem(idx_scores_kernel<16, false, kIdxSamples>, idx_max);
    e = e ? e : allow_smem(idx_scores_kernel<64, true, kIdxSamples>, idx_max);
    e = e ? e : allow_smem(idx_scores_kernel<16, true, kIdxSamples>, idx_max);
    const size_t cand_max = idx_smem_bytes(4, 64, false, true);
    e = e ? e : allow_smem(idx_scores_kernel<64, false, kIdxCand>, cand_max);
    e = e ? e : allow_smem(idx_scores_kernel<16, false, kIdxCand>, cand_max);
    e = e ? e : allow_smem(idx_scores_kernel<64, true, kIdxCand>, cand_max);
    e = e ? e : allow_smem(idx_scores_kernel<16, true, kIdxCand>, cand_max);
    e = e ? e : allow_smem(idx_cand_kernel<false>, idx_cand_smem_bytes(false));
    e = e ? e : allow_smem(idx_cand_kernel<true>, idx_cand_smem_bytes(true));
    e = e ? e : allow_smem(idx_scores_kernel<64, false, kIdxBlockMax>, cand_max);
    e = e ? e : allow_smem(idx_scores_kernel<16, false, kIdxBlockMax>, cand_max);
    e = e ? e : allow_smem(idx_scores_kernel<64, true, kIdxBlockMax>, cand_max);
    e = e ? e : allow_smem(idx_scores_kernel<16, true, kIdxBlockMax>, cand_max);
    e = e ? e : allow_smem(topk_kernel<kTopkScores>, topk_smem_bytes(0));
    e = e ? e : allow_smem(topk_fused_kernel, topk_fused_smem_bytes(kTopkFastCap, kTopkFusedMaxN));
    e = e ? e : allow_smem(topk_kernel<kTopkFallback>, topk_smem_bytes(0));
    e = e ? e : allow_smem(topk_rows_alone_kernel, topk_smem_bytes(0));
    e = e ? e : allow_smem(topk_thr_kernel, topk_thr_smem_bytes(kThrStageMax));
    e = e ? e : allow_smem(sparse_attn_kernel<1, 1, kAddrBytes32>, attn_smem_bytes());
    e = e ? e : allow_smem(sparse_attn_kernel<2, 1, kAddrBytes32>, attn_smem_bytes());
    e = e ? e : allow_smem(sparse_attn_kernel<1, 2, kAddrBytes32>, attn_smem_bytes());
    e = e ? e : allow_smem(sparse_attn_kernel<2, 2, kAddrBytes32>, attn_smem_bytes());
    e = e ? e : allow_smem(sparse_attn_kernel<1, 1, kAddrRows>, attn_smem_bytes());
    e = e ? e : allow_smem(sparse_attn_kernel<2, 1, kAddrRows>, attn_smem_bytes());
    e = e ? e : allow_smem(sparse_attn_kernel<1, 2, kAddrRows>, attn_smem_bytes());
    e = e ? e : allow_smem(sparse_attn_kernel<2, 2, kAddrRows>, attn_smem_bytes());
    e = e ? e : allow_smem(sparse_attn_kernel<1, 1, kAddrUnits32>, attn_smem_bytes());
    e = e ? e : allow_smem(sparse_attn_kernel<2, 1, kAddrUnits32>, attn_smem_bytes());
    e = e ? e : allow_smem(sparse_attn_kernel<1, 2, kAddrUnits32>, attn_smem_bytes());
    e = e ? e : allow_smem(sparse_attn_kernel<2, 2, kAddrUnits32>, attn_smem_bytes());
    if (e != cudaSuccess) return DSA_ERR_CUDA;
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return DSA_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    d.ctx = current_context_id();
    d.ready = true;
  }
  *out = &d;
  return DSA_OK;
}

// ---------------------------------------------------------------- validation
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

dsa_status check_common(const dsa_params* P, const dsa_ragged* R) {
  if (!P || !R) return DSA_ERR_INVALID_ARG;
  if (R->batch < 1 || !R->q_offsets || !R->kv_offsets) return DSA_ERR_INVALID_ARG;
  if (R->max_q_len < 0 || R->max_kv_len < 0 || R->total_q < 0 || R->total_kv < 0)
    return DSA_ERR_INVALID_ARG;
  if (R->total_q > INT32_MAX || R->total_kv > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  if (P->top_k < 1 || P->top_k > kMaxTopK) return DSA_ERR_UNSUPPORTED;
  if (R->block_table) {
    const int ps = R->page_size;
    if (ps < 128 || ps > (1 << 24) || (ps & (ps - 1)) != 0) return DSA_ERR_INVALID_ARG;
    if (R->max_pages < 1 || (int64_t)R->max_pages * ps < R->max_kv_len) return DSA_ERR_INVALID_ARG;
    if (R->total_kv % ps != 0) return DSA_ERR_INVALID_ARG;
  }
  return DSA_OK;
}

CachePages cache_pages(const dsa_ragged* R) {
  CachePages pg;
  pg.table = R->block_table;
  pg.max_pages = R->block_table ? R->max_pages : 0;
  pg.shift = 0;
  pg.n_pages = 0;
  if (R->block_table) {
    while ((1 << pg.shift) < R->page_size) ++pg.shift;
    pg.n_pages = (int)(R->total_kv >> pg.shift);
  }
  return pg;
}

dsa_status check_indexer(const dsa_params* P) {
  if (P->idx_dim != 64) return DSA_ERR_UNSUPPORTED;
  if (P->n_idx_heads < 1 || P->n_idx_heads > 4) return DSA_ERR_UNSUPPORTED;
  if (P->idx_dtype != DSA_BF16 && P->idx_dtype != DSA_FP8_E4M3) return DSA_ERR_INVALID_ARG;
  if (P->w_row_stride < 0) return DSA_ERR_INVALID_ARG;
  if (P->w_row_stride != 0 && P->w_row_stride < P->n_idx_heads) return DSA_ERR_INVALID_ARG;
  if (!(P->idx_scale_q > 0.f) || !(P->idx_scale_k > 0.f)) return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

dsa_status check_attn(const dsa_params* P) {
  if (P->head_dim != kHeadDim) return DSA_ERR_UNSUPPORTED;
  if (P->n_q_heads < 1 || P->n_kv_heads < 1) return DSA_ERR_INVALID_ARG;
  if (P->n_q_heads % P->n_kv_heads != 0) return DSA_ERR_INVALID_ARG;
  const int G = P->n_q_heads / P->n_kv_heads;
  if (G > 16) return DSA_ERR_UNSUPPORTED;
  const int hkv = P->n_kv_heads;
  if (!(hkv == 1 || hkv == 2 || hkv == 4 || hkv % 8 == 0)) return DSA_ERR_UNSUPPORTED;
  if (P->attn_scale < 0.f || !std::isfinite(P->attn_scale)) return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

#define DSA_TRY(x)                   \
  do {                               \
    dsa_status _s = (x);             \
    if (_s != DSA_OK) return _s;     \
  } while (0)

// Status of the launch just made: DSA_ERR_CUDA, with one line on stderr naming the kernel
// and CUDA's error, when it failed.
dsa_status launch_status(const char* kernel) {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return DSA_OK;
  std::fprintf(stderr, "dsa: launch of %s failed: %s\n", kernel, cudaGetErrorString(e));
  return DSA_ERR_CUDA;
}

// ---------------------------------------------------------------- launches
dsa_status make_idx_map(CUtensorMap* map, const void* base, int64_t rows, int n_heads, bool fp8,
                        int box_rows) {
  const int elem = fp8 ? 1 : 2;
  cuuint64_t gdim[2] = {(cuuint64_t)(n_heads * 64), (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)(n_heads * 64 * elem)};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t estride[2] = {1u, 1u};
  CUresult r = g_encode(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        2, const_cast<void*>(base), gdim, gstride, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        fp8 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DSA_OK : DSA_ERR_INVALID_ARG;
}

// Variants of the indexer launch used by the fused indexer -> Top-K path.
struct IdxVariant {
  int shift = 0;                   // > 0: keys are the sampled key tensor below
  const void* k_rows = nullptr;    // sampled key tensor
  int64_t k_rows_n = 0;            // its rows
  const float* thr = nullptr;      // non-null: candidate variant
  float2* cand = nullptr;
  int cap = 0;
  int32_t* cand_cnt = nullptr;
  bool bmax = false;               // 32-key maxima instead of scores (scores = ld-strided rows)
  bool samples16 = false;          // scores as bf16 rounded down (the sampled pass)
  int32_t* tile_order = nullptr;   // candidate pass: room for ceil(rows / 128) query tiles,
                                   // ordered longest first when the batch has several sequences
};

dsa_status launch_index_scores(const DeviceState& dev, const dsa_params* P, const dsa_ragged* R,
                               const void* q_idx, const void* k_idx, const float* w,
                               int64_t q_begin, int64_t q_count, float* scores, int64_t ld,
                               int bq, cudaStream_t stream, const IdxVariant& var = IdxVariant()) {
  if (q_count == 0 || R->total_kv == 0) return DSA_OK;
  const bool fp8 = P->idx_dtype == DSA_FP8_E4M3;
  const bool cand = var.thr != nullptr;
  const int mode = cand ? kIdxCand : var.bmax ? kIdxBlockMax : var.samples16 ? kIdxSamples : kIdxScores;
  CUtensorMap mq, mk;
  if (cand && bq > 16) {
    // query-major candidate pass: 128 query rows per CTA, 128-key tiles, 4 segments per row
    DSA_TRY(make_idx_map(&mq, q_idx, R->total_q, P->n_idx_heads, fp8, kCandBQ));
    DSA_TRY(make_idx_map(&mk, k_idx, R->total_kv, P->n_idx_heads, fp8, kCandKT));
    IdxArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q_offsets = R->q_offsets;
    a.kv_offsets = R->kv_offsets;
    a.batch = R->batch;
    a.n_heads = P->n_idx_heads;
    a.q_begin = q_begin;
    a.q_count = q_count;
    a.n_tiles = (int)((q_count + kCandBQ - 1) / kCandBQ);
    a.w = w;
    a.w_row_stride = P->w_row_stride;
    a.scale = P->idx_scale_q * P->idx_scale_k;
    a.status = dev.status;
    a.pages = cache_pages(R);
    a.thr = var.thr;
    a.cand = var.cand;
    a.cap = var.cap;
    a.cand_cnt = var.cand_cnt;
    a.tile_order = nullptr;
    if (var.tile_order && R->batch > 1 && a.n_tiles > 1 && a.n_tiles <= kCandOrderMax) {
      StageScope scope(0, stream);
      idx_cand_order_kernel<<<1, kCandOrderThreads, 0, stream>>>(a, var.tile_order);
      ++t_launches;
      DSA_TRY(launch_status("idx_cand_order_kernel"));
      a.tile_order = var.tile_order;
    }
    StageScope scope(0, stream);
    if (fp8)
      idx_cand_kernel<true><<<a.n_tiles, kCandThreads, idx_cand_smem_bytes(true), stream>>>(mq, mk, a);
    else
      idx_cand_kernel<false><<<a.n_tiles, kCandThreads, idx_cand_smem_bytes(false), stream>>>(mq, mk, a);
    ++t_launches;
    return launch_status("idx_cand_kernel");
  }
  DSA_TRY(make_idx_map(&mq, q_idx, R->total_q, P->n_idx_heads, fp8, bq));
  if (var.shift)
    DSA_TRY(make_idx_map(&mk, var.k_rows, var.k_rows_n, P->n_idx_heads, fp8, kIdxKeyTile));
  else
    DSA_TRY(make_idx_map(&mk, k_idx, R->total_kv, P->n_idx_heads, fp8, kIdxKeyTile));
  IdxArgs a;
  a.q_offsets = R->q_offsets;
  a.kv_offsets = R->kv_offsets;
  a.batch = R->batch;
  a.n_heads = P->n_idx_heads;
  a.q_begin = q_begin;
  a.q_count = q_count;
  a.n_tiles = (int)((q_count + bq - 1) / bq);
  const int64_t max_keys = R->max_kv_len > 0 ? ((int64_t)(R->max_kv_len - 1) >> var.shift) + 1 : 1;
  const int max_kt = (int)std::max<int64_t>(1, (max_keys + kIdxKeyTile - 1) / kIdxKeyTile);
  // enough CTAs to fill the GPU a few times over, at least 8 key tiles per CTA; the
  // candidate variant keeps every key tile of a row in one CTA
  const int64_t target = (int64_t)dev.num_sms * 8;
  int ysplit = (int)std::min<int64_t>((target + a.n_tiles - 1) / a.n_tiles,
                                      std::max(1, max_kt / 8));
  ysplit = cand ? 1 : std::max(ysplit, 1);
  a.kt_per_split = (max_kt + ysplit - 1) / ysplit;
  ysplit = (max_kt + a.kt_per_split - 1) / a.kt_per_split;
  a.w = w;
  a.w_row_stride = P->w_row_stride;
  a.scale = P->idx_scale_q * P->idx_scale_k;
  a.scores = scores;
  a.ld = ld;
  a.status = dev.status;
  a.shift = var.shift;
  a.pages = var.shift ? CachePages{nullptr, 0, 0, 0} : cache_pages(R);  // samples are contiguous
  a.thr = var.thr;
  a.cand = var.cand;
  a.cap = var.cap;
  a.cand_cnt = var.cand_cnt;
  const size_t smem =
      idx_smem_bytes(P->n_idx_heads, bq, fp8, mode == kIdxCand || mode == kIdxBlockMax);
  dim3 grid((unsigned)a.n_tiles, (unsigned)ysplit);
  StageScope scope(0, stream);
#define DSA_IDX_CASE(BQ, F8, M)                                                      \
  if (bq == BQ && fp8 == F8 && mode == M)                                            \
    idx_scores_kernel<BQ, F8, M><<<grid, kIdxThreads, smem, stream>>>(mq, mk, a);
  DSA_IDX_CASE(64, false, kIdxScores)
  DSA_IDX_CASE(64, true, kIdxScores)
  DSA_IDX_CASE(16, false, kIdxScores)
  DSA_IDX_CASE(16, true, kIdxScores)
  DSA_IDX_CASE(64, false, kIdxSamples)
  DSA_IDX_CASE(64, true, kIdxSamples)
  DSA_IDX_CASE(16, false, kIdxSamples)
  DSA_IDX_CASE(16, true, kIdxSamples)
  DSA_IDX_CASE(64, false, kIdxCand)
  DSA_IDX_CASE(64, true, kIdxCand)
  DSA_IDX_CASE(16, false, kIdxCand)
  DSA_IDX_CASE(16, true, kIdxCand)
  DSA_IDX_CASE(64, false, kIdxBlockMax)
  DSA_IDX_CASE(64, true, kIdxBlockMax)
  DSA_IDX_CASE(16, false, kIdxBlockMax)
  DSA_IDX_CASE(16, true, kIdxBlockMax)
#undef DSA_IDX_CASE
  ++t_launches;
  return launch_status("idx_scores_kernel");
}

dsa_status launch_topk(const dsa_params* P, const dsa_ragged* R, const float* scores, int64_t ld,
                       int64_t q_begin, int64_t q_count, int32_t* idx, int64_t ld_idx,
                       int32_t* cnt, cudaStream_t stream, int blk_shift = 0) {
  if (q_count == 0) return DSA_OK;
  TopkArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q_offsets = R->q_offsets;
  a.kv_offsets = R->kv_offsets;
  a.batch = R->batch;
  a.q_begin = q_begin;
  a.q_count = q_count;
  a.K = P->top_k;
  a.scores = scores;
  a.ld = ld;
  a.idx = idx;
  a.ld_idx = ld_idx;
  a.cnt = cnt;
  a.blk_shift = blk_shift;
  const size_t smem = topk_smem_bytes(R->max_kv_len);
  StageScope scope(1, stream);
  // at most one row per SM (decode): CTAs that have their SM alone pipeline their row loads
  DeviceState* dev = nullptr;
  DSA_TRY(device_setup(&dev));
  if (q_count <= dev->num_sms)
    topk_rows_alone_kernel<<<(unsigned)q_count, kTopkThreads, smem, stream>>>(a);
  else
    topk_kernel<kTopkScores><<<(unsigned)q_count, kTopkThreads, smem, stream>>>(a);
  ++t_launches;
  return launch_status("topk_kernel");
}

// ---------------------------------------------------------------- fused indexer -> Top-K
//
// Per pass of rows: (1) the indexer over every 16th key (samples), (2) a threshold estimate
// per row from its samples, (3) the indexer again over all keys keeping only the scores
// >= the estimate as candidates, (4) an exact selection over the candidates, (5) the rows
// whose estimate missed, recomputed and selected exactly.  The sampled key tensor is built
// once per call.
constexpr int kSampleShift = 4;
constexpr int kFallbackCtas = 128;

struct FusedGeom {
  int cap;              // candidate slots per row
  int64_t ld_s;         // samples (bf16) per sample row
  int64_t ld_fb;        // floats per fallback scratch row
  int64_t samp_rows;    // rows of the sampled key tensor
  int64_t key_row;      // bytes per key row
  int64_t fixed_bytes;  // sampled keys + fallback scratch
  int64_t row_bytes;    // per query row: samples / candidates (shared), threshold, count, list
};

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// false when the fused path cannot take this problem (K or the rows too long)
bool fused_geom(const dsa_params* P, const dsa_ragged* R, FusedGeom* g) {
  const int K = P->top_k;
  const double s = double(1 << kSampleShift);
  // samples of rank R = e + 5 sqrt(e) + 16 (e = K / 16 + 1 at most) leave about 16 R
  // candidates; the slots cover 6 standard deviations more
  const double e = K / s + 1.0;
  const double rr = std::ceil(e + 5.0 * std::sqrt(e) + 16.0);
  const int64_t cap = round_up((int64_t)std::ceil(s * (rr + 6.0 * std::sqrt(rr))), 256);
  if (cap > kTopkFastCap || cap < K) return false;
  if (R->max_kv_len > kTopkFusedMaxN) return false;
  g->cap = (int)cap;
  const int64_t max_n = std::max(R->max_kv_len, 1);
  g->ld_s = round_up(((max_n - 1) >> kSampleShift) + 1, 32);
  g->ld_fb = round_up(max_n, 4);
  // sampled rows are laid out by the logical offsets: sum_b L_b <= total_kv when contiguous,
  // <= batch * max_kv_len when paged (pages may be shared)
  const int64_t logical = R->block_table ? (int64_t)R->batch * R->max_kv_len : R->total_kv;
  g->samp_rows = (logical >> kSampleShift) + R->batch + 1;
  g->key_row = (int64_t)P->n_idx_heads * 64 * (P->idx_dtype == DSA_FP8_E4M3 ? 1 : 2);
  g->fixed_bytes = round_up(g->samp_rows * g->key_row, 256) +
                   round_up((int64_t)kFallbackCtas * g->ld_fb * 4, 256) + 256 * 6;
  // per row: samples / candidates (shared), threshold, largest sample key, 4 counts, a list
  // entry, and a byte for the tile order (4 bytes per 128 rows, one more tile at most)
  g->row_bytes = std::max<int64_t>(g->ld_s * 2, cap * 8) + 7 * 4 + 1;
  return true;
}

// Rows of one fused pass that `bytes` of workspace hold (0 if not even one).
int64_t fused_rows(const FusedGeom& g, int64_t bytes) {
  return bytes > g.fixed_bytes ? (bytes - g.fixed_bytes) / g.row_bytes : 0;
}

// The layer takes the fused path for prefill-shaped batches (few sequences, many query
// rows each) whose score matrix would be far larger than L2; smaller problems keep their
// scores in L2 anyway, and batches of many short sequences suit the split key ranges of
// the materialised path.
constexpr int64_t kFusedMinScoreBytes = int64_t(256) << 20;
constexpr int64_t kFusedMinRows = 2048;

bool fused_wanted(const dsa_params* P, const dsa_ragged* R, FusedGeom* g) {
  if (!fused_geom(P, R, g)) return false;
  if ((int64_t)R->batch * 256 > R->total_q) return false;
  return R->total_q * (int64_t)R->max_kv_len * 2 > kFusedMinScoreBytes;
}

struct FusedWs {
  uint4* k_samp;
  float* fb_scores;
  char* sc;        // samples [rows, ld_s] bf16, later candidates [rows, cap] float2
  float* thr;
  uint32_t* khi;   // [rows] largest sample key
  int32_t* ccnt;   // [rows, 4]
  int32_t* list;   // [1 + rows]
  int32_t* order;  // [ceil(rows / 128)] candidate-pass tile order
};

FusedWs fused_carve(const FusedGeom& g, void* ws, int64_t rows) {
  char* p = static_cast<char*>(ws);
  FusedWs f;
  f.k_samp = reinterpret_cast<uint4*>(p);
  p += round_up(g.samp_rows * g.key_row, 256);
  f.fb_scores = reinterpret_cast<float*>(p);
  p += round_up((int64_t)kFallbackCtas * g.ld_fb * 4, 256);
  f.sc = p;
  p += round_up(rows * std::max<int64_t>(g.ld_s * 2, (int64_t)g.cap * 8), 256);
  f.thr = reinterpret_cast<float*>(p);
  p += round_up(rows * 4, 256);
  f.khi = reinterpret_cast<uint32_t*>(p);
  p += round_up(rows * 4, 256);
  f.ccnt = reinterpret_cast<int32_t*>(p);
  p += round_up(rows * 16, 256);
  f.list = reinterpret_cast<int32_t*>(p);
  p += round_up((1 + rows) * 4, 256);
  f.order = reinterpret_cast<int32_t*>(p);
  return f;
}

dsa_status fused_prepare(const DeviceState& dev, const dsa_ragged* R, const void* k_idx, const FusedGeom& g, const FusedWs& f,
                         cudaStream_t stream) {
  const int vec = (int)(g.key_row / 16);
  const int64_t blocks = std::min<int64_t>((g.samp_rows + 7) / 8, (int64_t)dev.num_sms * 8);
  StageScope scope(0, stream);
  idx_sample_keys_kernel<<<(unsigned)std::max<int64_t>(blocks, 1), 256, 0, stream>>>(
      R->kv_offsets, R->batch, kSampleShift, static_cast<const uint4*>(k_idx), f.k_samp, vec,
      g.samp_rows, cache_pages(R));
  ++t_launches;
  return launch_status("idx_sample_keys_kernel");
}

dsa_status fused_pass(const DeviceState& dev, const dsa_params* P, const dsa_ragged* R,
                      const void* q_idx, const void* k_idx, const float* w, int64_t q_begin,
                      int64_t q_count, int32_t* idx, int64_t ld_idx, int32_t* cnt,
                      const FusedGeom& g, const FusedWs& f, cudaStream_t stream) {
  if (q_count == 0) return DSA_OK;
  const int bq = R->max_q_len <= 16 ? 16 : 64;
  // samples: bf16 [rows, ld_s], rounded toward -infinity
  float* samp = reinterpret_cast<float*>(f.sc);
  t_fused_rows += q_count;
  {  // (1) sampled scores
    IdxVariant v;
    v.samples16 = true;
    v.shift = kSampleShift;
    v.k_rows = f.k_samp;
    v.k_rows_n = g.samp_rows;
    DSA_TRY(launch_index_scores(dev, P, R, q_idx, k_idx, w, q_begin, q_count, samp, g.ld_s, bq,
                                stream, v));
  }
  {  // (2) thresholds
    TopkThrArgs t;
    t.q_offsets = R->q_offsets;
    t.kv_offsets = R->kv_offsets;
    t.batch = R->batch;
    t.q_begin = q_begin;
    t.q_count = q_count;
    t.K = P->top_k;
    t.cap = g.cap;
    t.shift = kSampleShift;
    t.samp = reinterpret_cast<const uint16_t*>(f.sc);
    t.ld_s = g.ld_s;
    t.stage = (int)std::min<int64_t>(kThrStageMax, g.ld_s);  // ld_s: a multiple of 32
    // rows of more than t.stage samples (possible when ld_s exceeds it) take a CTA each
    t.long_rows = g.ld_s > t.stage ? 1 : 0;
    t.thr = f.thr;
    t.khi = f.khi;
    t.fb_list = f.list;
    {
      StageScope scope(1, stream);
      topk_thr_kernel<<<(unsigned)((q_count + kThrWarps - 1) / kThrWarps), 32 * kThrWarps,
                        topk_thr_smem_bytes(t.stage), stream>>>(t);
      ++t_launches;
      DSA_TRY(launch_status("topk_thr_kernel"));
    }
    if (t.long_rows) {
      StageScope scope(1, stream);
      topk_thr_long_kernel<<<(unsigned)q_count, kThrLongThreads,
                             topk_thr_long_smem_bytes((int)g.ld_s), stream>>>(t, (int)g.ld_s);
      ++t_launches;
      DSA_TRY(launch_status("topk_thr_long_kernel"));
    }
  }
  {  // (3) candidates
    IdxVariant v;
    v.thr = f.thr;
    v.cand = reinterpret_cast<float2*>(f.sc);
    v.cap = g.cap;
    v.cand_cnt = f.ccnt;
    v.tile_order = f.order;
    DSA_TRY(launch_index_scores(dev, P, R, q_idx, k_idx, w, q_begin, q_count, nullptr, 0, bq,
                                stream, v));
  }
  TopkArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q_offsets = R->q_offsets;
  a.kv_offsets = R->kv_offsets;
  a.batch = R->batch;
  a.q_begin = q_begin;
  a.q_count = q_count;
  a.K = P->top_k;
  a.idx = idx;
  a.ld_idx = ld_idx;
  a.cnt = cnt;
  a.cand = reinterpret_cast<const float2*>(f.sc);
  a.cap = g.cap;
  a.cand_cnt = f.ccnt;
  a.thr = f.thr;
  a.khi = f.khi;
  a.fb_list = f.list;
  a.q_idx = q_idx;
  a.k_idx = k_idx;
  a.idx_heads = P->n_idx_heads;
  a.idx_fp8 = P->idx_dtype == DSA_FP8_E4M3 ? 1 : 0;
  a.w = w;
  a.w_row_stride = P->w_row_stride;
  a.idx_scale = P->idx_scale_q * P->idx_scale_k;
  a.fb_scores = f.fb_scores;
  a.ld_fb = g.ld_fb;
  a.pages = cache_pages(R);
  const size_t smem = topk_smem_bytes(R->max_kv_len);
  a.bm_words = topk_fused_bm_words(std::max(R->max_kv_len, 1));
  a.prefetch_ahead = kFusedCtasPerSm * dev.num_sms;  // about one wave of selection CTAs
  {  // (4) exact selection over the candidates
    StageScope scope(1, stream);
    topk_fused_kernel<<<(unsigned)q_count, kFusedThreads,
                        topk_fused_smem_bytes(g.cap, R->max_kv_len), stream>>>(a);
    ++t_launches;
    DSA_TRY(launch_status("topk_kernel (fused selection)"));
  }
  {  // (5) rows whose estimate missed
    StageScope scope(1, stream);
    topk_kernel<kTopkFallback><<<kFallbackCtas, kTopkThreads, smem, stream>>>(a);
    ++t_launches;
    DSA_TRY(launch_status("topk_kernel (fallback rows)"));
  }
  return DSA_OK;
}

dsa_status launch_attn(const DeviceState& dev, const dsa_params* P, const dsa_ragged* R,
                       const void* q, const void* k,
                       const void* v, const int32_t* idx, int64_t ld_idx, int64_t q_begin,
                       int64_t q_count, const void* gate, void* out, float* lse,
                       int32_t* err_count, cudaStream_t stream, const void* other = nullptr,
                       bool decode = false) {
  if (q_count == 0) return DSA_OK;
  AttnArgs a;
  a.q_offsets = R->q_offsets;
  a.kv_offsets = R->kv_offsets;
  a.batch = R->batch;
  a.q_begin = q_begin;
  a.q_count = q_count;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.idx = idx;
  a.ld_idx = ld_idx;
  a.K = P->top_k;
  a.gate = static_cast<const __nv_bfloat16*>(gate);
  a.other = static_cast<const __nv_bfloat16*>(other);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.err_count = err_count;
  a.status = dev.status;
  a.Hq = P->n_q_heads;
  a.Hkv = P->n_kv_heads;
  a.G = P->n_q_heads / P->n_kv_heads;
  const float scale = P->attn_scale > 0.f ? P->attn_scale : 1.0f / std::sqrt((float)P->head_dim);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.pages = cache_pages(R);
  // KV heads per CTA: two, or one for a single-KV-head layer and for decode (one query per
  // sequence gives too few rows to fill the GPU with two-head CTAs; one-head CTAs put four
  // warps on a head and halve each warp's chunks).  Fixed by the call type and the shape
  // alone, so that a row's result does not depend on how the rows are split into launches
  // (the warps' partial softmax states are merged in an order set by the CTA shape).
  const int hkv_cta = (decode || P->n_kv_heads == 1) ? 1 : 2;
  const int nt = a.G > 8 ? 2 : 1;
  // 32-bit offsets when each cache array (rows of Hkv x d bf16) spans at most 4 GiB (bytes) or
  // 64 GiB (16-byte units); the general form beyond, or everywhere when DSA_ATTN_ADDR_ROWS is
  // set to a non-zero value in the environment (so that tests reach it with small caches)
  const uint64_t cache_bytes = (uint64_t)R->total_kv * (uint64_t)P->n_kv_heads * kHeadDim * 2;
  static const bool force_rows = [] {
    const char* e = std::getenv("DSA_ATTN_ADDR_ROWS");
    return e && std::atoi(e) != 0;
  }();
  const int am = force_rows                    ? kAddrRows
                 : cache_bytes <= (1ull << 32) ? kAddrBytes32
                 : cache_bytes <= (1ull << 36) ? kAddrUnits32
                                               : kAddrRows;
  dim3 grid((unsigned)q_count, (unsigned)(P->n_kv_heads / hkv_cta));
  const size_t smem = attn_smem_bytes();
  StageScope scope(2, stream);
#define DSA_ATTN_CASE(H, N, O)                                                      \
  if (hkv_cta == H && nt == N && am == O)                                           \
    sparse_attn_kernel<H, N, O><<<grid, AttnGeom<H>::kThreads, smem, stream>>>(a);
  DSA_ATTN_CASE(1, 1, kAddrBytes32)
  DSA_ATTN_CASE(2, 1, kAddrBytes32)
  DSA_ATTN_CASE(1, 2, kAddrBytes32)
  DSA_ATTN_CASE(2, 2, kAddrBytes32)
  DSA_ATTN_CASE(1, 1, kAddrRows)
  DSA_ATTN_CASE(2, 1, kAddrRows)
  DSA_ATTN_CASE(1, 2, kAddrRows)
  DSA_ATTN_CASE(2, 2, kAddrRows)
  DSA_ATTN_CASE(1, 1, kAddrUnits32)
  DSA_ATTN_CASE(2, 1, kAddrUnits32)
  DSA_ATTN_CASE(1, 2, kAddrUnits32)
  DSA_ATTN_CASE(2, 2, kAddrUnits32)
#undef DSA_ATTN_CASE
  ++t_launches;
  return launch_status("sparse_attn_kernel");
}

// Workspace per pass row: scores row (ld floats) plus an index row when idx_out is absent.
int64_t scores_ld(const dsa_ragged* R) { return round_up(std::max(R->max_kv_len, 1), 32); }

// Rows of one indexer / Top-K sub-pass: bounded by kScorePassBytes of scores (more rows per
// launch amortise CTA set-up; fewer keep the scores closer to L2); attention passes take as
// many rows as the rest of the workspace holds.
constexpr int64_t kScorePassBytes = int64_t(512) << 20;

struct PassPlan {
  int64_t rows_s;  // query rows per indexer / Top-K sub-pass
  int64_t rows_a;  // query rows per attention pass
};

// srow / irow: workspace bytes of one score row / one index row (irow = 0 when the
// caller provides the index output).  Returns false if not even one row of each fits.
bool plan_passes(int64_t total_q, int64_t srow, int64_t irow, int64_t ws, int num_sms,
                 PassPlan* plan) {
  if (ws < srow + irow) return false;
  int64_t rows_s = std::max<int64_t>(kScorePassBytes / srow, std::min<int64_t>(total_q, num_sms));
  rows_s = std::max<int64_t>(1, std::min(rows_s, total_q));
  // a score pass never takes more than an attention pass of the same size leaves room for
  rows_s = std::max<int64_t>(1, std::min(rows_s, ws / (srow + irow)));
  int64_t rows_a = irow ? (ws - rows_s * srow) / irow : total_q;
  rows_a = std::max<int64_t>(rows_s, std::min(rows_a, total_q));
  plan->rows_s = rows_s;
  plan->rows_a = std::min(rows_a, total_q);
  return true;
}

dsa_status run_index(const DeviceState& dev, const dsa_params* P, const dsa_ragged* R,
                     const void* q_idx, const void* k_idx, const float* w, int64_t a0, int64_t a1,
                     int32_t* idx, void* ws, size_t ws_bytes, cudaStream_t stream, int fused,
                     int bq);

// ---------------------------------------------------------------- per-sequence planning
//
// With host copies of the offsets the layer sees each sequence's shape.  A stretch of
// consecutive sequences of one kind -- long query groups (prefill chunks, Q_b >= kLongQ) or
// short ones (decode tokens) -- is one contiguous range of packed query rows.
constexpr int kLongQ = 128;

struct RowRun {
  int64_t a0, a1;  // packed query rows
  bool lng;        // sequences with Q_b >= kLongQ
  int max_q;       // longest query group in the stretch
};

// Stretches of the batch within rows [row0, row1); empty without host offsets.
std::vector<RowRun> row_runs(const dsa_ragged* R, int64_t row0, int64_t row1) {
  std::vector<RowRun> runs;
  const int32_t* qo = R->q_offsets_host;
  if (!qo) return runs;
  for (int b = 0; b < R->batch; ++b) {
    const int64_t s0 = std::max<int64_t>(qo[b], row0), s1 = std::min<int64_t>(qo[b + 1], row1);
    if (s1 <= s0) continue;
    const int q = qo[b + 1] - qo[b];
    const bool lng = q >= kLongQ;
    if (!runs.empty() && runs.back().lng == lng && runs.back().a1 == s0) {
      runs.back().a1 = s1;
      runs.back().max_q = std::max(runs.back().max_q, q);
    } else {
      runs.push_back({s0, s1, lng, q});
    }
  }
  return runs;
}

bool mixed_runs(const std::vector<RowRun>& runs) {
  bool l = false, sh = false;
  for (const RowRun& r : runs) (r.lng ? l : sh) = true;
  return l && sh;
}

// Score rows of one materialised sub-pass over `rows` query rows (as plan_passes).
int64_t score_pass_rows(int64_t rows, int64_t srow) {
  return std::max<int64_t>(1, std::min(rows, std::max<int64_t>(kScorePassBytes / srow,
                                                                 std::min<int64_t>(rows, 148))));
}

dsa_status run_layer(const dsa_params* P, const dsa_ragged* R, const void* q_idx,
                     const void* k_idx, const float* w, const void* q, const void* k,
                     const void* v, const void* gate, void* out, int32_t* idx_out,
                     int32_t* err_count, void* ws, size_t ws_bytes, void* stream_v,
                     bool decode, int64_t row0 = 0, int64_t row1 = -1) {
  DSA_TRY(check_common(P, R));
  DSA_TRY(check_indexer(P));
  DSA_TRY(check_attn(P));
  if (!q_idx || !k_idx || !w || !q || !k || !v || !out) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(q) || !aligned16(k) ||
      !aligned16(v) || !aligned16(out) || (gate && !aligned16(gate)))
    return DSA_ERR_INVALID_ARG;
  if (decode && (R->max_q_len != 1 || R->total_q != R->batch)) return DSA_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return DSA_ERR_WORKSPACE;
  if (row1 < 0) row1 = R->total_q;
  if (row0 < 0 || row1 > R->total_q || row0 > row1) return DSA_ERR_INVALID_ARG;
  if (row0 == row1) return DSA_OK;
  const int64_t n_rows = row1 - row0;
  const int64_t ld = scores_ld(R);
  const int64_t K = P->top_k;
  const int64_t irow = idx_out ? 0 : round_up(K * 4, 16);
  if ((int64_t)ws_bytes < ld * 4 + irow) return DSA_ERR_WORKSPACE;
  DeviceState* dev = nullptr;
  DSA_TRY(device_setup(&dev));
  PassPlan plan;
  if (!plan_passes(n_rows, ld * 4, irow, (int64_t)ws_bytes, dev->num_sms, &plan))
    return DSA_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  if (!decode) {
    // a batch mixing prefill chunks with short query groups: steps 1-2 per stretch with the
    // tiles that suit it, then one attention launch over every row
    const std::vector<RowRun> runs = row_runs(R, row0, row1);
    const int64_t idx_bytes = idx_out ? 0 : round_up(n_rows * K * 4, 256);
    if (mixed_runs(runs) && (int64_t)ws_bytes >= idx_bytes + ld * 4) {
      int32_t* idx_all = idx_out ? idx_out + row0 * K : static_cast<int32_t*>(ws);
      void* scratch = static_cast<char*>(ws) + idx_bytes;
      const size_t sb = ws_bytes - (size_t)idx_bytes;
      for (const RowRun& r : runs)
        DSA_TRY(run_index(*dev, P, R, q_idx, k_idx, w, r.a0, r.a1, idx_all + (r.a0 - row0) * K,
                          scratch, sb, stream, r.lng ? 1 : 0,
                          r.lng ? 64 : (r.max_q <= 16 ? 16 : 64)));
      return launch_attn(*dev, P, R, q, k, v, idx_all, K, row0, n_rows, gate, out, nullptr,
                         err_count, stream);
    }
  }
  FusedGeom fg;
  if (!decode && fused_wanted(P, R, &fg)) {
    // fused indexer -> Top-K, in passes of as many rows as the workspace holds (with their
    // index rows when the caller keeps none)
    const int64_t rows = std::min<int64_t>(
        n_rows, std::max<int64_t>(0, ((int64_t)ws_bytes - fg.fixed_bytes - 256) /
                                          (fg.row_bytes + irow)));
    if (rows >= std::min<int64_t>(n_rows, kFusedMinRows)) {
      const FusedWs f = fused_carve(fg, ws, rows);
      int32_t* idx_ws = reinterpret_cast<int32_t*>(
          static_cast<char*>(ws) + round_up(fg.fixed_bytes + rows * fg.row_bytes, 256));
      DSA_TRY(fused_prepare(*dev, R, k_idx, fg, f, stream));
      for (int64_t a0 = row0; a0 < row1; a0 += rows) {
        const int64_t cnt_a = std::min<int64_t>(rows, row1 - a0);
        int32_t* idx = idx_out ? idx_out + a0 * K : idx_ws;
        DSA_TRY(fused_pass(*dev, P, R, q_idx, k_idx, w, a0, cnt_a, idx, K, nullptr, fg, f, stream));
        DSA_TRY(launch_attn(*dev, P, R, q, k, v, idx, K, a0, cnt_a, gate, out, nullptr, err_count,
                            stream));
      }
      return DSA_OK;
    }
  }
  float* scores = static_cast<float*>(ws);
  int32_t* idx_ws = idx_out ? nullptr
                            : reinterpret_cast<int32_t*>(static_cast<char*>(ws) +
                                                         plan.rows_s * ld * 4);
  const int bq = (decode || R->max_q_len <= 16) ? 16 : 64;
  for (int64_t a0 = row0; a0 < row1; a0 += plan.rows_a) {
    const int64_t cnt_a = std::min<int64_t>(plan.rows_a, row1 - a0);
    int32_t* idx = idx_out ? idx_out + a0 * K : idx_ws;
    for (int64_t s0 = a0; s0 < a0 + cnt_a; s0 += plan.rows_s) {
      const int64_t cnt_s = std::min<int64_t>(plan.rows_s, a0 + cnt_a - s0);
      DSA_TRY(launch_index_scores(*dev, P, R, q_idx, k_idx, w, s0, cnt_s, scores, ld, bq, stream));
      DSA_TRY(launch_topk(P, R, scores, ld, s0, cnt_s, idx + (s0 - a0) * K, K, nullptr, stream));
    }
    DSA_TRY(launch_attn(*dev, P, R, q, k, v, idx, K, a0, cnt_a, gate, out, nullptr, err_count,
                        stream, nullptr, decode));
  }
  return DSA_OK;
}

// Steps 1-2 alone for rows [a0, a1): index rows into idx (row r at idx + (r - a0) * K), in
// passes sized to the workspace.  fused: -1 as dsa_prefill decides for the whole batch, 1 the
// fused indexer -> Top-K whenever it supports the problem and the workspace holds enough
// rows, 0 never.  bq: query rows per score tile (16 or 64; 0: from max_q_len).
dsa_status run_index(const DeviceState& dev, const dsa_params* P, const dsa_ragged* R,
                     const void* q_idx, const void* k_idx, const float* w, int64_t a0, int64_t a1,
                     int32_t* idx, void* ws, size_t ws_bytes, cudaStream_t stream, int fused = -1,
                     int bq = 0) {
  const int64_t n_rows = a1 - a0;
  if (n_rows <= 0) return DSA_OK;
  const int64_t K = P->top_k;
  FusedGeom fg;
  if (fused < 0 ? fused_wanted(P, R, &fg) : fused > 0 && fused_geom(P, R, &fg)) {
    const int64_t rows = std::min<int64_t>(n_rows, fused_rows(fg, (int64_t)ws_bytes));
    if (rows >= std::min<int64_t>(n_rows, kFusedMinRows)) {
      const FusedWs f = fused_carve(fg, ws, rows);
      DSA_TRY(fused_prepare(dev, R, k_idx, fg, f, stream));
      for (int64_t s0 = a0; s0 < a1; s0 += rows) {
        const int64_t n = std::min<int64_t>(rows, a1 - s0);
        DSA_TRY(fused_pass(dev, P, R, q_idx, k_idx, w, s0, n, idx + (s0 - a0) * K, K, nullptr,
                           fg, f, stream));
      }
      return DSA_OK;
    }
  }
  const int64_t ld = scores_ld(R);
  int64_t rows_s = std::min<int64_t>((int64_t)ws_bytes / (ld * 4),
                                     std::max<int64_t>(kScorePassBytes / (ld * 4), 1));
  if (rows_s < 1) return DSA_ERR_WORKSPACE;
  float* scores = static_cast<float*>(ws);
  if (bq == 0) bq = R->max_q_len <= 16 ? 16 : 64;
  for (int64_t s0 = a0; s0 < a1; s0 += rows_s) {
    const int64_t n = std::min<int64_t>(rows_s, a1 - s0);
    DSA_TRY(launch_index_scores(dev, P, R, q_idx, k_idx, w, s0, n, scores, ld, bq, stream));
    DSA_TRY(launch_topk(P, R, scores, ld, s0, n, idx + (s0 - a0) * K, K, nullptr, stream));
  }
  return DSA_OK;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case DSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "bounded device wait timed out";
  }
  return "unknown status";
}

int32_t dsa_version(void) { return 102; }

dsa_status dsa_index_scores(const dsa_params* P, const dsa_ragged* R, const void* q_idx,
                            const void* k_idx, const float* w, int64_t q_begin, int64_t q_count,
                            float* scores, int64_t ld, void* stream) {
  DSA_TRY(check_common(P, R));
  DSA_TRY(check_indexer(P));
  if (!q_idx || !k_idx || !w || !scores) return DSA_ERR_INVALID_ARG;
  if (q_begin < 0 || q_count < 0 || q_begin + q_count > R->total_q) return DSA_ERR_INVALID_ARG;
  if (ld < R->max_kv_len || ld % 4 != 0) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx)) return DSA_ERR_INVALID_ARG;
  DeviceState* dev = nullptr;
  DSA_TRY(device_setup(&dev));
  const int bq = R->max_q_len <= 16 ? 16 : 64;
  return launch_index_scores(*dev, P, R, q_idx, k_idx, w, q_begin, q_count, scores, ld, bq,
                             static_cast<cudaStream_t>(stream));
}

dsa_status dsa_topk(const dsa_params* P, const dsa_ragged* R, const float* scores, int64_t ld,
                    int64_t q_begin, int64_t q_count, int32_t* idx, int64_t ld_idx, int32_t* cnt,
                    void* stream) {
  DSA_TRY(check_common(P, R));
  if (!scores || !idx) return DSA_ERR_INVALID_ARG;
  if (q_begin < 0 || q_count < 0 || q_begin + q_count > R->total_q) return DSA_ERR_INVALID_ARG;
  if (ld < R->max_kv_len || ld % 4 != 0 || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
  if (ld_idx < P->top_k) return DSA_ERR_INVALID_ARG;
  if (q_count > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  DeviceState* dev = nullptr;
  DSA_TRY(device_setup(&dev));
  return launch_topk(P, R, scores, ld, q_begin, q_count, idx, ld_idx, cnt,
                     static_cast<cudaStream_t>(stream));
}

dsa_status dsa_sparse_attn_gated(const dsa_params* P, const dsa_ragged* R, const void* q,
                                 const void* k_cache, const void* v_cache, const int32_t* idx,
                                 int64_t ld_idx, int64_t q_begin, int64_t q_count,
                                 const void* gate, void* out, float* lse, int32_t* err_count,
                                 void* stream) {
  DSA_TRY(check_common(P, R));
  DSA_TRY(check_attn(P));
  if (!q || !k_cache || !v_cache || !idx || !out) return DSA_ERR_INVALID_ARG;
  if (q_begin < 0 || q_count < 0 || q_begin + q_count > R->total_q) return DSA_ERR_INVALID_ARG;
  if (ld_idx < P->top_k) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      (gate && !aligned16(gate)))
    return DSA_ERR_INVALID_ARG;
  if (q_count > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  DeviceState* dev = nullptr;
  DSA_TRY(device_setup(&dev));
  return launch_attn(*dev, P, R, q, k_cache, v_cache, idx, ld_idx, q_begin, q_count, gate, out,
                     lse, err_count, static_cast<cudaStream_t>(stream));
}

dsa_status dsa_sparse_attn_gated_mix(const dsa_params* P, const dsa_ragged* R, const void* q,
                                     const void* k_cache, const void* v_cache,
                                     const int32_t* idx, int64_t ld_idx, int64_t q_begin,
                                     int64_t q_count, const void* gate, const void* other,
                                     void* out, float* lse, int32_t* err_count, void* stream) {
  DSA_TRY(check_common(P, R));
  DSA_TRY(check_attn(P));
  if (!q || !k_cache || !v_cache || !idx || !gate || !other || !out) return DSA_ERR_INVALID_ARG;
  if (q_begin < 0 || q_count < 0 || q_begin + q_count > R->total_q) return DSA_ERR_INVALID_ARG;
  if (ld_idx < P->top_k) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      !aligned16(gate) || !aligned16(other))
    return DSA_ERR_INVALID_ARG;
  if (q_count > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  DeviceState* dev = nullptr;
  DSA_TRY(device_setup(&dev));
  return launch_attn(*dev, P, R, q, k_cache, v_cache, idx, ld_idx, q_begin, q_count, gate, out,
                     lse, err_count, static_cast<cudaStream_t>(stream), other);
}

dsa_status dsa_workspace_size(const dsa_params* P, const dsa_ragged* R, int is_decode,
                              size_t* min_bytes, size_t* rec_bytes) {
  DSA_TRY(check_common(P, R));
  const int64_t srow = scores_ld(R) * 4;
  const int64_t irow = round_up((int64_t)P->top_k * 4, 16);
  if (min_bytes) *min_bytes = (size_t)(srow + irow);
  FusedGeom fg;
  const std::vector<RowRun> runs = is_decode ? std::vector<RowRun>() : row_runs(R, 0, R->total_q);
  if (rec_bytes && mixed_runs(runs)) {
    // index rows of every row, plus the largest stretch's steps 1-2 in one pass
    int64_t need = 0;
    const bool can_fuse = fused_geom(P, R, &fg);
    for (const RowRun& r : runs) {
      const int64_t n = r.a1 - r.a0;
      need = std::max(need, r.lng && can_fuse ? fg.fixed_bytes + 256 + n * fg.row_bytes
                                              : score_pass_rows(n, srow) * srow);
    }
    *rec_bytes = (size_t)(round_up(R->total_q * irow, 256) + need);
    return DSA_OK;
  }
  if (rec_bytes && !is_decode && fused_wanted(P, R, &fg)) {
    // one fused pass over every query row
    *rec_bytes = (size_t)(fg.fixed_bytes + 256 + std::max<int64_t>(1, R->total_q) * (fg.row_bytes + irow));
    return DSA_OK;
  }
  if (rec_bytes) {
    // a score sub-pass of up to kScorePassBytes (at least one row per SM) plus index rows
    // for attention passes of up to 16384 query rows
    const int64_t tq = std::max<int64_t>(1, R->total_q);
    int64_t rows_s = std::max<int64_t>(kScorePassBytes / srow, std::min<int64_t>(tq, 148));
    rows_s = std::max<int64_t>(1, std::min(rows_s, tq));
    const int64_t rows_a = std::max(rows_s, std::min<int64_t>(tq, 16384));
    *rec_bytes = (size_t)(rows_s * srow + rows_a * irow);
  }
  return DSA_OK;
}

dsa_status dsa_index_topk_workspace_size(const dsa_params* P, const dsa_ragged* R,
                                         int64_t q_count, size_t* min_bytes, size_t* rec_bytes) {
  DSA_TRY(check_common(P, R));
  DSA_TRY(check_indexer(P));
  if (q_count < 0) return DSA_ERR_INVALID_ARG;
  FusedGeom g;
  if (!fused_geom(P, R, &g)) return DSA_ERR_UNSUPPORTED;
  if (min_bytes) *min_bytes = (size_t)(g.fixed_bytes + g.row_bytes);
  if (rec_bytes) *rec_bytes = (size_t)(g.fixed_bytes + std::max<int64_t>(1, q_count) * g.row_bytes);
  return DSA_OK;
}

dsa_status dsa_index_topk(const dsa_params* P, const dsa_ragged* R, const void* q_idx,
                          const void* k_idx, const float* w, int64_t q_begin, int64_t q_count,
                          int32_t* idx, int64_t ld_idx, int32_t* cnt, void* workspace,
                          size_t ws_bytes, void* stream) {
  DSA_TRY(check_common(P, R));
  DSA_TRY(check_indexer(P));
  if (!q_idx || !k_idx || !w || !idx) return DSA_ERR_INVALID_ARG;
  if (q_begin < 0 || q_count < 0 || q_begin + q_count > R->total_q) return DSA_ERR_INVALID_ARG;
  if (ld_idx < P->top_k) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx)) return DSA_ERR_INVALID_ARG;
  if (q_count > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  FusedGeom g;
  if (!fused_geom(P, R, &g)) return DSA_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255)) return DSA_ERR_WORKSPACE;
  const int64_t rows = std::min<int64_t>(q_count, fused_rows(g, (int64_t)ws_bytes));
  if (fused_rows(g, (int64_t)ws_bytes) < 1) return DSA_ERR_WORKSPACE;
  if (q_count == 0) return DSA_OK;
  DeviceState* dev = nullptr;
  DSA_TRY(device_setup(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const FusedWs f = fused_carve(g, workspace, rows);
  DSA_TRY(fused_prepare(*dev, R, k_idx, g, f, st));
  for (int64_t s0 = q_begin; s0 < q_begin + q_count; s0 += rows) {
    const int64_t n = std::min<int64_t>(rows, q_begin + q_count - s0);
    DSA_TRY(fused_pass(*dev, P, R, q_idx, k_idx, w, s0, n, idx + (s0 - q_begin) * ld_idx, ld_idx,
                       cnt ? cnt + (s0 - q_begin) : nullptr, g, f, st));
  }
  return DSA_OK;
}

// ---------------------------------------------------------------- block granularity
namespace dsa {
namespace {
struct BlockGeom {
  int bshift;
  int64_t ld32, ldb, row_bytes;
};
bool block_geom(const dsa_params* P, const dsa_ragged* R, int block, BlockGeom* g) {
  if (block < 32 || block > 4096 || (block & (block - 1)) != 0) return false;
  g->bshift = 0;
  while ((1 << g->bshift) < block) ++g->bshift;
  const int64_t n = std::max(R->max_kv_len, 1);
  g->ld32 = round_up((n + 31) / 32, 32);
  g->ldb = block > 32 ? round_up((n + block - 1) / block, 32) : 0;
  g->row_bytes = (g->ld32 + g->ldb) * 4 + round_up(P->top_k, 4) * 4;
  return true;
}
}  // namespace
}  // namespace dsa

dsa_status dsa_index_topk_blocks_workspace_size(const dsa_params* P, const dsa_ragged* R,
                                                int32_t block, int64_t q_count, size_t* min_bytes,
                                                size_t* rec_bytes) {
  DSA_TRY(check_common(P, R));
  DSA_TRY(check_indexer(P));
  if (q_count < 0) return DSA_ERR_INVALID_ARG;
  BlockGeom g;
  if (!block_geom(P, R, block, &g)) return DSA_ERR_INVALID_ARG;
  if (min_bytes) *min_bytes = (size_t)(g.row_bytes + 3 * 256);
  if (rec_bytes) *rec_bytes = (size_t)(std::max<int64_t>(1, q_count) * g.row_bytes + 3 * 256);
  return DSA_OK;
}

dsa_status dsa_index_topk_blocks(const dsa_params* P, const dsa_ragged* R, const void* q_idx,
                                 const void* k_idx, const float* w, int32_t block,
                                 int64_t q_begin, int64_t q_count, int32_t* idx, int64_t ld_idx,
                                 int32_t* cnt, void* workspace, size_t ws_bytes, void* stream) {
  DSA_TRY(check_common(P, R));
  DSA_TRY(check_indexer(P));
  BlockGeom g;
  if (!block_geom(P, R, block, &g)) return DSA_ERR_INVALID_ARG;
  if (!q_idx || !k_idx || !w || !idx) return DSA_ERR_INVALID_ARG;
  if (q_begin < 0 || q_count < 0 || q_begin + q_count > R->total_q) return DSA_ERR_INVALID_ARG;
  if (ld_idx < (int64_t)P->top_k * block) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx)) return DSA_ERR_INVALID_ARG;
  if (q_count > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255)) return DSA_ERR_WORKSPACE;
  const int64_t rows = std::min<int64_t>(q_count, ((int64_t)ws_bytes - 3 * 256) / g.row_bytes);
  if (((int64_t)ws_bytes - 3 * 256) / g.row_bytes < 1) return DSA_ERR_WORKSPACE;
  if (q_count == 0) return DSA_OK;
  DeviceState* dev = nullptr;
  DSA_TRY(device_setup(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* p = static_cast<char*>(workspace);
  float* s32 = reinterpret_cast<float*>(p);
  p += round_up(rows * g.ld32 * 4, 256);
  float* sb = reinterpret_cast<float*>(p);
  p += round_up(rows * g.ldb * 4, 256);
  int32_t* blk = reinterpret_cast<int32_t*>(p);
  const int bq = R->max_q_len <= 16 ? 16 : 64;
  for (int64_t s0 = q_begin; s0 < q_begin + q_count; s0 += rows) {
    const int64_t n = std::min<int64_t>(rows, q_begin + q_count - s0);
    IdxVariant v;
    v.bmax = true;
    DSA_TRY(launch_index_scores(*dev, P, R, q_idx, k_idx, w, s0, n, s32, g.ld32, bq, st, v));
    BlockArgs ba;
    std::memset(&ba, 0, sizeof(ba));
    ba.q_offsets = R->q_offsets;
    ba.kv_offsets = R->kv_offsets;
    ba.batch = R->batch;
    ba.q_begin = s0;
    ba.bshift = g.bshift;
    if (block > 32) {
      ba.in = s32;
      ba.ld_in = g.ld32;
      ba.out = sb;
      ba.ld_out = g.ldb;
      StageScope scope(1, st);
      block_max_kernel<<<(unsigned)n, 256, 0, st>>>(ba);
      ++t_launches;
      DSA_TRY(launch_status("block_max_kernel"));
    }
    DSA_TRY(launch_topk(P, R, block > 32 ? sb : s32, block > 32 ? g.ldb : g.ld32, s0, n, blk,
                        P->top_k, nullptr, st, g.bshift));
    ba.blk = blk;
    ba.Kb = P->top_k;
    ba.idx = idx + (s0 - q_begin) * ld_idx;
    ba.ld_idx = ld_idx;
    ba.cnt = cnt ? cnt + (s0 - q_begin) : nullptr;
    {
      StageScope scope(1, st);
      block_expand_kernel<<<(unsigned)n, 256, 0, st>>>(ba);
      ++t_launches;
      DSA_TRY(launch_status("block_expand_kernel"));
    }
  }
  return DSA_OK;
}

// ---------------------------------------------------------------- host buffers, pipelined
namespace dsa {
namespace {
std::mutex g_copy_mu;

dsa_status copy_streams(DeviceState* d, int n_events) {
  std::lock_guard<std::mutex> lock(g_copy_mu);
  if (!d->s_in && cudaStreamCreateWithFlags(&d->s_in, cudaStreamNonBlocking) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (!d->s_out && cudaStreamCreateWithFlags(&d->s_out, cudaStreamNonBlocking) != cudaSuccess)
    return DSA_ERR_CUDA;
  while ((int)d->events.size() < n_events) {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return DSA_ERR_CUDA;
    d->events.push_back(e);
  }
  return DSA_OK;
}

dsa_status h2d(void* dst, const void* src, size_t bytes, cudaStream_t st) {
  if (!bytes) return DSA_OK;
  return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, st) == cudaSuccess ? DSA_OK
                                                                                     : DSA_ERR_CUDA;
}
}  // namespace
}  // namespace dsa

dsa_status dsa_prefill_from_host(const dsa_params* P, const dsa_ragged* R,
                                 const dsa_layer_buffers* host, const dsa_layer_buffers* dev,
                                 int32_t n_chunks, int32_t order, void* workspace,
                                 size_t ws_bytes, void* stream) {
  DSA_TRY(check_common(P, R));
  if (!host || !dev) return DSA_ERR_INVALID_ARG;
  if (R->block_table) return DSA_ERR_UNSUPPORTED;
  if (!host->q_offsets || !host->kv_offsets || !dev->q_offsets || !dev->kv_offsets ||
      !host->q_idx || !host->k_idx || !host->w || !host->q || !host->k_cache ||
      !host->v_cache || !host->out || (dev->gate != nullptr) != (host->gate != nullptr))
    return DSA_ERR_INVALID_ARG;
  const int B = R->batch;
  const int32_t* qo = host->q_offsets;
  const int32_t* ko = host->kv_offsets;
  if (qo[0] != 0 || ko[0] != 0 || qo[B] != R->total_q || ko[B] != R->total_kv)
    return DSA_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b)
    if (qo[b + 1] < qo[b] || ko[b + 1] < ko[b] || qo[b + 1] - qo[b] > ko[b + 1] - ko[b])
      return DSA_ERR_INVALID_ARG;
  dsa_ragged Rd = *R;  // the device offsets are the copies made below
  Rd.q_offsets = dev->q_offsets;
  Rd.kv_offsets = dev->kv_offsets;
  const int64_t TQ = R->total_q;
  if (order < 0 || order > 2) return DSA_ERR_INVALID_ARG;
  if (n_chunks <= 0) n_chunks = (int32_t)std::max<int64_t>(1, std::min<int64_t>(16, TQ / 2048));
  // heaviest ranges first for a few long sequences (causal cost grows along the rows; their
  // cache is small next to the query side); in order otherwise, so that the cache arrives
  // progressively
  const bool reverse = order == 2 || (order == 0 && (int64_t)R->batch * 256 <= TQ);
  n_chunks = (int32_t)std::max<int64_t>(1, std::min<int64_t>(n_chunks, std::max<int64_t>(TQ, 1)));
  DeviceState* d = nullptr;
  DSA_TRY(device_setup(&d));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t e_idx = P->idx_dtype == DSA_FP8_E4M3 ? 1 : 2;
  const size_t idx_row = (size_t)P->n_idx_heads * P->idx_dim * e_idx;
  const size_t q_row = (size_t)P->n_q_heads * P->head_dim * 2;
  const size_t kv_row = (size_t)P->n_kv_heads * P->head_dim * 2;
  const size_t w_bytes = (P->w_row_stride ? (size_t)TQ * P->w_row_stride : P->n_idx_heads) * 4;
  auto at = [](const void* base, size_t off) {
    return const_cast<char*>(static_cast<const char*>(base)) + off;
  };
  // cache rows the queries of rows [a0, a1) see: for every sequence the range touches, up
  // to its last query's position (sequences are packed in order, so this grows with a1)
  auto kv_need_of = [&](int64_t a0, int64_t a1) {
    int b_lo = (int)(std::upper_bound(qo, qo + B + 1, (int32_t)a0) - qo) - 1;
    b_lo = std::max(0, std::min(b_lo, B - 1));
    int64_t need = 0;
    for (int b = b_lo; b < B && qo[b] < a1; ++b) {
      const int64_t last = std::min<int64_t>(a1, qo[b + 1]) - 1;
      if (last < qo[b]) continue;
      const int64_t p = (ko[b + 1] - ko[b]) - (qo[b + 1] - qo[b]) + (last - qo[b]);
      need = std::max<int64_t>(need, ko[b] + p + 1);
    }
    return need;
  };
  // Index rows for every row at the start of the workspace, if it holds them and a pass of
  // steps 1-2 over all rows: then steps 1-2 run once, as soon as the (small) indexer tensors
  // have landed, and only the attention runs per range.
  const int64_t K = P->top_k;
  const int64_t idx_bytes = round_up(TQ * K * 4, 256);
  FusedGeom fg;
  const bool fused = fused_wanted(P, &Rd, &fg);
  const bool split = (int64_t)ws_bytes > idx_bytes &&
                     (fused ? fused_rows(fg, (int64_t)ws_bytes - idx_bytes) >= TQ
                            : ((int64_t)ws_bytes - idx_bytes) / (scores_ld(R) * 4) >= 1);
  // Row ranges.  When only the attention runs per range, what follows the last upload is
  // that range's attention and output read-back: the last range is cut into halves of
  // halves (at most three cuts, none below 256 rows) so that this tail stays short.
  std::vector<int64_t> cut;
  for (int c = 0; c < n_chunks; ++c) cut.push_back(TQ * c / n_chunks);
  if (split)
    for (int s = 0; s < 3 && TQ - cut.back() >= 512; ++s)
      cut.push_back(cut.back() + (TQ - cut.back()) / 2);
  cut.push_back(TQ);
  const int n_ranges = (int)cut.size() - 1;
  // the copy streams and events are shared by the device's calls: one enqueue at a time
  // (a later call's records do not disturb the waits an earlier call already enqueued).
  // The event list grows under the same lock, so no call reads it while it is reallocated.
  std::lock_guard<std::mutex> enqueue_lock(d->enqueue_mu);
  DSA_TRY(copy_streams(d, 2 * n_ranges + 3));
  cudaEvent_t ev_start = d->events[0], ev_end = d->events[1];
  if (cudaEventRecord(ev_start, st) != cudaSuccess ||
      cudaStreamWaitEvent(d->s_in, ev_start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(d->s_out, ev_start, 0) != cudaSuccess)
    return DSA_ERR_CUDA;
  DSA_TRY(h2d(at(dev->q_offsets, 0), qo, (size_t)(B + 1) * 4, d->s_in));
  DSA_TRY(h2d(at(dev->kv_offsets, 0), ko, (size_t)(B + 1) * 4, d->s_in));
  DSA_TRY(h2d(at(dev->w, 0), host->w, w_bytes, d->s_in));
  int64_t kv_done = 0;
  if (split) {
    DSA_TRY(check_indexer(P));
    DSA_TRY(check_attn(P));
    int32_t* idx_all = static_cast<int32_t*>(workspace);
    void* scratch = static_cast<char*>(workspace) + idx_bytes;
    DSA_TRY(h2d(at(dev->q_idx, 0), host->q_idx, (size_t)TQ * idx_row, d->s_in));
    DSA_TRY(h2d(at(dev->k_idx, 0), host->k_idx, (size_t)R->total_kv * idx_row, d->s_in));
    cudaEvent_t ev_idx = d->events[2 + 2 * n_ranges];
    if (cudaEventRecord(ev_idx, d->s_in) != cudaSuccess ||
        cudaStreamWaitEvent(st, ev_idx, 0) != cudaSuccess)
      return DSA_ERR_CUDA;
    DSA_TRY(run_index(*d, P, &Rd, dev->q_idx, dev->k_idx, dev->w, 0, TQ, idx_all, scratch,
                      (size_t)((int64_t)ws_bytes - idx_bytes), st, -1, 0));
    for (int c = 0; c < n_ranges; ++c) {
      const int64_t a0 = cut[c], a1 = cut[c + 1];
      if (a0 == a1) continue;
      const int64_t kv_need = std::max(kv_done, kv_need_of(a0, a1));
      cudaEvent_t ev_in = d->events[2 + 2 * c], ev_done = d->events[3 + 2 * c];
      const size_t r0 = (size_t)kv_done, rn = (size_t)(kv_need - kv_done);
      DSA_TRY(h2d(at(dev->k_cache, r0 * kv_row), at(host->k_cache, r0 * kv_row), rn * kv_row, d->s_in));
      DSA_TRY(h2d(at(dev->v_cache, r0 * kv_row), at(host->v_cache, r0 * kv_row), rn * kv_row, d->s_in));
      kv_done = kv_need;
      const size_t q0 = (size_t)a0, qn = (size_t)(a1 - a0);
      DSA_TRY(h2d(at(dev->q, q0 * q_row), at(host->q, q0 * q_row), qn * q_row, d->s_in));
      if (host->gate)
        DSA_TRY(h2d(at(dev->gate, q0 * q_row), at(host->gate, q0 * q_row), qn * q_row, d->s_in));
      if (cudaEventRecord(ev_in, d->s_in) != cudaSuccess ||
          cudaStreamWaitEvent(st, ev_in, 0) != cudaSuccess)
        return DSA_ERR_CUDA;
      DSA_TRY(launch_attn(*d, P, &Rd, dev->q, dev->k_cache, dev->v_cache, idx_all + a0 * K, K, a0,
                          a1 - a0, dev->gate, dev->out, nullptr, nullptr, st));
      if (cudaEventRecord(ev_done, st) != cudaSuccess ||
          cudaStreamWaitEvent(d->s_out, ev_done, 0) != cudaSuccess ||
          cudaMemcpyAsync(at(host->out, q0 * q_row), at(dev->out, q0 * q_row), qn * q_row,
                          cudaMemcpyDeviceToHost, d->s_out) != cudaSuccess)
        return DSA_ERR_CUDA;
    }
  } else {
    // the layer per range, each range's inputs uploaded just before it
    for (int ci = 0; ci < n_ranges; ++ci) {
      const int c = reverse ? n_chunks - 1 - ci : ci;
      const int64_t a0 = TQ * c / n_chunks, a1 = TQ * (c + 1) / n_chunks;
      if (a0 == a1) continue;
      const int64_t kv_need = std::max(kv_done, kv_need_of(a0, a1));
      cudaEvent_t ev_in = d->events[2 + 2 * ci], ev_done = d->events[3 + 2 * ci];
      const size_t r0 = (size_t)kv_done, rn = (size_t)(kv_need - kv_done);
      DSA_TRY(h2d(at(dev->k_idx, r0 * idx_row), at(host->k_idx, r0 * idx_row), rn * idx_row, d->s_in));
      DSA_TRY(h2d(at(dev->k_cache, r0 * kv_row), at(host->k_cache, r0 * kv_row), rn * kv_row, d->s_in));
      DSA_TRY(h2d(at(dev->v_cache, r0 * kv_row), at(host->v_cache, r0 * kv_row), rn * kv_row, d->s_in));
      kv_done = kv_need;
      const size_t q0 = (size_t)a0, qn = (size_t)(a1 - a0);
      DSA_TRY(h2d(at(dev->q_idx, q0 * idx_row), at(host->q_idx, q0 * idx_row), qn * idx_row, d->s_in));
      DSA_TRY(h2d(at(dev->q, q0 * q_row), at(host->q, q0 * q_row), qn * q_row, d->s_in));
      if (host->gate)
        DSA_TRY(h2d(at(dev->gate, q0 * q_row), at(host->gate, q0 * q_row), qn * q_row, d->s_in));
      if (cudaEventRecord(ev_in, d->s_in) != cudaSuccess ||
          cudaStreamWaitEvent(st, ev_in, 0) != cudaSuccess)
        return DSA_ERR_CUDA;
      DSA_TRY(run_layer(P, &Rd, dev->q_idx, dev->k_idx, dev->w, dev->q, dev->k_cache,
                        dev->v_cache, dev->gate, dev->out, nullptr, nullptr, workspace, ws_bytes,
                        stream, false, a0, a1));
      if (cudaEventRecord(ev_done, st) != cudaSuccess ||
          cudaStreamWaitEvent(d->s_out, ev_done, 0) != cudaSuccess ||
          cudaMemcpyAsync(at(host->out, q0 * q_row), at(dev->out, q0 * q_row), qn * q_row,
                          cudaMemcpyDeviceToHost, d->s_out) != cudaSuccess)
        return DSA_ERR_CUDA;
    }
  }
  // the caller's stream completes after the last copy back
  if (cudaEventRecord(ev_end, d->s_out) != cudaSuccess ||
      cudaStreamWaitEvent(st, ev_end, 0) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status dsa_prefill(const dsa_params* P, const dsa_ragged* R, const void* q_idx,
                       const void* k_idx, const float* w, const void* q, const void* k_cache,
                       const void* v_cache, const void* gate, void* out, int32_t* idx_out,
                       int32_t* err_count, void* workspace, size_t ws_bytes, void* stream) {
  return run_layer(P, R, q_idx, k_idx, w, q, k_cache, v_cache, gate, out, idx_out, err_count,
                   workspace, ws_bytes, stream, false);
}

dsa_status dsa_decode(const dsa_params* P, const dsa_ragged* R, const void* q_idx,
                      const void* k_idx, const float* w, const void* q, const void* k_cache,
                      const void* v_cache, const void* gate, void* out, int32_t* idx_out,
                      int32_t* err_count, void* workspace, size_t ws_bytes, void* stream) {
  return run_layer(P, R, q_idx, k_idx, w, q, k_cache, v_cache, gate, out, idx_out, err_count,
                   workspace, ws_bytes, stream, true);
}

// ---------------------------------------------------------------- allocation-free decode
//
// Scratch for dsa_decode_noalloc: one fixed array in the library's own device memory,
// so callers that cannot allocate never have to.  It is reserved on every GPU that
// loads the library and kept until the process exits.  Host code must not pass the
// symbol itself to a kernel (on the host it names a stand-in, not device memory): the
// first call on each device looks up its device address with cudaGetSymbolAddress.  The
// address belongs to the device's current CUDA context: it is looked up again when the
// context changes (a context created after cudaDeviceReset loads the module anew).
namespace dsa {
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_ptr[kMaxDevices] = {};
uint64_t g_noalloc_ctx[kMaxDevices] = {};
std::mutex g_noalloc_mu;

dsa_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  const uint64_t ctx = current_context_id();
  if (!g_noalloc_ptr[dev] || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
      return DSA_ERR_CUDA;
    g_noalloc_ptr[dev] = ptr;
    g_noalloc_ctx[dev] = current_context_id();
  }
  *out = g_noalloc_ptr[dev];
  return DSA_OK;
}
}  // namespace
}  // namespace dsa

dsa_status dsa_decode_noalloc(const dsa_params* P, const dsa_ragged* R, const void* q_idx,
                              const void* k_idx, const float* w, const void* q,
                              const void* k_cache, const void* v_cache, const void* gate,
                              void* out, int32_t* idx_out, int32_t* err_count, void* stream) {
  DSA_TRY(check_common(P, R));
  // one query row of scores (and its index row) must fit the fixed scratch
  const int64_t row = scores_ld(R) * 4 + (idx_out ? 0 : round_up((int64_t)P->top_k * 4, 16));
  if (row > (int64_t)kNoAllocScratchBytes) return DSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  DSA_TRY(noalloc_scratch(&scratch));
  // Nothing in the scratch has to start at zero: each pass writes every score and index
  // entry it later reads.
  return run_layer(P, R, q_idx, k_idx, w, q, k_cache, v_cache, gate, out, idx_out, err_count,
                   scratch, kNoAllocScratchBytes, stream, true);
}

dsa_status dsa_device_status(void* stream, int32_t* status, int clear) {
  if (!status) return DSA_ERR_INVALID_ARG;
  DeviceState* dev = nullptr;
  DSA_TRY(device_setup(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, dev->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return DSA_ERR_CUDA;
  *status = v;
  if (clear && v != 0) {
    const int zero = 0;
    if (cudaMemcpy(dev->status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

int64_t dsa_launch_count(void) { return t_launches; }

int64_t dsa_fused_rows(int reset) {
  const int64_t n = t_fused_rows;
  if (reset) t_fused_rows = 0;
  return n;
}

dsa_status dsa_stage_timing(int enable) {
  t_timing = enable != 0;
  return DSA_OK;
}

dsa_status dsa_stage_times(double* ms, int64_t* launches, int reset) {
  for (auto& rec : t_pending) {
    if (cudaEventSynchronize(rec.stop) != cudaSuccess) return DSA_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, rec.start, rec.stop) != cudaSuccess) return DSA_ERR_CUDA;
    t_stage_ms[rec.stage] += t;
    t_free_events.push_back(rec.start);
    t_free_events.push_back(rec.stop);
  }
  t_pending.clear();
  for (int s = 0; s < 3; ++s) {
    if (ms) ms[s] = t_stage_ms[s];
    if (launches) launches[s] = t_stage_launches[s];
    if (reset) {
      t_stage_ms[s] = 0;
      t_stage_launches[s] = 0;
    }
  }
  return DSA_OK;
}

}  // extern "C"
