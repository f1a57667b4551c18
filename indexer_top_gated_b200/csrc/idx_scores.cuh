// idx_scores.cuh - step 1 of the layer, the indexer, on tcgen05 tensor cores.
//
//   s[t, j] = sum_h w_h * max(0, c * q_idx[t,h,:] . k_idx[j,h,:]),   j = 0..p(t)
//
// Design (sm_100a):
//  - One CTA owns a tile of BQ consecutive packed query rows (BQ = 64 for prefill,
//    16 when sequences have one query each) and a range of 128-position key tiles.
//  - The key tile is the MMA's M side (128 TMEM lanes = 128 key positions) and the
//    query tile its N side, so in the epilogue each warp holds 32 consecutive key
//    positions of one query row: every score store is a coalesced 128-byte line.
//  - Warp 0 issues TMA loads (128-byte swizzled, one box per indexer head) into a
//    3-stage ring; warp 1 issues tcgen05.mma (one per head and 16-wide K step) into one
//    of two TMEM accumulator buffers; warps 2-17 drain TMEM (tcgen05.ld; four warps per
//    lane quadrant, each taking every fourth 16-column chunk), apply ReLU, the head
//    weights and the head sum, mask causally and store fp32 scores.  Sixteen draining
//    warps (at most 96 registers each) hide the TMEM-load and store latencies better
//    than fewer, larger ones.
//  - Tiles may straddle sequences of a ragged batch: the CTA runs one pass per
//    sequence it touches and masks the other rows.  Tiles are scheduled largest
//    first (the last rows of a sequence see the most keys).
//  - Every wait is bounded; on a timeout the CTA records it, waits (bounded) for its
//    own copies and MMAs in flight, frees TMEM and returns.
//
// Two variants serve the fused indexer -> Top-K path (no score matrix in HBM):
//  - sampled keys (shift > 0): the key tensor holds every 2^shift-th cache position of
//    each sequence (sequence b's samples start at row (kv_offsets[b] >> shift) + b), and
//    sample m stands for position m << shift, so the causal bound becomes m <= p >> shift;
//  - candidates (CAND): instead of storing every score, the epilogue keeps only the
//    scores >= a per-row threshold as (position, score) pairs.  A CTA then owns every
//    key tile of its rows (kt_per_split covers the whole range).  A row's list has one
//    segment per TMEM lane quadrant (cap / 4 slots each), written only by the epilogue
//    warp of that quadrant that owns the row's chunk of 16 rows, so a plain shared
//    counter per (quadrant, row) suffices.  The warp stashes its 16 x 32 block of scores
//    in shared memory and reads it back transposed: each lane then compares 16 keys of
//    one row, counts its hits with one popcount and stores them in a short loop.  The
//    2 KiB per warp come out of the key ring, which has 2 stages in this variant.
//  - 32-key maxima (BMAX), for block-granular selection: through the same transposed
//    block, each row gets the maximum of its scores over every 32 keys it may see (one
//    value per 32 positions instead of 32).
#pragma once

#include "common.cuh"

namespace dsa {

struct IdxArgs {
  const int32_t* q_offsets;
  const int32_t* kv_offsets;
  int batch;
  int n_heads;         // H_i (<= 4)
  int64_t q_begin;     // first packed query row of this launch
  int64_t q_count;     // rows in this launch
  int n_tiles;         // ceil(q_count / BQ)
  int kt_per_split;    // key tiles per blockIdx.y
  const float* w;
  int w_row_stride;
  float scale;         // idx_scale_q * idx_scale_k
  float* scores;
  int64_t ld;
  int* status;
  int shift;           // > 0: key rows are every 2^shift-th position (sampled keys)
  // candidate variant
  const float* thr;    // [q_count] keep scores >= thr[row - q_begin]
  float2* cand;        // [q_count, cap]: 4 segments of cap/4 (position as int bits, score)
  int cap;             // a multiple of 4
  int32_t* cand_cnt;   // [q_count, 4] candidates found per segment (may exceed cap/4)
  CachePages pages;    // paged k_idx (not with sampled keys, which are always contiguous)
  const int32_t* tile_order;  // candidate pass: query tile of each CTA (longest first), or null
};

// first key-tensor row of sequence b
DSA_DEV int64_t idx_key_base(const IdxArgs& a, int b) {
  const int64_t ko = __ldg(a.kv_offsets + b);
  return a.shift ? (ko >> a.shift) + b : ko;
}

constexpr int kIdxStages = 3;      // key ring depth (the candidate variant uses 2)
constexpr int kIdxCandStages = 2;
constexpr int kIdxTileStride = 36;  // floats per row of a warp's score block (no bank conflicts)
constexpr int kIdxTileBytes = 16 * kIdxTileStride * 4;
constexpr int kIdxKeyTile = 128;
constexpr int kIdxEpiWarps = 16;  // four warps per TMEM lane quadrant
constexpr int kIdxSubs = kIdxEpiWarps / 4;
constexpr int kIdxThreads = 64 + 32 * kIdxEpiWarps;

template <bool FP8>
struct IdxGeom {
  static constexpr int kRowBytes = FP8 ? 64 : 128;   // D_i = 64 elements
  static constexpr int kKStep = FP8 ? 32 : 16;       // MMA K per instruction
  static constexpr int kKSteps = 64 / kKStep;
  static constexpr uint32_t kLayout = FP8 ? 4u : 2u; // 64B / 128B swizzle
  static constexpr uint32_t kSbo = 8 * kRowBytes;    // 8-row group stride
};

__host__ __device__ inline int idx_tmem_cols(int n_heads, int bq) {
  int need = 2 * n_heads * bq;
  int c = 32;
  while (c < need) c <<= 1;
  return c;
}

// Dynamic shared memory of one CTA.  A CTA whose TMEM allocation exceeds a quarter of
// the 512 columns asks for enough shared memory that CTAs sharing an SM can never
// oversubscribe TMEM (an allocation that cannot be met would block).
__host__ inline size_t idx_smem_bytes(int n_heads, int bq, bool fp8, bool cand = false) {
  // cand: the variants with the shared score block (candidates, 32-key maxima)
  size_t row = fp8 ? 64 : 128;
  size_t q = (size_t)n_heads * bq * row;
  size_t k = (size_t)(cand ? kIdxCandStages : kIdxStages) * n_heads * kIdxKeyTile * row;
  size_t bytes = 1024 /*align slack*/ + q + k + 256 /*barriers*/ +
                 (cand ? (size_t)kIdxEpiWarps * kIdxTileBytes : 0);
  const int cols = idx_tmem_cols(n_heads, bq);
  if (cols > 256 && bytes < 120 * 1024) bytes = 120 * 1024;       // 1 CTA per SM
  else if (cols > 128 && bytes < 80 * 1024) bytes = 80 * 1024;    // <= 2 CTAs per SM
  else if (cols > 64 && bytes < 58 * 1024) bytes = 58 * 1024;     // <= 3 CTAs per SM
  return bytes;
}

// Variants of the epilogue: every score, candidates only, or the maximum of each 32 keys.
// kIdxSamples: as kIdxScores, stored as bf16 rounded toward -infinity (the sampled pass of
// the fused path: its samples only set a lower bound of a threshold, so rounding them down
// keeps every bound valid and halves their bytes).
enum IdxMode { kIdxScores = 0, kIdxCand = 1, kIdxBlockMax = 2, kIdxSamples = 3 };

template <int BQ, bool FP8, int MODE>
__global__ void __launch_bounds__(kIdxThreads, 1)
    idx_scores_kernel(const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_k, IdxArgs a) {
  using Geo = IdxGeom<FP8>;
  constexpr bool CAND = MODE == kIdxCand;
  constexpr bool BMAX = MODE == kIdxBlockMax;
  constexpr bool TILE = CAND || BMAX;  // the epilogue goes through the shared score block
  constexpr int ST = TILE ? kIdxCandStages : kIdxStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int H = a.n_heads;
  const uint32_t q_head_bytes = BQ * Geo::kRowBytes;
  const uint32_t k_head_bytes = kIdxKeyTile * Geo::kRowBytes;
  uint8_t* sQ = smem;
  uint8_t* sK = smem + H * q_head_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sK + (size_t)ST * H * k_head_bytes);
  uint64_t* full = bars;            // [ST]
  uint64_t* empty = bars + ST;      // [ST]
  uint64_t* tfull = bars + 2 * ST;  // [2]
  uint64_t* tempty = tfull + 2;     // [2]
  uint64_t* qfull = tempty + 2;     // [1]
  float* tiles = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 256);  // TILE
  __shared__ uint32_t s_tmem;
  __shared__ int s_bfirst, s_blast;
  __shared__ volatile int s_abort;
  __shared__ int s_consumed;  // jobs whose smem stage the MMA warp has released
  __shared__ float s_thr[CAND ? BQ : 1];
  __shared__ uint32_t s_cnt[CAND ? 4 : 1][CAND ? BQ : 1];  // candidates per (quadrant, row)

  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  const int tile = a.n_tiles - 1 - (int)blockIdx.x;  // largest first
  const int64_t r0 = a.q_begin + (int64_t)tile * BQ;
  const int64_t q_end = a.q_begin + a.q_count;
  const int64_t r_last = (r0 + BQ < q_end ? r0 + BQ : q_end) - 1;
  const int kt_lo = (int)blockIdx.y * a.kt_per_split;

  if (threadIdx.x == 0) {
    s_bfirst = seq_of_row(a.q_offsets, a.batch, r0);
    s_blast = seq_of_row(a.q_offsets, a.batch, r_last);
    s_abort = 0;
    s_consumed = 0;
  }
  __syncthreads();
  const int b_first = s_bfirst, b_last = s_blast;

  // Jobs of this CTA: for each sequence b in the tile, key tiles [kt_lo, kt_hi(b)).
  auto seq_range = [&](int b, int64_t& rs, int64_t& re, int& kt_hi, int64_t& pbase) -> bool {
    int64_t qo = __ldg(a.q_offsets + b), qn = __ldg(a.q_offsets + b + 1);
    int64_t ko = __ldg(a.kv_offsets + b), kn = __ldg(a.kv_offsets + b + 1);
    rs = r0 > qo ? r0 : qo;
    re = (r_last + 1) < qn ? (r_last + 1) : qn;
    if (rs >= re) return false;
    pbase = (kn - ko) - (qn - qo) - qo;  // p(r) = pbase + r
    int64_t pmax = pbase + re - 1;
    if (pmax < 0) return false;
    int n_kt = (int)((pmax >> a.shift) / kIdxKeyTile) + 1;
    kt_hi = n_kt < kt_lo + a.kt_per_split ? n_kt : kt_lo + a.kt_per_split;
    return kt_lo < kt_hi;
  };

  int n_jobs = 0;
  for (int b = b_first; b <= b_last; ++b) {
    int64_t rs, re, pb;
    int kh;
    if (seq_range(b, rs, re, kh, pb)) n_jobs += kh - kt_lo;
  }
  if (n_jobs == 0) {  // uniform across the CTA
    if (CAND)
      for (int c = threadIdx.x; c < 4 * BQ; c += blockDim.x)
        if (r0 + c / 4 <= r_last) a.cand_cnt[(r0 - a.q_begin) * 4 + c] = 0;
    return;
  }
  if (CAND) {
    for (int c = threadIdx.x; c < BQ; c += blockDim.x)
      s_thr[c] = r0 + c <= r_last ? __ldg(a.thr + (r0 + c - a.q_begin)) : INFINITY;
    for (int c = threadIdx.x; c < 4 * BQ; c += blockDim.x) s_cnt[c / BQ][c % BQ] = 0;
  }

  const int ncols = idx_tmem_cols(H, BQ);
  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), kIdxEpiWarps);
    }
    mbar_init(smem_u32(qfull), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&s_tmem), (uint32_t)ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmap_q);
      prefetch_tensormap(&tmap_k);
      mbar_arrive_expect_tx(smem_u32(qfull), H * q_head_bytes);
      for (int h = 0; h < H; ++h)
        tma_load_2d(smem_u32(sQ + h * q_head_bytes), &tmap_q, smem_u32(qfull), h * 64, (int)r0);
      int i = 0;
      bool ok = true;
      for (int b = b_first; b <= b_last && ok; ++b) {
        int64_t rs, re, pb;
        int kh;
        if (!seq_range(b, rs, re, kh, pb)) continue;
        const int64_t kbase = idx_key_base(a, b);
        for (int kt = kt_lo; kt < kh; ++kt, ++i) {
          // a key tile never straddles a page (pages are multiples of 128 positions)
          const int64_t krow = a.pages.table ? cache_row(a.kv_offsets, a.pages, b, (int64_t)kt * kIdxKeyTile)
                                             : kbase + (int64_t)kt * kIdxKeyTile;
          const int s = i % ST;
          if (!mbar_wait_bounded(smem_u32(&empty[s]), ((i / ST) & 1) ^ 1, a.status, &s_abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(smem_u32(&full[s]), H * k_head_bytes);
          for (int h = 0; h < H; ++h)
            tma_load_2d(smem_u32(sK + ((size_t)s * H + h) * k_head_bytes), &tmap_k,
                        smem_u32(&full[s]), h * 64, (int)krow);
        }
      }
      if (!ok) {
        // drain: every issued load lands before the CTA exits
        mbar_wait_bounded(smem_u32(qfull), 0, nullptr, nullptr);
        for (int j = s_consumed; j < i; ++j)
          mbar_wait_bounded(smem_u32(&full[j % ST]), (j / ST) & 1, nullptr, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = umma_idesc(128, BQ, FP8 ? 0u : 1u);
    int i = 0;
    int issued = 0;
    bool ok = mbar_wait_bounded(smem_u32(qfull), 0, a.status, &s_abort);
    for (int b = b_first; b <= b_last && ok; ++b) {
      int64_t rs, re, pb;
      int kh;
      if (!seq_range(b, rs, re, kh, pb)) continue;
      for (int kt = kt_lo; kt < kh; ++kt, ++i) {
        const int s = i % ST, buf = i & 1;
        if (!mbar_wait_bounded(smem_u32(&full[s]), (i / ST) & 1, a.status, &s_abort) ||
            !mbar_wait_bounded(smem_u32(&tempty[buf]), ((i >> 1) & 1) ^ 1, a.status, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          for (int h = 0; h < H; ++h) {
            const uint32_t a_base = smem_u32(sK + ((size_t)s * H + h) * k_head_bytes);
            const uint32_t b_base = smem_u32(sQ + h * q_head_bytes);
            const uint32_t d = tmem + (uint32_t)(buf * H * BQ + h * BQ);
#pragma unroll
            for (int kk = 0; kk < Geo::kKSteps; ++kk) {
              const uint64_t ad = umma_smem_desc(a_base + kk * 32, Geo::kSbo, Geo::kLayout);
              const uint64_t bd = umma_smem_desc(b_base + kk * 32, Geo::kSbo, Geo::kLayout);
              if (FP8) umma_fp8(d, ad, bd, idesc, kk > 0);
              else umma_bf16(d, ad, bd, idesc, kk > 0);
            }
          }
          umma_commit(smem_u32(&empty[s]));
          umma_commit(smem_u32(&tfull[buf]));
        }
        __syncwarp();
        issued = i + 1;
        if (lane == 0) s_consumed = i + 1;
      }
    }
    if (!ok && issued > 0 && lane == 0) {
      // the last commit completes after every MMA issued before it
      const int j = issued - 1;
      mbar_wait_bounded(smem_u32(&tfull[j & 1]), (j >> 1) & 1, nullptr, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-17)
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
    const int sub = (warp - 2) >> 2;  // the warps of a quadrant take every kIdxSubs-th chunk
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    // shared head weights with the (positive) dequantisation scale folded in:
    // w * max(0, c * x) = (w * c) * max(0, x) for c > 0
    // (unrolled with constant indices, so that the weights stay in registers)
    float wsh[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) wsh[h] = (a.w_row_stride == 0 && h < H) ? __ldg(a.w + h) * a.scale : 0.f;
    // candidate variant: this warp's score block (the chunk of rows c0 always goes to
    // the warp with sub = (c0 / 16) % kIdxSubs, so each (quadrant, row) has one writer)
    float* tile = tiles + (warp - 2) * (kIdxTileBytes / 4);
    int i = 0;
    bool ok = true;
    for (int b = b_first; b <= b_last && ok; ++b) {
      int64_t rs, re, pbase;
      int kh;
      if (!seq_range(b, rs, re, kh, pbase)) continue;
      // 32-bit from here on (positions and rows of a launch stay below 2^31): p0 is the
      // position of tile row 0 in sequence b (row cc sees keys up to (p0 + cc) >> shift)
      const int p0 = (int)(pbase + r0);
      const int row0 = (int)(r0 - a.q_begin);
      for (int kt = kt_lo; kt < kh; ++kt, ++i) {
        const int buf = i & 1;
        if (!mbar_wait_bounded(smem_u32(&tfull[buf]), (i >> 1) & 1, a.status, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int j = kt * kIdxKeyTile + quad * 32 + lane;  // key position
        // columns c of this tile that belong to sequence b: rows rs..re-1
        const int c_lo = (int)(rs - r0), c_hi = (int)(re - r0);
        for (int c0 = 16 * sub; c0 < c_hi; c0 += 16 * kIdxSubs) {
          if (c0 + 16 <= c_lo) continue;  // rows of an earlier sequence of the tile
          // skip chunks whose rows all precede this key tile (causal)
          const int p_chunk_max = (p0 + (c0 + 15 < c_hi - 1 ? c0 + 15 : c_hi - 1)) >> a.shift;
          if (p_chunk_max < kt * kIdxKeyTile) continue;
          // heads in groups of HPB (two, or one in the candidate variant, which needs the
          // registers): HPB TMEM loads in flight, then their ReLU-weighted sum (the
          // accumulation order over heads is 0, 1, 2, 3 either way)
          constexpr int HPB = TILE ? 1 : 2;
          float acc[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) acc[c] = 0.f;
#pragma unroll
          for (int hp = 0; hp < 4; hp += HPB) {
            if (hp >= H) break;
            uint32_t v[HPB][16];
#pragma unroll
            for (int q = 0; q < HPB; ++q)
              if (hp + q < H)
                tmem_ld16_async(tmem + lane_base + (uint32_t)(buf * H * BQ + (hp + q) * BQ + c0), v[q]);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < HPB; ++q) {
              const int h = hp + q;
              if (h >= H) break;
              reg_fence(v[q]);
              if (a.w_row_stride == 0) {
                // two columns per packed fma (each lane of it rounds like fmaf)
                const float2 w2 = make_float2(wsh[h], wsh[h]);
#pragma unroll
                for (int c = 0; c < 16; c += 2) {
                  const float2 x = make_float2(fmaxf(__uint_as_float(v[q][c]), 0.f),
                                               fmaxf(__uint_as_float(v[q][c + 1]), 0.f));
                  const float2 r2 = __ffma2_rn(w2, x, make_float2(acc[c], acc[c + 1]));
                  acc[c] = r2.x;
                  acc[c + 1] = r2.y;
                }
              } else {
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                  int64_t r = r0 + c0 + c;
                  if (r > r_last) r = r_last;
                  const float wv = __ldg(a.w + r * a.w_row_stride + h);
                  acc[c] = fmaf(wv, fmaxf(__uint_as_float(v[q][c]) * a.scale, 0.f), acc[c]);
                }
              }
            }
          }
          // rows r0+c0 .. r0+c0+15; key j.  Interior chunk: every row belongs to this
          // sequence and sees the whole key tile, so no per-element predicate is needed.
          const bool inside = c0 >= c_lo && c0 + 16 <= c_hi &&
                              kt * kIdxKeyTile + (kIdxKeyTile - 1) <= ((p0 + c0) >> a.shift);
          if (BMAX) {
            // the maximum of each row over this warp's 32 keys (those the row may see)
#pragma unroll
            for (int c = 0; c < 16; ++c) tile[c * kIdxTileStride + lane] = acc[c];
            __syncwarp();
            const int rr = lane & 15, kh = (lane >> 4) * 16;
            const float* trow = tile + rr * kIdxTileStride + kh;
            const int cc = c0 + rr;
            int k_lim = 16;
            if (!inside) {
              const int pr = (p0 + cc) >> a.shift;
              const int lim = pr - (kt * kIdxKeyTile + quad * 32 + kh) + 1;
              k_lim = (cc < c_lo || cc >= c_hi || lim <= 0) ? 0 : lim >= 16 ? 16 : lim;
            }
            float mx = -INFINITY;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 x = *reinterpret_cast<const float4*>(trow + 4 * q);
              if (4 * q < k_lim) mx = fmaxf(mx, x.x);
              if (4 * q + 1 < k_lim) mx = fmaxf(mx, x.y);
              if (4 * q + 2 < k_lim) mx = fmaxf(mx, x.z);
              if (4 * q + 3 < k_lim) mx = fmaxf(mx, x.w);
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 16));
            const int seen = __shfl_xor_sync(0xFFFFFFFFu, k_lim, 16) + k_lim;
            if (lane < 16 && seen > 0)
              a.scores[(int64_t)(row0 + cc) * a.ld + kt * 4 + quad] = mx;
            __syncwarp();  // the block is read before the next chunk overwrites it
            continue;
          }
          if (CAND) {
            // keep the scores >= the row's threshold (float order; -0.0 == +0.0)
#pragma unroll
            for (int c = 0; c < 16; ++c) tile[c * kIdxTileStride + lane] = acc[c];
            __syncwarp();
            // lane l: row rr = l & 15 of the chunk, keys kh .. kh+15 of the warp's 32
            const int rr = lane & 15, kh = (lane >> 4) * 16;
            const float* trow = tile + rr * kIdxTileStride + kh;
            const int cc = c0 + rr;
            const float th = s_thr[cc];
            // keys of this lane that the row may see: k < k_lim
            int k_lim = 16;
            if (!inside) {
              const int pr = (p0 + cc) >> a.shift;  // last key row the row sees
              const int lim = pr - (kt * kIdxKeyTile + quad * 32 + kh) + 1;
              k_lim = (cc < c_lo || cc >= c_hi || lim <= 0) ? 0 : lim >= 16 ? 16 : lim;
            }
            uint32_t m = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 x = *reinterpret_cast<const float4*>(trow + 4 * q);
              m |= ((uint32_t)(x.x >= th) | ((uint32_t)(x.y >= th) << 1) | ((uint32_t)(x.z >= th) << 2) |
                    ((uint32_t)(x.w >= th) << 3)) << (4 * q);
            }
            m &= k_lim >= 16 ? 0xFFFFu : ((1u << k_lim) - 1u);
            const uint32_t n_lo = __shfl_sync(0xFFFFFFFFu, (uint32_t)__popc(m), lane & 15);
            uint32_t base = lane < 16 ? s_cnt[quad][cc] : 0u;
            base = __shfl_sync(0xFFFFFFFFu, base, lane & 15) + (lane >= 16 ? n_lo : 0u);
            const uint32_t n_hi = __shfl_sync(0xFFFFFFFFu, (uint32_t)__popc(m), 16 + (lane & 15));
            if (lane < 16) s_cnt[quad][cc] = base + n_lo + n_hi;
            const int seg = a.cap >> 2;
            float2* dst = a.cand + (int64_t)(row0 + cc) * a.cap + quad * seg;
            const int j0 = kt * kIdxKeyTile + quad * 32 + kh;
            while (m) {
              const int k = __ffs(m) - 1;
              m &= m - 1;
              if (base < (uint32_t)seg) dst[base] = make_float2(__int_as_float(j0 + k), trow[k]);
              ++base;
            }
            __syncwarp();  // the block is read before the next chunk overwrites it
            continue;
          }
          const bool interior = inside && (int64_t)kt * kIdxKeyTile + kIdxKeyTile <= a.ld;
          if (MODE == kIdxSamples) {
            __nv_bfloat16* dst16 =
                reinterpret_cast<__nv_bfloat16*>(a.scores) + (int64_t)(row0 + c0) * a.ld + j;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int cc = c0 + c;
              if (interior || (cc >= c_lo && cc < c_hi && j <= ((p0 + cc) >> a.shift) && j < a.ld))
                *dst16 = __float2bfloat16_rd(acc[c]);
              dst16 += a.ld;
            }
          } else {
            float* dst = a.scores + (int64_t)(row0 + c0) * a.ld + j;
            if (interior) {
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                *dst = acc[c];
                dst += a.ld;
              }
            } else {
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                const int cc = c0 + c;
                if (cc >= c_lo && cc < c_hi && j <= ((p0 + cc) >> a.shift) && j < a.ld) *dst = acc[c];
                dst += a.ld;
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&tempty[buf]));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, (uint32_t)ncols);
  }
  if (CAND)
    for (int c = threadIdx.x; c < 4 * BQ; c += blockDim.x)
      if (r0 + c / 4 <= r_last) a.cand_cnt[(r0 - a.q_begin) * 4 + c] = (int32_t)s_cnt[c % 4][c / 4];
}

// Sampled key tensor of the fused path: row (kv_offsets[b] >> shift) + b + m holds position
// m << shift of sequence b (cache row kv_offsets[b] + (m << shift), or its page), for every
// sequence b and m < ceil(L_b / 2^shift); rows between sequences are zero.  One warp per
// row, `vec` 16-byte words per row.
__global__ void __launch_bounds__(256) idx_sample_keys_kernel(const int32_t* kv_offsets,
                                                              int batch, int shift,
                                                              const uint4* k, uint4* ks,
                                                              int vec, int64_t rows,
                                                              CachePages pages) {
  const int lane = lane_id();
  const int64_t n_warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); g < rows;
       g += n_warps) {
    int lo = 0, hi = batch - 1;  // last sequence whose sample rows start at or before g
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (((int64_t)__ldg(kv_offsets + mid) >> shift) + mid <= g) lo = mid;
      else hi = mid - 1;
    }
    const int64_t ko = __ldg(kv_offsets + lo), kn = __ldg(kv_offsets + lo + 1);
    const int64_t m = g - ((ko >> shift) + lo);
    const bool real = m >= 0 && ko + (m << shift) < kn;
    const int64_t src = real ? cache_row(kv_offsets, pages, lo, m << shift) : 0;
    for (int v = lane; v < vec; v += 32)
      ks[g * vec + v] = real ? __ldg(k + src * vec + v) : make_uint4(0u, 0u, 0u, 0u);
  }
}

}  // namespace dsa
