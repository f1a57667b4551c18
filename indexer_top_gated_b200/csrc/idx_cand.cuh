// idx_cand.cuh - the candidate pass of the fused indexer -> Top-K path, query-major.
//
//   s[t, j] = sum_h w_h * max(0, c * q_idx[t,h,:] . k_idx[j,h,:]),   j = 0..p(t)
//
// keeping only the (position, score) pairs with s >= thr[t] (the row's sampled threshold).
// Same scores as idx_scores_kernel, laid out the other way round on the tensor core:
//  - One CTA owns 128 consecutive packed query rows and every key tile they can see (so it
//    owns their candidate lists).  The query tile is the MMA's M side: TMEM lane = query
//    row, columns = keys (128 per tile and head), so each epilogue thread owns one query
//    row.  The ReLU-weighted head sum, the threshold compare and the candidate emission are
//    then private to the thread: no transposition, no shuffles, no shared counters.
//  - The accumulators are two TMEM slots of 256 columns, one per head pair (heads 0-1 and
//    2-3 of a 128-key tile).  A 128 x 128 x 16 UMMA runs at the tensor core's full rate
//    where a 128 x 64 one is bound by its shared-memory operand reads, and the slot of one
//    head pair is drained while the MMAs of the other run, so the commit -> drain -> release
//    round trip overlaps tensor-core work.
//  - Warp 0 issues TMA loads (128-byte swizzle, one box per indexer head; the query tile
//    once, then a 3-stage ring of half key tiles, one head pair each); warp 1 issues
//    tcgen05.mma (A = query tile, B = key tile, one UMMA per head and K step); warps 2-17
//    drain TMEM: the four warps of a lane quadrant take 32 key columns each (segment
//    sub = 0..3 of the row's candidate list), so that four warps per scheduler hide each
//    other's TMEM-load and dependency latencies.
//  - A thread appends its hits to a small staging area of its own in shared memory and
//    writes them to its segment in whole 32-byte sectors (4 pairs), so the candidate stream
//    leaves the SM in full sectors instead of one scattered 8-byte store per hit.
//  - The TMEM buffer is released as soon as its four heads are in registers, before the
//    emission, so the MMAs of the next tiles overlap it.
// Tiles may straddle sequences of a ragged batch (one pass per sequence, other rows masked
// by an infinite threshold).  Every wait is bounded; on a timeout the CTA records it, waits
// (bounded) for its own copies and MMAs in flight, frees TMEM and returns.
#pragma once

#include "common.cuh"
#include "idx_scores.cuh"

namespace dsa {

constexpr int kCandBQ = 128;       // query rows per CTA (MMA M, TMEM lanes)
constexpr int kCandKT = 128;       // keys per tile (MMA N)
constexpr int kCandStages = 3;     // ring depth in half key tiles (one head pair each)
constexpr int kCandEpiWarps = 16;  // four per TMEM lane quadrant
constexpr int kCandThreads = 64 + 32 * kCandEpiWarps;
constexpr int kCandSegs = 4;       // candidate segments per row (one per 32 key columns)
constexpr int kCandCols = kCandKT / kCandSegs;   // key columns per epilogue warp and tile
constexpr int kCandSlotCols = 2 * kCandKT;       // TMEM columns of one head-pair slot
constexpr int kCandSlots = 14;     // staging slots (8-byte pairs) per (row, segment)
constexpr int kCandSlotStride = kCandSlots * 8;  // 112 B: 16-byte aligned, banks spread by row

template <bool FP8>
__host__ __device__ constexpr size_t cand_q_bytes() { return (size_t)4 * kCandBQ * (FP8 ? 64 : 128); }
template <bool FP8>
__host__ __device__ constexpr size_t cand_k_stage_bytes() { return (size_t)2 * kCandKT * (FP8 ? 64 : 128); }

__host__ inline size_t idx_cand_smem_bytes(bool fp8) {
  const size_t q = fp8 ? cand_q_bytes<true>() : cand_q_bytes<false>();
  const size_t k = kCandStages * (fp8 ? cand_k_stage_bytes<true>() : cand_k_stage_bytes<false>());
  size_t bytes = 1024 /*align*/ + q + k + 256 /*barriers*/ +
                 (size_t)kCandSegs * kCandBQ * kCandSlotStride;
  // the CTA takes all 512 TMEM columns: ask for enough shared memory that no second CTA
  // can share the SM (an allocation that cannot be met would block)
  if (bytes < 120 * 1024) bytes = 120 * 1024;
  return bytes;
}

template <bool FP8>
__global__ void __launch_bounds__(kCandThreads, 1)
    idx_cand_kernel(const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_k, IdxArgs a) {
  using Geo = IdxGeom<FP8>;
  constexpr uint32_t kQHead = kCandBQ * Geo::kRowBytes;  // one head of the query tile
  constexpr uint32_t kKHead = kCandKT * Geo::kRowBytes;  // one head of a key tile
  constexpr int ST = kCandStages;
  constexpr int kCols = 2 * kCandSlotCols;               // TMEM columns (2 head-pair slots)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + 4 * kQHead;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sK + (size_t)ST * 2 * kKHead);
  uint64_t* full = bars;            // [ST]
  uint64_t* empty = bars + ST;      // [ST]
  uint64_t* tfull = bars + 2 * ST;  // [2] per head-pair slot
  uint64_t* tempty = tfull + 2;     // [2]
  uint64_t* qfull = tempty + 2;     // [1]
  uint8_t* stage_base = reinterpret_cast<uint8_t*>(bars) + 256;  // [segs][128 rows][slots]
  __shared__ uint32_t s_tmem;
  __shared__ int s_bfirst, s_blast;
  __shared__ volatile int s_abort;
  __shared__ int s_consumed;

  const int H = a.n_heads;
  const int n_pairs = (H + 1) >> 1;  // head pairs (the last may hold one head)
  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  // longest first: for one sequence the last tiles; for a batch the order idx_cand_order_kernel
  // found
  const int tile = a.tile_order ? __ldg(a.tile_order + blockIdx.x) : a.n_tiles - 1 - (int)blockIdx.x;
  const int64_t r0 = a.q_begin + (int64_t)tile * kCandBQ;
  const int64_t q_end = a.q_begin + a.q_count;
  const int64_t r_last = (r0 + kCandBQ < q_end ? r0 + kCandBQ : q_end) - 1;

  if (threadIdx.x == 0) {
    s_bfirst = seq_of_row(a.q_offsets, a.batch, r0);
    s_blast = seq_of_row(a.q_offsets, a.batch, r_last);
    s_abort = 0;
    s_consumed = 0;
  }
  __syncthreads();
  const int b_first = s_bfirst, b_last = s_blast;

  // rows rs..re-1 of the tile belong to sequence b; its key tiles are 0..kt_hi-1
  auto seq_range = [&](int b, int64_t& rs, int64_t& re, int& kt_hi, int64_t& pbase) -> bool {
    const int64_t qo = __ldg(a.q_offsets + b), qn = __ldg(a.q_offsets + b + 1);
    const int64_t ko = __ldg(a.kv_offsets + b), kn = __ldg(a.kv_offsets + b + 1);
    rs = r0 > qo ? r0 : qo;
    re = (r_last + 1) < qn ? (r_last + 1) : qn;
    if (rs >= re) return false;
    pbase = (kn - ko) - (qn - qo) - qo;  // p(r) = pbase + r
    const int64_t pmax = pbase + re - 1;
    if (pmax < 0) return false;
    kt_hi = (int)(pmax / kCandKT) + 1;
    return true;
  };

  int n_jobs = 0;
  for (int b = b_first; b <= b_last; ++b) {
    int64_t rs, re, pb;
    int kh;
    if (seq_range(b, rs, re, kh, pb)) n_jobs += kh;
  }
  if (n_jobs == 0) {  // uniform across the CTA
    for (int c = threadIdx.x; c < 4 * kCandBQ; c += blockDim.x)
      if (r0 + c / 4 <= r_last) a.cand_cnt[(r0 - a.q_begin) * 4 + c] = 0;
    return;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), kCandEpiWarps);
    }
    mbar_init(smem_u32(qfull), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&s_tmem), (uint32_t)kCols);
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
      mbar_arrive_expect_tx(smem_u32(qfull), H * kQHead);
      for (int h = 0; h < H; ++h)
        tma_load_2d(smem_u32(sQ + h * kQHead), &tmap_q, smem_u32(qfull), h * 64, (int)r0);
      int u = 0;  // half key tiles issued
      bool ok = true;
      for (int b = b_first; b <= b_last && ok; ++b) {
        int64_t rs, re, pb;
        int kh;
        if (!seq_range(b, rs, re, kh, pb)) continue;
        const int64_t kbase = __ldg(a.kv_offsets + b);
        for (int kt = 0; kt < kh && ok; ++kt) {
          // a 128-key tile never straddles a page (pages are multiples of 128 positions)
          const int64_t krow = a.pages.table ? cache_row(a.kv_offsets, a.pages, b, (int64_t)kt * kCandKT)
                                             : kbase + (int64_t)kt * kCandKT;
          for (int pr = 0; pr < n_pairs; ++pr, ++u) {
            const int s = u % ST;
            const int nh = H - 2 * pr < 2 ? H - 2 * pr : 2;
            if (!mbar_wait_bounded(smem_u32(&empty[s]), ((u / ST) & 1) ^ 1, a.status, &s_abort)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(smem_u32(&full[s]), nh * kKHead);
            for (int hh = 0; hh < nh; ++hh)
              tma_load_2d(smem_u32(sK + ((size_t)s * 2 + hh) * kKHead), &tmap_k, smem_u32(&full[s]),
                          (2 * pr + hh) * 64, (int)krow);
          }
        }
      }
      if (!ok) {
        mbar_wait_bounded(smem_u32(qfull), 0, nullptr, nullptr);
        for (int j = s_consumed; j < u; ++j)
          mbar_wait_bounded(smem_u32(&full[j % ST]), (j / ST) & 1, nullptr, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = umma_idesc(kCandBQ, kCandKT, FP8 ? 0u : 1u);
    int i = 0, u = 0;                // key tiles, half key tiles consumed
    int last_pr = -1, last_i = 0;    // slot and tile of the last commit
    bool ok = mbar_wait_bounded(smem_u32(qfull), 0, a.status, &s_abort);
    for (int b = b_first; b <= b_last && ok; ++b) {
      int64_t rs, re, pb;
      int kh;
      if (!seq_range(b, rs, re, kh, pb)) continue;
      for (int kt = 0; kt < kh && ok; ++kt, ++i) {
        for (int pr = 0; pr < n_pairs; ++pr, ++u) {
          // slot pr is used once per key tile: its i-th use waits for the (i-1)-th release
          const int s = u % ST;
          const int nh = H - 2 * pr < 2 ? H - 2 * pr : 2;
          if (!mbar_wait_bounded(smem_u32(&full[s]), (u / ST) & 1, a.status, &s_abort) ||
              !mbar_wait_bounded(smem_u32(&tempty[pr]), (i & 1) ^ 1, a.status, &s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            for (int hh = 0; hh < nh; ++hh) {
              const uint32_t a_base = smem_u32(sQ + (2 * pr + hh) * kQHead);
              const uint32_t b_base = smem_u32(sK + ((size_t)s * 2 + hh) * kKHead);
              const uint32_t d = tmem + (uint32_t)(pr * kCandSlotCols + hh * kCandKT);
#pragma unroll
              for (int kk = 0; kk < Geo::kKSteps; ++kk) {
                const uint64_t ad = umma_smem_desc(a_base + kk * 32, Geo::kSbo, Geo::kLayout);
                const uint64_t bd = umma_smem_desc(b_base + kk * 32, Geo::kSbo, Geo::kLayout);
                if (FP8) umma_fp8(d, ad, bd, idesc, kk > 0);
                else umma_bf16(d, ad, bd, idesc, kk > 0);
              }
            }
            umma_commit(smem_u32(&empty[s]));
            umma_commit(smem_u32(&tfull[pr]));
          }
          __syncwarp();
          last_pr = pr;
          last_i = i;
          if (lane == 0) s_consumed = u + 1;
        }
      }
    }
    if (!ok && last_pr >= 0 && lane == 0)  // the last commit completes after every earlier MMA
      mbar_wait_bounded(smem_u32(&tfull[last_pr]), last_i & 1, nullptr, nullptr);
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-17)
    const int quad = warp & 3;          // TMEM lanes 32 quad .. 32 quad + 31
    const int sub = (warp - 2) >> 2;    // key columns 32 sub .. 32 sub + 31 of each tile
    const int rr = quad * 32 + lane;    // this thread's row within the tile
    const int64_t row = r0 + rr;
    const bool in_launch = row <= r_last;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    // shared head weights with the (positive) dequantisation scale folded in:
    // w * max(0, c * x) = (w * c) * max(0, x) for c > 0; per-row weights take c on the dot
    float wsh[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      if (h >= H) wsh[h] = 0.f;
      else if (a.w_row_stride == 0) wsh[h] = __ldg(a.w + h) * a.scale;
      else wsh[h] = in_launch ? __ldg(a.w + row * a.w_row_stride + h) : 0.f;
    }
    const bool row_w = a.w_row_stride != 0;
    const float thr_row = in_launch ? __ldg(a.thr + (row - a.q_begin)) : INFINITY;
    const int seg = a.cap / kCandSegs;
    float2* dst = a.cand + (in_launch ? (row - a.q_begin) : 0) * (int64_t)a.cap + sub * seg;
    uint8_t* stg = stage_base + ((size_t)sub * kCandBQ + rr) * kCandSlotStride;
    const uint32_t stg_u32 = smem_u32(stg);
    uint32_t cnt = 0;      // hits so far (may exceed seg: the selection then falls back)
    uint32_t written = 0;  // pairs moved to global memory (multiple of 4 until the tail)
    uint32_t pend = 0;     // pairs waiting in the staging slots 0 .. pend-1

    // write every complete group of 4 pending pairs (whole 32-byte sectors) and move the
    // rest (< 4) to the front of the staging area.  At most 3 + 8 pairs are pending, so at
    // most two groups.  Only the lanes with a group to write read their staging area (a
    // lane's hits fill a group every few calls), so the shared-memory loads scale with the
    // sectors written rather than with the calls.
    auto flush = [&]() {
      const uint32_t groups = pend >> 2;
      if (!__any_sync(0xFFFFFFFFu, groups > 0)) return;
      if (groups > 0) {
        float4* d4 = reinterpret_cast<float4*>(dst + written);
        const float4 x0 = *reinterpret_cast<const float4*>(stg);
        const float4 x1 = *reinterpret_cast<const float4*>(stg + 16);
        if (written + 4 <= (uint32_t)seg) {
          d4[0] = x0;
          d4[1] = x1;
        }
        if (groups > 1) {
          const float4 y0 = *reinterpret_cast<const float4*>(stg + 32);
          const float4 y1 = *reinterpret_cast<const float4*>(stg + 48);
          if (written + 8 <= (uint32_t)seg) {
            d4[2] = y0;
            d4[3] = y1;
          }
        }
        const uint32_t rest = pend & 3u;
        const uint8_t* src = stg + groups * 32;
        if (rest > 0) {
          const float2 r0 = *reinterpret_cast<const float2*>(src);
          const float2 r1 = *reinterpret_cast<const float2*>(src + 8);
          const float2 r2 = *reinterpret_cast<const float2*>(src + 16);
          *reinterpret_cast<float2*>(stg) = r0;
          if (rest > 1) *reinterpret_cast<float2*>(stg + 8) = r1;
          if (rest > 2) *reinterpret_cast<float2*>(stg + 16) = r2;
        }
        written += groups * 4;
        pend = rest;
      }
    };

    int i = 0;
    bool ok = true;
    for (int b = b_first; b <= b_last && ok; ++b) {
      int64_t rs, re, pbase;
      int kh;
      if (!seq_range(b, rs, re, kh, pbase)) continue;
      const bool in_seq = row >= rs && row < re;
      const float thr = in_seq ? thr_row : INFINITY;  // rows of other sequences keep nothing
      const int prow = in_seq ? (int)(pbase + row) : -1;
      // the warp's rows are all in this sequence and its first row sees every key of a
      // chunk that ends at or below p_min: such chunks need no causal compare
      const int p_min = (int)(pbase + r0 + quad * 32);
      const bool warp_in_seq = r0 + quad * 32 >= rs && r0 + quad * 32 + 31 < re;
      for (int kt = 0; kt < kh; ++kt, ++i) {
        float acc[kCandCols];
        bool waited = true;
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {
          if (pr >= n_pairs) break;
          if (!mbar_wait_bounded(smem_u32(&tfull[pr]), i & 1, a.status, &s_abort)) {
            waited = false;
            break;
          }
          tc_fence_after();
          const uint32_t tbase = tmem + lane_base + (uint32_t)(pr * kCandSlotCols + sub * kCandCols);
          // one head and 16 key columns per TMEM wait: the 96 registers a thread has at 18
          // warps per SM hold the 32 partial sums, one load and the emission state (two
          // heads per wait spill)
#pragma unroll
          for (int c0 = 0; c0 < kCandCols; c0 += 16) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int h = 2 * pr + q;
              if (h >= H) break;
              uint32_t v[16];
              tmem_ld16_async(tbase + (uint32_t)(q * kCandKT + c0), v);
              tmem_wait_ld();
              reg_fence(v);
              if (!row_w) {
                const float2 w2 = make_float2(wsh[h], wsh[h]);
#pragma unroll
                for (int c = 0; c < 16; c += 2) {
                  const float2 x = make_float2(fmaxf(__uint_as_float(v[c]), 0.f),
                                               fmaxf(__uint_as_float(v[c + 1]), 0.f));
                  const float2 prev =
                      h == 0 ? make_float2(0.f, 0.f) : make_float2(acc[c0 + c], acc[c0 + c + 1]);
                  const float2 r2 = __ffma2_rn(w2, x, prev);
                  acc[c0 + c] = r2.x;
                  acc[c0 + c + 1] = r2.y;
                }
              } else {
#pragma unroll
                for (int c = 0; c < 16; ++c)
                  acc[c0 + c] = fmaf(wsh[h], fmaxf(__uint_as_float(v[c]) * a.scale, 0.f),
                                     h == 0 ? 0.f : acc[c0 + c]);
              }
            }
          }
          // the pair is in registers: hand its TMEM slot back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&tempty[pr]));
        }
        if (!waited) {
          ok = false;
          break;
        }

        const int j0 = kt * kCandKT + sub * kCandCols;  // position of key column 0
        const bool interior = __all_sync(0xFFFFFFFFu, warp_in_seq && j0 + kCandCols - 1 <= p_min);
        const int lim = prow - j0;                      // keys k <= lim are visible to this row
#pragma unroll
        for (int grp = 0; grp < kCandCols / 8; ++grp) {
          // straight-line predicated appends (no branch per key): compare, then the store
          // and the slot advance under the same predicate
          uint32_t sp = stg_u32 + pend * 8;
          if (interior) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const int k = grp * 8 + c;
              asm volatile(
                  "{\n\t.reg .pred p;\n\t"
                  "setp.ge.f32 p, %1, %2;\n\t"
                  "@p st.shared.v2.b32 [%0], {%3, %4};\n\t"
                  "@p add.u32 %0, %0, 8;\n\t}"
                  : "+r"(sp)
                  : "f"(acc[k]), "f"(thr), "r"(j0 + k), "r"(__float_as_uint(acc[k]))
                  : "memory");
            }
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const int k = grp * 8 + c;
              asm volatile(
                  "{\n\t.reg .pred p;\n\t"
                  "setp.ge.f32 p, %1, %2;\n\t"
                  "setp.le.and.s32 p, %5, %6, p;\n\t"
                  "@p st.shared.v2.b32 [%0], {%3, %4};\n\t"
                  "@p add.u32 %0, %0, 8;\n\t}"
                  : "+r"(sp)
                  : "f"(acc[k]), "f"(thr), "r"(j0 + k), "r"(__float_as_uint(acc[k])), "r"(k),
                    "r"(lim)
                  : "memory");
            }
          }
          const uint32_t now = (sp - stg_u32) >> 3;
          cnt += now - pend;
          pend = now;
          flush();
        }
      }
    }
    // tail: the last (< 4) pending pairs, one by one
    if (in_launch) {
#pragma unroll
      for (uint32_t t = 0; t < 3; ++t)
        if (t < pend && written + t < (uint32_t)seg)
          dst[written + t] = *reinterpret_cast<const float2*>(stg + t * 8);
      a.cand_cnt[(row - a.q_begin) * 4 + sub] = (int32_t)cnt;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, (uint32_t)kCols);
  }
}

// Launch order of the candidate pass for a batch of several sequences: the query tiles sorted
// by their number of key tiles (the CTA's work), longest first, ties by tile index, so that the
// CTAs of the longest histories start first and the shorter ones fill in (list scheduling in
// decreasing order).  One CTA of kCandOrderThreads; n_tiles <= kCandOrderMax (else the launch
// keeps the default order).  Bitonic sort of (work, tile) keys in shared memory.
constexpr int kCandOrderThreads = 1024;
constexpr int kCandOrderMax = 4096;
__global__ void __launch_bounds__(kCandOrderThreads) idx_cand_order_kernel(IdxArgs a, int32_t* order) {
  __shared__ uint64_t key[kCandOrderMax];
  const int n = a.n_tiles;
  int m = 1;
  while (m < n) m <<= 1;
  const int64_t q_end = a.q_begin + a.q_count;
  for (int t = threadIdx.x; t < m; t += kCandOrderThreads) {
    uint64_t k = ~0ull;  // padding sorts last
    if (t < n) {
      const int64_t r0 = a.q_begin + (int64_t)t * kCandBQ;
      const int64_t r_last = (r0 + kCandBQ < q_end ? r0 + kCandBQ : q_end) - 1;
      const int b_first = seq_of_row(a.q_offsets, a.batch, r0);
      const int b_last = seq_of_row(a.q_offsets, a.batch, r_last);
      uint32_t work = 0;
      for (int b = b_first; b <= b_last; ++b) {
        const int64_t qo = __ldg(a.q_offsets + b), qn = __ldg(a.q_offsets + b + 1);
        const int64_t ko = __ldg(a.kv_offsets + b), kn = __ldg(a.kv_offsets + b + 1);
        const int64_t rs = r0 > qo ? r0 : qo;
        const int64_t re = (r_last + 1) < qn ? (r_last + 1) : qn;
        const int64_t pmax = (kn - ko) - (qn - qo) - qo + re - 1;
        if (rs < re && pmax >= 0) work += (uint32_t)(pmax / kCandKT) + 1;
      }
      // descending work, then ascending tile: sort ascending on (~work, tile)
      k = ((uint64_t)(~work) << 32) | (uint32_t)t;
    }
    key[t] = k;
  }
  __syncthreads();
  for (int size = 2; size <= m; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < m; t += kCandOrderThreads) {
        const int u = t ^ stride;
        if (u > t) {
          const bool up = (t & size) == 0;
          const uint64_t x = key[t], y = key[u];
          if ((x > y) == up) {
            key[t] = y;
            key[u] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int t = threadIdx.x; t < n; t += kCandOrderThreads) order[t] = (int32_t)(key[t] & 0xFFFFFFFFu);
}

}  // namespace dsa
