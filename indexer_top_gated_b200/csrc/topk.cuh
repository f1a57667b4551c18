// topk.cuh - step 2 of the layer: per-row Top-K selection by radix select.
//
// For a score row s[0..n) (n = p+1 causal candidates) and K < n, every fp32 score becomes
// an order-preserving 32-bit key (-0.0 folded onto +0.0).
//
// Fast path (almost every row):
//  - 1024 samples (64 evenly spaced runs of 16 consecutive scores) give an estimate t of
//    the K-th largest key: the sample of rank S*K/n plus a margin of 4 sigma + 8, found to
//    22 bits by a radix select over the samples (12 + 10 bits), so that with overwhelming
//    probability at least K keys of the row are >= t;
//  - one ordered pass keeps every key >= t, with its position, as a candidate in shared
//    memory (each warp owns a contiguous run of positions; packed warp scans and one
//    block scan per run of 16384 positions give the slots, so candidates stay in
//    position order);
//  - an exact radix select (12 + 10 + 10 bits) over the candidates alone finds the
//    threshold key tau and how many keys equal to tau are still needed; an ordered pass
//    over the candidates writes the selected positions in ascending order, ties going to
//    the lower position.
// Exact path (if the estimate was off: fewer than K candidates, or more than fit): the
//  same radix select over the whole row (histogram of the top 12 bits, the threshold
//  bin's keys refined by two 10-bit digits), then one ordered pass over the whole row.
// Bins are picked by a single warp (two-level warp scan), every histogram is zeroed once
// up front and block scans cost one barrier, so a row needs few block-wide barriers; two
// CTAs share an SM.  No sort and no global scratch.
//
// Fused indexer -> Top-K (no score matrix): the indexer first scores every 16th key
// (samples), topk_thr_kernel turns each row's samples into a threshold estimate t, the
// candidate indexer pass keeps only the (position, score) pairs with score >= t, and
// topk_fused_kernel selects among them: when the row has between K and `cap` candidates
// they contain every score >= t, hence the whole Top-K with all of its ties, and the
// selection is exact.  The candidates arrive in no particular order, which one radix
// level (12 bits of the keys, spread over the candidates' range -- for a sampled row the
// range the threshold kernel found) does not need; the few candidates in the threshold bin
// are then ranked exactly (score descending, position ascending), the selected positions
// are marked in a bitmap over the row, and one ordered scan lists them in shared memory,
// from where the ascending index row leaves in coalesced stores.  A row whose estimate missed (fewer than
// K candidates, or more than its slots) or whose threshold bin is too crowded goes to a
// list that topk_kernel<kTopkFallback> works through: it recomputes the row's scores on
// CUDA cores into a scratch row and runs the full selection on it.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkBatch = 8;                      // row loads kept in flight per thread
constexpr int kTopkRun = 4 * kTopkThreads * kTopkBatch;  // positions per batched pass step
constexpr int kTopkFastCap = 8192;                 // fast-path candidates (key + position)
constexpr int kTopkExactCap = 2 * kTopkFastCap;    // exact-path candidates (keys only)
// shared memory (32-bit words): six histograms (4096 + 1024 + 1024, twice), then the
// candidate area
constexpr int kTopkHistWords = 2 * (4096 + 1024 + 1024);
constexpr int kTopkSmemWords = kTopkHistWords + 2 * kTopkFastCap;

__host__ inline size_t topk_smem_bytes(int64_t /*max_kv_len*/) {
  return (size_t)kTopkSmemWords * sizeof(uint32_t);
}

// Fused selection: shared memory of one CTA = a 4096-bin histogram (which later holds the
// listing of the index row, K <= 4096), a position bitmap of ceil(max_n / 32) words (rounded
// up to a multiple of 4) and the threshold bin's keys and positions (kTopkBinMax each).
constexpr int kTopkFusedMaxN = 314496;
constexpr int kTopkCandBatch = 8;    // candidate loads in flight per thread
constexpr int kTopkBinMax = 512;     // threshold-bin candidates ranked directly
__host__ __device__ inline int topk_fused_bm_words(int64_t max_n) {
  return (int)(((max_n + 31) / 32 + 3) / 4 * 4);
}
// The fused selection runs 256-thread CTAs (up to six per SM): it re-reads a row's candidates
// from L2 in each of its passes instead of staging them, so a CTA's shared memory is the
// histogram, the position bitmap and the threshold bin only.
constexpr int kFusedThreads = 256;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kFusedCtasPerSm = 6;
__host__ inline size_t topk_fused_smem_bytes(int /*cap*/, int64_t max_n) {
  return (size_t)(4096 + topk_fused_bm_words(max_n) + 2 * kTopkBinMax) * 4;
}

enum TopkMode { kTopkScores = 0, kTopkFallback = 2 };

struct TopkArgs {
  const int32_t* q_offsets;
  const int32_t* kv_offsets;
  int batch;
  int64_t q_begin;
  int64_t q_count;
  int K;
  const float* scores;
  int64_t ld;
  int32_t* idx;
  int64_t ld_idx;
  int32_t* cnt;
  // fused selection: candidate lists of the candidate indexer pass
  const float2* cand;       // [q_count, cap]: 4 segments of cap/4 (position bits, score)
  int cap;
  const int32_t* cand_cnt;  // [q_count, 4] per segment
  const float* thr;         // [q_count] the candidates' threshold (every candidate >= it)
  const uint32_t* khi;      // [q_count] largest sample key of the row, 0 if not sampled
  int32_t* fb_list;         // [1 + q_count]: count, then rows (within the launch) to redo
  int blk_shift;            // rows of block scores: n = (p >> blk_shift) + 1 entries
  int prefetch_ahead;       // fused selection: warm L2 with the candidates of the row this
                            // many rows later in launch order (about one wave of CTAs)
  int bm_words;             // words of each position bitmap (topk_fused_bm_words)
  // fallback: recompute a row's scores on CUDA cores (same formula as the indexer)
  const void* q_idx;
  const void* k_idx;
  int idx_heads;
  int idx_fp8;
  const float* w;
  int w_row_stride;
  float idx_scale;
  float* fb_scores;         // [gridDim.x, ld_fb]
  int64_t ld_fb;
  CachePages pages;         // paged k_idx
};

// Threshold estimate from sampled scores (fused path).
struct TopkThrArgs {
  const int32_t* q_offsets;
  const int32_t* kv_offsets;
  int batch;
  int64_t q_begin;
  int64_t q_count;
  int K;
  int cap;
  int shift;          // sample m of a row is the score of position m << shift
  const uint16_t* samp;  // [q_count, ld_s] bf16 samples, rounded toward -infinity
  int64_t ld_s;
  int stage;          // samples a warp stages in shared memory (a multiple of 8)
  int long_rows;      // non-zero: rows of more than `stage` samples are left to
                      // topk_thr_long_kernel
  float* thr;         // [q_count]
  uint32_t* khi;      // [q_count] largest sample key (0: the row was not sampled)
  int32_t* fb_list;   // its count is reset here
};

DSA_DEV uint32_t topk_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0.0 == +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inverse of topk_key: the float whose key is k (finite for every key of a finite score
// with low bits cleared, since such keys stay >= key(-FLT_MAX)).
DSA_DEV float topk_key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

DSA_DEV uint32_t warp_incl_scan(uint32_t x) {
  const int lane = lane_id();
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// Block-wide exclusive scan of one value per thread with a single barrier.  `tot` holds
// two banks of per-warp totals used alternately (`bank` flips on every call), so a bank
// is rewritten only after every thread has passed the next call's barrier.
template <int NW>
DSA_DEV uint32_t block_scan_w(uint32_t v, uint32_t* tot, int& bank, uint32_t& total) {
  const int lane = lane_id(), warp = threadIdx.x >> 5;
  const uint32_t x = warp_incl_scan(v);
  uint32_t* t = tot + bank * 32;
  if (lane == 31) t[warp] = x;
  __syncthreads();
  const uint32_t wt = lane < NW ? t[lane] : 0u;
  const uint32_t wi = warp_incl_scan(wt);
  total = __shfl_sync(0xFFFFFFFFu, wi, 31);
  const uint32_t wbase = __shfl_sync(0xFFFFFFFFu, wi - wt, warp);
  bank ^= 1;
  return wbase + x - v;
}

DSA_DEV uint32_t block_scan(uint32_t v, uint32_t* tot, int& bank, uint32_t& total) {
  const int lane = lane_id(), warp = threadIdx.x >> 5;
  const uint32_t x = warp_incl_scan(v);
  uint32_t* t = tot + bank * 32;
  if (lane == 31) t[warp] = x;
  __syncthreads();
  const uint32_t wt = lane < kTopkWarps ? t[lane] : 0u;
  const uint32_t wi = warp_incl_scan(wt);
  total = __shfl_sync(0xFFFFFFFFu, wi, 31);
  const uint32_t wbase = __shfl_sync(0xFFFFFFFFu, wi - wt, warp);
  bank ^= 1;
  return wbase + x - v;
}

// Warp-level bin pick over hist[0 .. NB), scanned from the top bin down: the bin in which
// the count of larger keys first reaches `remaining`.  Writes s_sel = {bin, still needed
// from that bin, bin kept whole}.  Called by one full warp.
template <int NB>
DSA_DEV void warp_select(const uint32_t* hist, uint32_t remaining, uint32_t* s_sel) {
  constexpr int PER = NB / 32;   // bins per lane in the first level
  constexpr int SUB = PER / 32;  // bins per lane in the second level
  const int lane = lane_id();
  // level 1: lane l owns the l-th block of PER bins counted from the top.  The blocks
  // are PER words apart (the same banks), so each lane walks its block in a rotated
  // order: at step q lane l reads quad (q + l) mod (PER / 4), and a warp's 16-byte reads
  // spread over all banks.
  const int hi1 = NB - 1 - lane * PER;
  uint32_t sum = 0;
#pragma unroll
  for (int q = 0; q < PER / 4; ++q) {
    const int qq = (q + lane) & (PER / 4 - 1);
    const uint4 u = *reinterpret_cast<const uint4*>(hist + hi1 - PER + 1 + 4 * qq);
    sum += u.x + u.y + u.z + u.w;
  }
  uint32_t incl = warp_incl_scan(sum);
  const unsigned own1 = __ballot_sync(0xFFFFFFFFu, incl - sum < remaining && remaining <= incl);
  const int o1 = __ffs(own1) - 1;
  const uint32_t above1 = __shfl_sync(0xFFFFFFFFu, incl - sum, o1);
  // level 2: lane l owns SUB bins of block o1, again from the top
  const int hi2 = NB - 1 - o1 * PER - lane * SUB;
  uint32_t c[SUB > 0 ? SUB : 1];
  uint32_t sum2 = 0;
#pragma unroll
  for (int q = 0; q < SUB; ++q) {
    c[q] = hist[hi2 - q];
    sum2 += c[q];
  }
  incl = warp_incl_scan(sum2) + above1;
  const uint32_t excl2 = incl - sum2;
  if (excl2 < remaining && remaining <= incl) {
    uint32_t above = excl2;
#pragma unroll
    for (int q = 0; q < SUB; ++q) {
      if (above < remaining && remaining <= above + c[q]) {
        s_sel[0] = (uint32_t)(hi2 - q);
        s_sel[1] = remaining - above;
        s_sel[2] = (remaining - above == c[q]) ? 1u : 0u;
      }
      above += c[q];
    }
  }
}

// Shared state of a Top-K CTA besides the dynamic area.
struct TopkShared {
  uint32_t tot[64];
  uint32_t sel[3];
  uint32_t ncand;
  uint32_t kmin, kmax;
};

// Radix select over `count` keys get(c) (strided over the block) with the zeroed histograms
// h12 / h10a / h10b: finds the key threshold *tau of the want-th largest key and returns
// how many keys equal to it are still needed (0 when the threshold bin is kept whole,
// *whole = true, and every key >= *tau belongs to the selection).
template <class Get>
DSA_DEV uint32_t topk_select(uint32_t* h12, uint32_t* h10a, uint32_t* h10b, uint32_t want,
                             Get&& get, uint32_t count, int levels, TopkShared& sh,
                             uint32_t* tau, bool* whole) {
  const int tid = threadIdx.x, warp = tid >> 5;
  for (uint32_t c = tid; c < count; c += kTopkThreads) atomicAdd(&h12[get(c) >> 20], 1u);
  __syncthreads();
  if (warp == 0) warp_select<4096>(h12, want, sh.sel);
  __syncthreads();
  uint32_t t = sh.sel[0] << 20, need = sh.sel[1];
  bool w = sh.sel[2] != 0;
  if (!w) {
    for (uint32_t c = tid; c < count; c += kTopkThreads) {
      const uint32_t key = get(c);
      if ((key & 0xFFF00000u) == t) atomicAdd(&h10a[(key >> 10) & 1023u], 1u);
    }
    __syncthreads();
    if (warp == 0) warp_select<1024>(h10a, need, sh.sel);
    __syncthreads();
    t |= sh.sel[0] << 10;
    need = sh.sel[1];
    w = sh.sel[2] != 0;
    if (!w && levels > 2) {
      for (uint32_t c = tid; c < count; c += kTopkThreads) {
        const uint32_t key = get(c);
        if ((key & 0xFFFFFC00u) == t) atomicAdd(&h10b[key & 1023u], 1u);
      }
      __syncthreads();
      if (warp == 0) warp_select<1024>(h10b, need, sh.sel);
      __syncthreads();
      t |= sh.sel[0];
      need = sh.sel[1];
      w = sh.sel[2] != 0;
    }
  }
  *tau = t;
  *whole = w;
  return w ? 0u : need;
}

// Ordered output over C candidates fk / fp held in position order: the keys above tau (or
// >= tau when ge) and the first ties_needed keys equal to tau, ascending by position.
DSA_DEV void topk_emit_candidates(const uint32_t* fk, const uint32_t* fp, uint32_t C,
                                  uint32_t tau, bool ge, uint32_t ties_needed, int32_t* out,
                                  TopkShared& sh, int& bank) {
  const int tid = threadIdx.x;
  uint32_t run_def = 0, run_tie = 0;
  for (uint32_t base = 0; base < C; base += 4 * kTopkThreads) {
    const uint32_t c0 = base + 4 * tid;
    uint32_t dflag = 0, tflag = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const bool valid = c0 + q < C;
      const uint32_t key = valid ? fk[c0 + q] : 0u;
      dflag |= (uint32_t)(valid && (ge ? key >= tau : key > tau)) << q;
      tflag |= (uint32_t)(valid && !ge && key == tau) << q;
    }
    const uint32_t packed = (uint32_t)__popc(dflag) | ((uint32_t)__popc(tflag) << 16);
    uint32_t total;
    const uint32_t before = block_scan(packed, sh.tot, bank, total);
    uint32_t d_before = run_def + (before & 0xFFFFu);
    uint32_t t_before = run_tie + (before >> 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if ((dflag >> q) & 1u) {
        out[d_before + (t_before < ties_needed ? t_before : ties_needed)] = (int32_t)fp[c0 + q];
        ++d_before;
      } else if ((tflag >> q) & 1u) {
        if (t_before < ties_needed) out[d_before + t_before] = (int32_t)fp[c0 + q];
        ++t_before;
      }
    }
    run_def += total & 0xFFFFu;
    run_tie += total >> 16;
  }
}

template <bool NC>
DSA_DEV float4 topk_ld4(const float* p) {
  if (NC) return __ldg(reinterpret_cast<const float4*>(p));
  return *reinterpret_cast<const float4*>(p);
}
template <bool NC>
DSA_DEV float topk_ld1(const float* p) {
  if (NC) return __ldg(p);
  return *p;
}

// Top-K of one materialised score row row[0 .. nn), nn > K, into out[0 .. K).  NC: the row
// was written by an earlier launch (read through the non-coherent cache); otherwise this
// CTA wrote it, and it is read with coherent loads.  PIPE: the candidate pass loads the
// next run of the row while it compacts the current one (twice the registers for the
// loads: for a CTA that has its SM alone).
template <bool NC, bool PIPE = false>
DSA_DEV void topk_scores_row(const TopkArgs& a, int nn, const float* row, int32_t* out,
                             uint32_t* dyn, TopkShared& sh) {
  uint32_t* hA = dyn;            // 4096: sample, top 12 bits
  uint32_t* hB = hA + 4096;      // 1024: sample, next 10 bits
  uint32_t* hC = hB + 1024;      // 1024: sample, last 10 bits
  uint32_t* hD = hC + 1024;      // 4096: candidates / row, top 12 bits
  uint32_t* hE = hD + 4096;      // 1024
  uint32_t* hF = hE + 1024;      // 1024
  uint32_t* cand = dyn + kTopkHistWords;
  uint32_t* fk = cand;                 // fast path: candidate keys      [kTopkFastCap]
  uint32_t* fp = cand + kTopkFastCap;  // fast path: candidate positions [kTopkFastCap]
  const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;
  const int K = a.K;
  int bank = 0;
  {
    // pull the whole row towards L2 now, so that its DRAM latency overlaps the threshold
    // estimate below and the candidate pass reads from L2 (the row is 16-byte aligned and
    // its padded length round4(n) fits its allocation)
    const int64_t bytes = (((int64_t)nn + 3) & ~int64_t(3)) * 4;
    constexpr int64_t kPiece = 16384;
    for (int64_t off = (int64_t)tid * kPiece; off < bytes; off += (int64_t)kTopkThreads * kPiece)
      bulk_prefetch_l2(reinterpret_cast<const char*>(row) + off,
                       (uint32_t)(bytes - off < kPiece ? bytes - off : kPiece));
  }
  // four consecutive keys starting at j0 (a multiple of 4; 0 past the end)
  auto load4 = [&](int j0, uint32_t (&k4)[4]) {
    if (j0 + 3 < nn) {
      const float4 f = topk_ld4<NC>(row + j0);
      k4[0] = topk_key(f.x);
      k4[1] = topk_key(f.y);
      k4[2] = topk_key(f.z);
      k4[3] = topk_key(f.w);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) k4[q] = j0 + q < nn ? topk_key(topk_ld1<NC>(row + j0 + q)) : 0u;
    }
  };

  // ---- zero every histogram once
  for (int t = tid; t < kTopkHistWords; t += kTopkThreads) dyn[t] = 0;
  if (tid == 0) sh.ncand = 0;
  __syncthreads();

  // ================================================================ fast path
  {
    const int S = nn < 1024 ? nn : 1024;
    const float m_exp = (float)S * (float)K / (float)nn;
    int m = (int)ceilf(m_exp + 4.f * sqrtf(m_exp) + 8.f);
    if (m > S) m = S;
    // samples: 64 evenly spaced runs of 16 consecutive scores (one float4 per thread for
    // 256 threads), or the whole row when it is shorter than 1024; kept in the candidate
    // area, which the candidate pass overwrites only afterwards
    if (nn >= 1024) {
      if (tid < 256) {
        const int blk = tid >> 2;
        const int start = (int)(((int64_t)blk * (nn - 16)) / 63) & ~3;
        uint32_t k4[4];
        load4(start + 4 * (tid & 3), k4);
        *reinterpret_cast<uint4*>(fk + 4 * tid) = make_uint4(k4[0], k4[1], k4[2], k4[3]);
      }
    } else {
      for (int j = tid; j < nn; j += kTopkThreads) fk[j] = topk_key(topk_ld1<NC>(row + j));
    }
    __syncthreads();
    uint32_t t_est;
    bool sw;
    // 22 bits of the estimate are plenty: every sample >= t_est counts towards m
    topk_select(hA, hB, hC, (uint32_t)m, [&](uint32_t c) { return fk[c]; }, (uint32_t)S, 2, sh,
                &t_est, &sw);
    __syncthreads();  // samples read; the candidate pass may overwrite them

    // -- candidates: every key >= t_est, in position order.  The comparison is done on the
    // raw scores (key order = float order, -0.0 == +0.0); keys are formed only for the
    // candidates.
    const float t_val = topk_key_value(t_est);
    uint32_t run = 0;
    bool overflow = false;
    // one run of kTopkRun positions: warp w owns positions cb + 1024 w .. + 1023
    auto load_run = [&](int cb, float4 (&xr)[kTopkBatch]) {
#pragma unroll
      for (int it = 0; it < kTopkBatch; ++it) {
        const int j0 = cb + warp * 1024 + it * 128 + lane * 4;
        if (j0 + 3 < nn) {
          xr[it] = topk_ld4<NC>(row + j0);
        } else {
          xr[it].x = j0 < nn ? topk_ld1<NC>(row + j0) : -INFINITY;
          xr[it].y = j0 + 1 < nn ? topk_ld1<NC>(row + j0 + 1) : -INFINITY;
          xr[it].z = j0 + 2 < nn ? topk_ld1<NC>(row + j0 + 2) : -INFINITY;
          xr[it].w = j0 + 3 < nn ? topk_ld1<NC>(row + j0 + 3) : -INFINITY;
        }
      }
    };
    float4 xb[kTopkBatch], xn[kTopkBatch];
    if (PIPE) load_run(0, xn);
    for (int cb = 0; cb < nn && !overflow; cb += kTopkRun) {
      if (PIPE) {
#pragma unroll
        for (int it = 0; it < kTopkBatch; ++it) xb[it] = xn[it];
        if (cb + kTopkRun < nn) load_run(cb + kTopkRun, xn);
      } else {
        load_run(cb, xb);
      }
      uint32_t fl = 0;                  // bit 4*it + q: score q of step it is kept
      uint32_t cnt_lo = 0, cnt_hi = 0;  // per-step counts packed in bytes
#pragma unroll
      for (int it = 0; it < kTopkBatch; ++it) {
        const uint32_t f = (uint32_t)(xb[it].x >= t_val) | ((uint32_t)(xb[it].y >= t_val) << 1) |
                           ((uint32_t)(xb[it].z >= t_val) << 2) | ((uint32_t)(xb[it].w >= t_val) << 3);
        fl |= f << (4 * it);
        if (it < 4) cnt_lo |= (uint32_t)__popc(f) << (8 * it);
        else cnt_hi |= (uint32_t)__popc(f) << (8 * (it - 4));
      }
      const uint32_t inc_lo = warp_incl_scan(cnt_lo), inc_hi = warp_incl_scan(cnt_hi);
      const uint32_t exc_lo = inc_lo - cnt_lo, exc_hi = inc_hi - cnt_hi;
      const uint32_t tot_lo = __shfl_sync(0xFFFFFFFFu, inc_lo, 31);
      const uint32_t tot_hi = __shfl_sync(0xFFFFFFFFu, inc_hi, 31);
      uint32_t wtot = 0;
#pragma unroll
      for (int it = 0; it < 4; ++it)
        wtot += ((tot_lo >> (8 * it)) & 255u) + ((tot_hi >> (8 * it)) & 255u);
      uint32_t chunk_total;
      const uint32_t wb = block_scan(lane == 31 ? wtot : 0u, sh.tot, bank, chunk_total);
      // only lane 31 contributed, so lane 0's exclusive prefix is the count before warp w
      const uint32_t warp_base = __shfl_sync(0xFFFFFFFFu, wb, 0);
      if (run + chunk_total > (uint32_t)kTopkFastCap) {
        overflow = true;  // uniform: chunk_total is the block total
        break;
      }
      uint32_t pre = run + warp_base;  // candidates before step `it` of this warp
#pragma unroll
      for (int it = 0; it < kTopkBatch; ++it) {
        const uint32_t lo = it < 4 ? (exc_lo >> (8 * it)) & 255u : (exc_hi >> (8 * (it - 4))) & 255u;
        const uint32_t tt = it < 4 ? (tot_lo >> (8 * it)) & 255u : (tot_hi >> (8 * (it - 4))) & 255u;
        uint32_t nib = (fl >> (4 * it)) & 15u;
        if (nib) {
          uint32_t slot = pre + lo;
          const int j0 = cb + warp * 1024 + it * 128 + lane * 4;
          while (nib) {
            const int q = __ffs(nib) - 1;
            nib &= nib - 1;
            const float x = q == 0 ? xb[it].x : q == 1 ? xb[it].y : q == 2 ? xb[it].z : xb[it].w;
            fk[slot] = topk_key(x);
            fp[slot] = (uint32_t)(j0 + q);
            ++slot;
          }
        }
        pre += tt;
      }
      run += chunk_total;
    }
    __syncthreads();
    if (!overflow && run >= (uint32_t)K) {
      // -- exact selection among the candidates, then ordered output over them (they are
      // in position order)
      uint32_t tau;
      bool ge;
      const uint32_t ties_needed =
          topk_select(hD, hE, hF, (uint32_t)K, [&](uint32_t c) { return fk[c]; }, run, 3, sh,
                      &tau, &ge);
      topk_emit_candidates(fk, fp, run, tau, ge, ties_needed, out, sh, bank);
      return;  // uniform
    }
  }

  // ================================================================ exact path
  // (the fast path used hA..hC and maybe fk/fp; hD..hF are still zero)
  uint32_t* ck = cand;  // candidate keys of the threshold bin [kTopkExactCap]
  // pass A: histogram of the top 12 bits of the whole row
  for (int cb = 0; cb < nn; cb += kTopkRun) {
    uint32_t kb[kTopkBatch][4];
#pragma unroll
    for (int it = 0; it < kTopkBatch; ++it) load4(cb + it * 4 * kTopkThreads + 4 * tid, kb[it]);
#pragma unroll
    for (int it = 0; it < kTopkBatch; ++it) {
      const int j0 = cb + it * 4 * kTopkThreads + 4 * tid;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (j0 + q < nn) atomicAdd(&hD[kb[it][q] >> 20], 1u);
    }
  }
  __syncthreads();
  if (warp == 0) warp_select<4096>(hD, (uint32_t)K, sh.sel);
  __syncthreads();
  const uint32_t b12 = sh.sel[0];
  uint32_t remaining = sh.sel[1];
  uint32_t prefix = b12 << 20;
  bool ge_mode = sh.sel[2] != 0;
  if (!ge_mode) {
    const uint32_t n_bin = hD[b12];
    const bool use_cand = n_bin <= (uint32_t)kTopkExactCap;
    if (use_cand) {
      // the threshold bin's keys (order is irrelevant for the threshold)
      for (int cb = 0; cb < nn; cb += kTopkRun) {
        uint32_t kb[kTopkBatch][4];
#pragma unroll
        for (int it = 0; it < kTopkBatch; ++it) load4(cb + it * 4 * kTopkThreads + 4 * tid, kb[it]);
#pragma unroll
        for (int it = 0; it < kTopkBatch; ++it) {
          const int j0 = cb + it * 4 * kTopkThreads + 4 * tid;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const bool mm = (j0 + q < nn) && ((kb[it][q] >> 20) == b12);
            const unsigned bal = __ballot_sync(0xFFFFFFFFu, mm);
            if (bal) {
              uint32_t slot = 0;
              if (lane == 0) slot = atomicAdd(&sh.ncand, (uint32_t)__popc(bal));
              slot = __shfl_sync(0xFFFFFFFFu, slot, 0);
              if (mm) ck[slot + __popc(bal & ((1u << lane) - 1u))] = kb[it][q];
            }
          }
        }
      }
      __syncthreads();
    }
    for (int level = 0; level < 2 && !ge_mode; ++level) {
      uint32_t* h = level == 0 ? hE : hF;
      const int shift = level == 0 ? 10 : 0;
      const uint32_t want_mask = level == 0 ? 0xFFF00000u : 0xFFFFFC00u;
      if (use_cand) {
        for (uint32_t c = tid; c < n_bin; c += kTopkThreads) {
          const uint32_t key = ck[c];
          if ((key & want_mask) == prefix) atomicAdd(&h[(key >> shift) & 1023u], 1u);
        }
      } else {
        for (int cb = 0; cb < nn; cb += kTopkRun) {
          uint32_t kb[kTopkBatch][4];
#pragma unroll
          for (int it = 0; it < kTopkBatch; ++it) load4(cb + it * 4 * kTopkThreads + 4 * tid, kb[it]);
#pragma unroll
          for (int it = 0; it < kTopkBatch; ++it) {
            const int j0 = cb + it * 4 * kTopkThreads + 4 * tid;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (j0 + q < nn && (kb[it][q] & want_mask) == prefix)
                atomicAdd(&h[(kb[it][q] >> shift) & 1023u], 1u);
          }
        }
      }
      __syncthreads();
      if (warp == 0) warp_select<1024>(h, remaining, sh.sel);
      __syncthreads();
      prefix |= sh.sel[0] << shift;
      remaining = sh.sel[1];
      ge_mode = sh.sel[2] != 0;
    }
  }

  // Ordered output.  Definite: key > tau (or >= prefix in ge_mode).  Ties: key == tau,
  // the first `remaining` of them in position order are kept.
  const uint32_t tau = prefix;
  const uint32_t ties_needed = ge_mode ? 0u : remaining;
  uint32_t run_def = 0, run_tie = 0;
  for (int base = 0; base < nn; base += kTopkRun) {
    uint32_t kb[kTopkBatch][4];
#pragma unroll
    for (int it = 0; it < kTopkBatch; ++it) load4(base + it * 4 * kTopkThreads + 4 * tid, kb[it]);
#pragma unroll
    for (int it = 0; it < kTopkBatch; ++it) {
      if (base + it * 4 * kTopkThreads >= nn) continue;  // uniform across the block
      const int j0 = base + it * 4 * kTopkThreads + 4 * tid;
      uint32_t dflag = 0, tflag = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool valid = j0 + q < nn;
        dflag |= (uint32_t)(valid && (ge_mode ? kb[it][q] >= tau : kb[it][q] > tau)) << q;
        tflag |= (uint32_t)(valid && !ge_mode && kb[it][q] == tau) << q;
      }
      // packed counts: low 16 bits definite, high 16 bits ties (each <= 2048 per step)
      const uint32_t packed = (uint32_t)__popc(dflag) | ((uint32_t)__popc(tflag) << 16);
      uint32_t total;
      const uint32_t before = block_scan(packed, sh.tot, bank, total);
      uint32_t d_before = run_def + (before & 0xFFFFu);
      uint32_t t_before = run_tie + (before >> 16);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if ((dflag >> q) & 1u) {
          out[d_before + (t_before < ties_needed ? t_before : ties_needed)] = (int32_t)(j0 + q);
          ++d_before;
        } else if ((tflag >> q) & 1u) {
          if (t_before < ties_needed) out[d_before + t_before] = (int32_t)(j0 + q);
          ++t_before;
        }
      }
      run_def += total & 0xFFFFu;
      run_tie += total >> 16;
    }
  }
}

// Fused selection over the row's candidates: cnt[s] <= seg of them at the start of segment s
// (seg slots each) of cl, C = sum >= K in all, nn <= kTopkFusedMaxN.  Keys are mapped onto
// the full 32-bit range by the order-preserving (key - kmin) << clz(kmax - kmin), so that
// the 12-bit digit spreads although all candidates lie close together.  A sampled row brings
// its range: every candidate is >= the threshold, key k_lo, and about 16 of them exceed the
// largest sample, key k_hi; keys are clamped into [k_lo, k_hi] for the binning only (the top
// bin takes those few), and the threshold bin is ranked on the exact keys.  Other rows
// (k_hi = 0) take the range in a first pass.  Returns false (nothing written) when the
// threshold bin holds more than kTopkBinMax candidates.
// kFusedThreads threads: each quarter of the block reads one segment in every pass (the key
// range, the histogram, the marking), straight from global memory -- the first pass brings
// the row's candidates into L2, the later ones hit there.
DSA_DEV bool topk_candidates_row(const TopkArgs& a, int nn, const float2* cl, int seg,
                                 const uint32_t (&cnt)[4], uint32_t C, uint32_t k_lo,
                                 uint32_t k_hi, int32_t* out, uint32_t* dyn, TopkShared& sh) {
  constexpr int kQuarter = kFusedThreads / 4;
  uint32_t* h = dyn;                     // [4096]
  uint32_t* bm = h + 4096;               // [bm_words] selected positions
  uint32_t* bk = bm + a.bm_words;        // [kTopkBinMax] threshold-bin keys
  uint32_t* bp = bk + kTopkBinMax;       // [kTopkBinMax] threshold-bin positions
  const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;
  const int W = (nn + 31) >> 5;
  int bank = 0;
  const int sg = tid / kQuarter;
  const uint32_t ns = cnt[sg];
  const float2* src = cl + (int64_t)sg * seg;
  const uint32_t x0 = (uint32_t)(tid % kQuarter);
  constexpr uint32_t kStep = (uint32_t)kQuarter * kTopkCandBatch;
  // one pass over this thread's candidates (score, position), kTopkCandBatch loads in flight
  auto for_pairs = [&](auto&& f) {
    for (uint32_t e0 = x0; e0 < ns; e0 += kStep) {
      float2 e[kTopkCandBatch];
#pragma unroll
      for (int u = 0; u < kTopkCandBatch; ++u) {
        const uint32_t x = e0 + (uint32_t)kQuarter * u;
        e[u] = x < ns ? __ldg(src + x) : make_float2(0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kTopkCandBatch; ++u)
        if (e0 + (uint32_t)kQuarter * u < ns) f(e[u].y, (uint32_t)__float_as_int(e[u].x));
    }
  };
  auto for_cands = [&](auto&& f) {
    for_pairs([&](float x, uint32_t pos) { f(topk_key(x), pos); });
  };
  const bool ranged = k_hi != 0u && k_hi >= k_lo;  // uniform
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  if (!ranged)
    for_cands([&](uint32_t key, uint32_t) {
      lo = key < lo ? key : lo;
      hi = key > hi ? key : hi;
    });
  for (int t = tid; t < 1024; t += kFusedThreads)
    reinterpret_cast<uint4*>(h)[t] = make_uint4(0u, 0u, 0u, 0u);
  for (int t = tid; t < W; t += kFusedThreads) bm[t] = 0;
  if (tid == 0) {
    sh.kmin = ranged ? k_lo : 0xFFFFFFFFu;
    sh.kmax = ranged ? k_hi : 0u;
    sh.ncand = 0;
  }
  if (!ranged) {
    lo = __reduce_min_sync(0xFFFFFFFFu, lo);
    hi = __reduce_max_sync(0xFFFFFFFFu, hi);
    __syncthreads();  // kmin / kmax initialised
    if (lane == 0) {
      atomicMin(&sh.kmin, lo);
      atomicMax(&sh.kmax, hi);
    }
  }
  __syncthreads();  // range known, histogram and bitmap zeroed
  const uint32_t kmin = sh.kmin, kmax = sh.kmax, span = kmax - kmin;
  const int z = span ? __clz(span) : 0;
  // order-preserving map of a key onto the 32-bit range (clamped to [kmin, kmax])
  auto norm = [&](uint32_t key) -> uint32_t {
    key = key < kmin ? kmin : key;
    key = key > kmax ? kmax : key;
    return (key - kmin) << z;
  };
  for_cands([&](uint32_t key, uint32_t) { atomicAdd(&h[norm(key) >> 20], 1u); });
  __syncthreads();
  if (warp == 0) warp_select<4096>(h, (uint32_t)a.K, sh.sel);
  __syncthreads();
  const uint32_t b = sh.sel[0], need = sh.sel[1];
  const bool whole = sh.sel[2] != 0;
  const uint32_t n_bin = h[b];
  if (!whole && n_bin > (uint32_t)kTopkBinMax) return false;  // uniform
  // keys in higher bins (or the whole threshold bin) are selected; the threshold bin's
  // keys are set aside for ranking.  The bins are intervals of keys: a (clamped) key's bin
  // is >= bb iff the key is >= kmin + ceil(bb 2^20 / 2^z), so with the order-preserving key
  // map (-0.0 == +0.0) two float compares against the bounds of bins b and b + 1 classify a
  // candidate, and only the threshold bin's few candidates form their key.  Keys above kmax
  // share the bin of kmax (bin_top), keys below kmin (none but in a corrupted workspace) bin 0,
  // as in the histogram.  (Positions outside the row, which only a corrupted workspace can
  // hold, are skipped: they never index the bitmap.)
  auto first_key = [&](uint32_t bb) -> uint32_t {
    return (uint32_t)((uint64_t)kmin + ((((uint64_t)bb << 20) + ((1ull << z) - 1ull)) >> z));
  };
  const uint32_t bin_top = (span << z) >> 20;
  const bool none_above = b >= bin_top;  // no key lies in a bin above b
  const bool all_from_b = b == 0;         // every key lies in bin b or above
  const float f_above = none_above ? 0.f : topk_key_value(first_key(b + 1));
  const float f_in_b = all_from_b ? 0.f : topk_key_value(first_key(b));
  for_pairs([&](float x, uint32_t pos) {
    if (pos >= (uint32_t)nn) return;
    const bool above = !none_above && x >= f_above;
    const bool in_b = !above && (all_from_b || x >= f_in_b);
    if (above || (whole && in_b)) {
      atomicOr(&bm[pos >> 5], 1u << (pos & 31u));
    } else if (in_b) {
      const uint32_t slot = atomicAdd(&sh.ncand, 1u);
      if (slot < (uint32_t)kTopkBinMax) {
        bk[slot] = topk_key(x);  // the exact key: clamping may have merged keys of the top bin
        bp[slot] = pos;
      }
    }
  });
  __syncthreads();
  const uint32_t n_set = sh.ncand < (uint32_t)kTopkBinMax ? sh.ncand : (uint32_t)kTopkBinMax;
  if (!whole) {
    // rank among the bin (larger keys first, then lower positions), spread over every warp:
    // warp w ranks candidates w, w + kFusedWarps, ...; its lanes compare 32 others at a time
    for (uint32_t x = (uint32_t)warp; x < n_set; x += kFusedWarps) {
      const uint32_t k0 = bk[x], p0 = bp[x];
      uint32_t rank = 0;
      for (uint32_t y0 = 0; y0 < n_set; y0 += 32) {
        const uint32_t y = y0 + (uint32_t)lane;
        const bool before = y < n_set && (bk[y] > k0 || (bk[y] == k0 && bp[y] < p0));
        rank += (uint32_t)__popc(__ballot_sync(0xFFFFFFFFu, before));
      }
      if (lane == 0 && rank < need) atomicOr(&bm[p0 >> 5], 1u << (p0 & 31u));
    }
  }
  __syncthreads();
  // ascending output: each thread lists the positions of its run of bitmap words, into the
  // histogram's words (free since the bin pick) when the row fits there, and the row then
  // leaves in coalesced stores.  (At most K bits are set: the bins above b hold fewer than
  // K candidates, the ranking marks the rest, and a position is marked once.)
  const int wpt = (W + kFusedThreads - 1) / kFusedThreads;
  const int w0 = tid * wpt, w1 = w0 + wpt < W ? w0 + wpt : W;
  uint32_t mine = 0;
  for (int w = w0; w < w1; ++w) mine += __popc(bm[w]);
  uint32_t total;
  uint32_t at = block_scan_w<kFusedWarps>(mine, sh.tot, bank, total);
  const bool staged = a.K <= 4096;  // uniform
  uint32_t* ob = h;
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = bm[w];
    while (bits) {
      const int q = __ffs(bits) - 1;
      bits &= bits - 1;
      if (staged) ob[at] = (uint32_t)(w * 32 + q);
      else out[at] = w * 32 + q;
      ++at;
    }
  }
  if (staged) {
    __syncthreads();
    const uint32_t n_out = total < (uint32_t)a.K ? total : (uint32_t)a.K;
    if ((reinterpret_cast<uintptr_t>(out) & 15u) == 0 && (n_out & 3u) == 0) {
      for (uint32_t j = tid; j < n_out / 4; j += kFusedThreads)
        reinterpret_cast<int4*>(out)[j] = reinterpret_cast<const int4*>(ob)[j];
    } else {
      for (uint32_t j = tid; j < n_out; j += kFusedThreads) out[j] = (int32_t)ob[j];
    }
  }
  return true;
}

// e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no infinities) to float.
DSA_DEV float topk_e4m3(uint32_t v) {
  const uint32_t e = (v >> 3) & 15u, m = v & 7u;
  const float x = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;
  return (v & 0x80u) ? -x : x;
}

// Recompute the indexer scores of packed row r (sequence b, positions 0 .. nn-1) into
// srow on CUDA cores, with the head weights applied as the indexer's epilogue does.
DSA_DEV void topk_recompute_scores(const TopkArgs& a, int64_t r, int b, int nn, float* srow,
                                   float* s_q, float* s_w) {
  const int tid = threadIdx.x;
  const int H = a.idx_heads;
  const int D = 64 * H;
  if (tid < D) {
    if (a.idx_fp8) s_q[tid] = topk_e4m3(static_cast<const uint8_t*>(a.q_idx)[r * D + tid]);
    else s_q[tid] = __uint_as_float((uint32_t)static_cast<const uint16_t*>(a.q_idx)[r * D + tid] << 16);
  }
  if (tid < H)
    s_w[tid] = a.w_row_stride ? __ldg(a.w + r * a.w_row_stride + tid) : __ldg(a.w + tid) * a.idx_scale;
  __syncthreads();
  for (int j = tid; j < nn; j += kTopkThreads) {
    const int64_t krow = cache_row(a.kv_offsets, a.pages, b, j);
    float acc = 0.f;
    for (int h = 0; h < H; ++h) {
      float dot = 0.f;
      if (a.idx_fp8) {
        const uint4* kr = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.k_idx) +
                                                         krow * D + h * 64);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 u = __ldg(kr + v);
          const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int q = 0; q < 16; ++q)
            dot = fmaf(s_q[h * 64 + v * 16 + q], topk_e4m3((wds[q >> 2] >> (8 * (q & 3))) & 255u), dot);
        }
      } else {
        const uint4* kr = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.k_idx) +
                                                         krow * D + h * 64);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const uint4 u = __ldg(kr + v);
          const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t bits = (q & 1) ? (wds[q >> 1] & 0xFFFF0000u) : (wds[q >> 1] << 16);
            dot = fmaf(s_q[h * 64 + v * 8 + q], __uint_as_float(bits), dot);
          }
        }
      }
      acc = a.w_row_stride ? fmaf(s_w[h], fmaxf(dot * a.idx_scale, 0.f), acc)
                           : fmaf(s_w[h], fmaxf(dot, 0.f), acc);
    }
    srow[j] = acc;
  }
  __syncthreads();
}

DSA_DEV int64_t topk_row_len(const TopkArgs& a, int64_t r, int* b_out) {
  const int b = seq_of_row(a.q_offsets, a.batch, r);
  const int64_t qo = __ldg(a.q_offsets + b), qn = __ldg(a.q_offsets + b + 1);
  const int64_t L = (int64_t)__ldg(a.kv_offsets + b + 1) - __ldg(a.kv_offsets + b);
  const int64_t p = L - (qn - qo) + (r - qo);
  *b_out = b;
  return p >= 0 ? (p >> a.blk_shift) + 1 : 0;
}

template <int MODE>
__global__ void __launch_bounds__(kTopkThreads, 2) topk_kernel(TopkArgs a) {
  extern __shared__ uint32_t dyn[];
  __shared__ TopkShared sh;
  const int tid = threadIdx.x;
  const int K = a.K;

  if (MODE == kTopkFallback) {
    __shared__ float s_q[256];
    __shared__ float s_w[4];
    __shared__ int s_rows;
    if (tid == 0) s_rows = a.fb_list[0];
    __syncthreads();
    const int rows = s_rows;
    float* srow = a.fb_scores + (int64_t)blockIdx.x * a.ld_fb;
    for (int k = blockIdx.x; k < rows; k += gridDim.x) {
      const int64_t i = a.fb_list[1 + k];
      const int64_t r = a.q_begin + i;
      int b;
      const int nn = (int)topk_row_len(a, r, &b);
      __syncthreads();  // the previous row is finished with the shared areas
      topk_recompute_scores(a, r, b, nn, srow, s_q, s_w);
      topk_scores_row<false>(a, nn, srow, a.idx + i * a.ld_idx, dyn, sh);
      if (tid == 0 && a.cnt) a.cnt[i] = K;
    }
    return;
  }

  const int64_t i = a.q_count - 1 - (int64_t)blockIdx.x;  // rows late in a sequence first
  const int64_t r = a.q_begin + i;
  int b;
  const int64_t n = topk_row_len(a, r, &b);
  int32_t* out = a.idx + i * a.ld_idx;
  if (n <= K) {
    for (int j = tid; j < K; j += kTopkThreads) out[j] = j < n ? j : -1;
    if (a.cnt && tid == 0) a.cnt[i] = (int32_t)n;
    return;
  }
  topk_scores_row<true>(a, (int)n, a.scores + i * a.ld, out, dyn, sh);
  if (tid == 0 && a.cnt) a.cnt[i] = K;
}

// topk_kernel<kTopkScores> for launches of at most one row per SM (decode): one CTA per SM,
// so the candidate pass can hold the next run of the row in registers while it compacts the
// current one.
__global__ void __launch_bounds__(kTopkThreads, 1) topk_rows_alone_kernel(TopkArgs a) {
  extern __shared__ uint32_t dyn[];
  __shared__ TopkShared sh;
  const int tid = threadIdx.x;
  const int K = a.K;
  const int64_t i = a.q_count - 1 - (int64_t)blockIdx.x;
  const int64_t r = a.q_begin + i;
  int b;
  const int64_t n = topk_row_len(a, r, &b);
  int32_t* out = a.idx + i * a.ld_idx;
  if (n <= K) {
    for (int j = tid; j < K; j += kTopkThreads) out[j] = j < n ? j : -1;
    if (a.cnt && tid == 0) a.cnt[i] = (int32_t)n;
    return;
  }
  topk_scores_row<true, true>(a, (int)n, a.scores + i * a.ld, out, dyn, sh);
  if (tid == 0 && a.cnt) a.cnt[i] = K;
}

// Fused selection, one CTA of kFusedThreads per row (up to six CTAs share an SM).
__global__ void __launch_bounds__(kFusedThreads, kFusedCtasPerSm) topk_fused_kernel(TopkArgs a) {
  extern __shared__ uint32_t dyn[];
  __shared__ TopkShared sh;
  const int tid = threadIdx.x;
  const int K = a.K;
  const int64_t i = a.q_count - 1 - (int64_t)blockIdx.x;
  const int64_t r = a.q_begin + i;
  // the row's counts and range do not depend on its length: load them with it
  const int4 c4 = __ldg(reinterpret_cast<const int4*>(a.cand_cnt) + i);
  const uint32_t k_hi = a.khi ? __ldg(a.khi + i) : 0u;
  const float thr_i = __ldg(a.thr + i);
  int b;
  const int64_t n = topk_row_len(a, r, &b);
  int32_t* out = a.idx + i * a.ld_idx;
  if (n <= K) {
    for (int j = tid; j < K; j += kFusedThreads) out[j] = j < n ? j : -1;
    if (a.cnt && tid == 0) a.cnt[i] = (int32_t)n;
    return;
  }
  const int seg = a.cap >> 2;
  if (tid == kFusedThreads - 32 && a.prefetch_ahead > 0 && i >= a.prefetch_ahead) {
    // the CTA that will take row i2 starts about when this one ends: pull its candidate
    // segments towards L2 now (a hint only; nothing waits for it)
    const int64_t i2 = i - a.prefetch_ahead;
    const int4 n4 = __ldg(reinterpret_cast<const int4*>(a.cand_cnt) + i2);
    const int nseg[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int n = nseg[q] < seg ? nseg[q] : seg;
      if (n > 0)
        bulk_prefetch_l2(a.cand + i2 * (int64_t)a.cap + (int64_t)q * seg,
                         (uint32_t)(((int64_t)n * 8 + 15) & ~int64_t(15)));
    }
  }
  const uint32_t cnt[4] = {(uint32_t)c4.x, (uint32_t)c4.y, (uint32_t)c4.z, (uint32_t)c4.w};
  const uint32_t C = cnt[0] + cnt[1] + cnt[2] + cnt[3];
  const bool over = cnt[0] > (uint32_t)seg || cnt[1] > (uint32_t)seg || cnt[2] > (uint32_t)seg ||
                    cnt[3] > (uint32_t)seg;
  const uint32_t k_lo = k_hi ? topk_key(thr_i) : 0u;
  if (over || C < (uint32_t)K ||
      !topk_candidates_row(a, (int)n, a.cand + i * (int64_t)a.cap, seg, cnt, C, k_lo, k_hi, out,
                           dyn, sh)) {
    if (tid == 0) a.fb_list[1 + atomicAdd(a.fb_list, 1)] = (int32_t)i;
    return;
  }
  if (tid == 0 && a.cnt) a.cnt[i] = K;
}

// ---------------------------------------------------------------- block granularity
// Scores of blocks of 2^bshift positions from the indexer's 32-key maxima: out[row][m] =
// max of in[row][m G .. m G + G - 1] (G = 2^bshift / 32) over the row's n32 = p/32 + 1
// entries.  One CTA of 256 threads per row.
struct BlockArgs {
  const int32_t* q_offsets;
  const int32_t* kv_offsets;
  int batch;
  int64_t q_begin;
  const float* in;
  int64_t ld_in;
  float* out;
  int64_t ld_out;
  int bshift;
  // expansion
  const int32_t* blk;  // [rows, Kb] selected blocks, ascending, -1 padded
  int Kb;
  int32_t* idx;        // [rows, ld_idx] positions
  int64_t ld_idx;
  int32_t* cnt;        // [rows] positions selected, or nullptr
};

DSA_DEV int64_t block_row_p(const BlockArgs& a, int64_t r) {
  const int b = seq_of_row(a.q_offsets, a.batch, r);
  const int64_t qo = __ldg(a.q_offsets + b), qn = __ldg(a.q_offsets + b + 1);
  const int64_t L = (int64_t)__ldg(a.kv_offsets + b + 1) - __ldg(a.kv_offsets + b);
  return L - (qn - qo) + (r - qo);
}

__global__ void __launch_bounds__(256) block_max_kernel(BlockArgs a) {
  const int64_t i = blockIdx.x;
  const int64_t p = block_row_p(a, a.q_begin + i);
  if (p < 0) return;
  const int64_t n32 = (p >> 5) + 1, nb = (p >> a.bshift) + 1;
  const int G = 1 << (a.bshift - 5);
  const float* in = a.in + i * a.ld_in;
  float* out = a.out + i * a.ld_out;
  for (int64_t m = threadIdx.x; m < nb; m += blockDim.x) {
    float mx = -INFINITY;
    for (int g = 0; g < G; ++g) {
      const int64_t e = m * G + g;
      if (e < n32) mx = fmaxf(mx, __ldg(in + e));
    }
    out[m] = mx;
  }
}

// Positions of the selected blocks, ascending (only the block holding p can be partial and
// it is the last one selected), then -1 up to Kb << bshift.
__global__ void __launch_bounds__(256) block_expand_kernel(BlockArgs a) {
  const int64_t i = blockIdx.x;
  const int64_t p = block_row_p(a, a.q_begin + i);
  const int B = 1 << a.bshift;
  const int32_t* blk = a.blk + i * (int64_t)a.Kb;
  int32_t* out = a.idx + i * a.ld_idx;
  __shared__ int s_cnt;
  if (threadIdx.x == 0) s_cnt = 0;
  __syncthreads();
  int mine = 0;
  for (int e = threadIdx.x; e < a.Kb * B; e += blockDim.x) {
    const int m = __ldg(blk + e / B);
    const int64_t j = (int64_t)m * B + (e % B);
    const bool ok = m >= 0 && j <= p;
    out[e] = ok ? (int32_t)j : -1;
    mine += ok;
  }
  if (a.cnt) {
    atomicAdd(&s_cnt, mine);
    __syncthreads();
    if (threadIdx.x == 0) a.cnt[i] = s_cnt;
  }
}

// One warp per row: the R-th largest of the row's S samples, R = S K / n plus a margin of
// 5 sigma + 16, so that at least K scores of the row are >= it with overwhelming probability
// while about R n / S are.  The samples are bf16 rounded toward -infinity (each is at most its
// score), so the R-th largest of them is a lower bound of the exact one and the estimate stays
// on the safe side.  They become 16-bit order-preserving keys (-0.0 folded onto +0.0), mapped
// onto the full 16-bit range ((key - kmin) << clz16(kmax - kmin)), and two 8-bit radix levels
// find the R-th largest exactly.  Rows with n <= K need no candidates (+inf); rows with
// n <= cap keep every score (-inf).  The largest sample's key (as a 32-bit score key) is kept
// for the selection's key range.  A warp stages up to a.stage samples in shared memory; longer
// rows are read from global memory in each pass.
constexpr int kThrWarps = 4;
constexpr int kThrStageMax = 2048;  // samples a warp stages at most (4 KiB)
__host__ inline size_t topk_thr_smem_bytes(int stage) {
  return (size_t)kThrWarps * stage * 2;
}
DSA_DEV uint32_t thr_key16(uint32_t b) {
  b &= 0xFFFFu;
  if (b == 0x8000u) b = 0u;  // -0.0 == +0.0
  return (b & 0x8000u) ? (~b & 0xFFFFu) : (b | 0x8000u);
}
DSA_DEV float thr_key16_value(uint32_t k) {
  const uint32_t b = (k & 0x8000u) ? (k ^ 0x8000u) : (~k & 0xFFFFu);
  return __uint_as_float(b << 16);
}
__global__ void __launch_bounds__(32 * kThrWarps) topk_thr_kernel(TopkThrArgs a) {
  __shared__ uint32_t hist[kThrWarps][256];
  extern __shared__ __align__(16) uint16_t thr_stage[];  // [kThrWarps][a.stage]
  const int warp = threadIdx.x >> 5, lane = lane_id();
  if (blockIdx.x == 0 && threadIdx.x == 0) a.fb_list[0] = 0;
  const int64_t i = (int64_t)blockIdx.x * kThrWarps + warp;
  if (i >= a.q_count) return;  // warp-uniform; only warp-level syncs below
  const int64_t r = a.q_begin + i;
  const int b = seq_of_row(a.q_offsets, a.batch, r);
  const int64_t qo = __ldg(a.q_offsets + b), qn = __ldg(a.q_offsets + b + 1);
  const int64_t L = (int64_t)__ldg(a.kv_offsets + b + 1) - __ldg(a.kv_offsets + b);
  const int64_t p = L - (qn - qo) + (r - qo);
  const int64_t n = p + 1;
  if (n <= a.K || n <= a.cap) {
    if (lane == 0) {
      a.thr[i] = n <= a.K ? INFINITY : -INFINITY;
      a.khi[i] = 0u;
    }
    return;
  }
  const int S = (int)(p >> a.shift) + 1;
  if (a.long_rows && S > a.stage) return;  // a CTA of topk_thr_long_kernel takes the row
  const float e = (float)a.K * (float)S / (float)n;
  int R = (int)ceilf(e + 5.f * sqrtf(e) + 16.f);
  if (R > S) R = S;
  uint32_t* h = hist[warp];
#pragma unroll
  for (int q = 0; q < 8; ++q) h[lane * 8 + q] = 0;
  const uint16_t* row = a.samp + i * a.ld_s;
  const bool staged = S <= a.stage;
  uint16_t* st = thr_stage + (size_t)warp * a.stage;
  uint32_t lo = 0xFFFFu, hi = 0u;
  // every key of the row, f(key), from the staged keys or from global memory (8 samples per
  // 16-byte load, several loads in flight per lane)
  auto for_keys = [&](auto&& f) {
    if (staged) {
      for (int m = lane; m < S; m += 32) f((uint32_t)st[m]);
    } else {
      for (int m0 = 0; m0 < S; m0 += 4 * 32 * 8) {
        uint4 u[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int m = m0 + (v * 32 + lane) * 8;
          u[v] = m < S ? __ldg(reinterpret_cast<const uint4*>(row + m)) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int m = m0 + (v * 32 + lane) * 8;
          const uint32_t w4[4] = {u[v].x, u[v].y, u[v].z, u[v].w};
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (m + q < S) f(thr_key16(w4[q >> 1] >> (16 * (q & 1))));
        }
      }
    }
  };
  if (staged) {
    // stage the keys and take their range on the way (rows are 16-byte aligned and padded to
    // ld_s >= a multiple of 8 >= S)
    const int S8 = (S + 7) & ~7;
    for (int m0 = 0; m0 < S8; m0 += 4 * 32 * 8) {
      uint4 u[4];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int m = m0 + (v * 32 + lane) * 8;
        u[v] = m < S8 ? __ldg(reinterpret_cast<const uint4*>(row + m)) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int m = m0 + (v * 32 + lane) * 8;
        if (m < S8) {
          const uint32_t w4[4] = {u[v].x, u[v].y, u[v].z, u[v].w};
          uint32_t k[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            k[q] = thr_key16(w4[q >> 1] >> (16 * (q & 1)));
            if (m + q < S) {
              lo = k[q] < lo ? k[q] : lo;
              hi = k[q] > hi ? k[q] : hi;
            }
          }
          *reinterpret_cast<uint4*>(st + m) =
              make_uint4(k[0] | (k[1] << 16), k[2] | (k[3] << 16), k[4] | (k[5] << 16),
                         k[6] | (k[7] << 16));
        }
      }
    }
    __syncwarp();
  } else {
    for_keys([&](uint32_t k) {
      lo = k < lo ? k : lo;
      hi = k > hi ? k : hi;
    });
  }
  lo = __reduce_min_sync(0xFFFFFFFFu, lo);
  hi = __reduce_max_sync(0xFFFFFFFFu, hi);
  const int z = hi != lo ? __clz(hi - lo) - 16 : 0;  // normalised keys fill 16 bits
  __syncwarp();
  uint32_t prefix = 0, mask = 0, remaining = (uint32_t)R;
  for (int level = 0; level < 2; ++level) {
    const int sh = 8 - 8 * level;
    for_keys([&](uint32_t k) {
      const uint32_t nk = ((k - lo) << z) & 0xFFFFu;
      if ((nk & mask) == prefix) atomicAdd(&h[(nk >> sh) & 255u], 1u);
    });
    __syncwarp();
    // lane l owns bins 255 - 8l - q, q = 0..7 (from the top)
    uint32_t c[8], sum = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      c[q] = h[255 - 8 * lane - q];
      sum += c[q];
    }
    const uint32_t incl = warp_incl_scan(sum);
    const unsigned own = __ballot_sync(0xFFFFFFFFu, incl - sum < remaining && remaining <= incl);
    const int o = __ffs(own) - 1;
    uint32_t bin = 0, rem = 0;
    if (lane == o) {
      uint32_t above = incl - sum;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (above < remaining && remaining <= above + c[q]) {
          bin = 255u - 8u * (uint32_t)lane - (uint32_t)q;
          rem = remaining - above;
        }
        above += c[q];
      }
    }
    bin = __shfl_sync(0xFFFFFFFFu, bin, o);
    rem = __shfl_sync(0xFFFFFFFFu, rem, o);
    prefix |= bin << sh;
    mask |= 255u << sh;
    remaining = rem;
    __syncwarp();
#pragma unroll
    for (int q = 0; q < 8; ++q) h[lane * 8 + q] = 0;
    __syncwarp();
  }
  if (lane == 0) {
    a.thr[i] = thr_key16_value(lo + (prefix >> z));
    a.khi[i] = topk_key(thr_key16_value(hi));
  }
}

// topk_thr_kernel's selection for rows of more than a.stage samples, one CTA of
// kThrLongThreads per row: the row's bf16 samples are read once, with many loads in flight, and
// staged as 16-bit keys in shared memory (long_stage >= every row's sample count: the launch
// passes ld_s), and the CTA's warps build the two 8-bit radix histograms together; one warp
// picks each level's bin.  The result is the one topk_thr_kernel would give for the row.
// Other rows return at once.
constexpr int kThrLongThreads = 256;
__host__ inline size_t topk_thr_long_smem_bytes(int long_stage) { return (size_t)long_stage * 2; }
__global__ void __launch_bounds__(kThrLongThreads) topk_thr_long_kernel(TopkThrArgs a, int long_stage) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_lo, s_hi, s_sel[2];
  extern __shared__ __align__(16) uint16_t thr_long_stage[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = lane_id();
  const int64_t i = blockIdx.x;
  const int64_t r = a.q_begin + i;
  const int b = seq_of_row(a.q_offsets, a.batch, r);
  const int64_t qo = __ldg(a.q_offsets + b), qn = __ldg(a.q_offsets + b + 1);
  const int64_t L = (int64_t)__ldg(a.kv_offsets + b + 1) - __ldg(a.kv_offsets + b);
  const int64_t p = L - (qn - qo) + (r - qo);
  const int64_t n = p + 1;
  if (n <= a.K || n <= a.cap) return;  // topk_thr_kernel writes these rows
  const int S = (int)(p >> a.shift) + 1;
  if (S <= a.stage || S > long_stage) return;  // uniform (S > long_stage never happens)
  const float e = (float)a.K * (float)S / (float)n;
  int R = (int)ceilf(e + 5.f * sqrtf(e) + 16.f);
  if (R > S) R = S;
  const uint16_t* row = a.samp + i * a.ld_s;
  uint16_t* st = thr_long_stage;
  for (int t = tid; t < 256; t += kThrLongThreads) hist[t] = 0;
  if (tid == 0) {
    s_lo = 0xFFFFu;
    s_hi = 0u;
  }
  __syncthreads();
  // stage the keys (8 per 16-byte load, every thread's loads in flight) and their range
  uint32_t lo = 0xFFFFu, hi = 0u;
  const int S8 = (S + 7) & ~7;  // rows are 16-byte aligned and padded to ld_s >= S8
  constexpr int kLd = 4;
  for (int m0 = 0; m0 < S8; m0 += kLd * kThrLongThreads * 8) {
    uint4 u[kLd];
#pragma unroll
    for (int v = 0; v < kLd; ++v) {
      const int m = m0 + (v * kThrLongThreads + tid) * 8;
      u[v] = m < S8 ? __ldg(reinterpret_cast<const uint4*>(row + m)) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int v = 0; v < kLd; ++v) {
      const int m = m0 + (v * kThrLongThreads + tid) * 8;
      if (m < S8) {
        const uint32_t w4[4] = {u[v].x, u[v].y, u[v].z, u[v].w};
        uint32_t k[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          k[q] = thr_key16(w4[q >> 1] >> (16 * (q & 1)));
          if (m + q < S) {
            lo = k[q] < lo ? k[q] : lo;
            hi = k[q] > hi ? k[q] : hi;
          }
        }
        *reinterpret_cast<uint4*>(st + m) =
            make_uint4(k[0] | (k[1] << 16), k[2] | (k[3] << 16), k[4] | (k[5] << 16),
                       k[6] | (k[7] << 16));
      }
    }
  }
  lo = __reduce_min_sync(0xFFFFFFFFu, lo);
  hi = __reduce_max_sync(0xFFFFFFFFu, hi);
  if (lane == 0) {
    atomicMin(&s_lo, lo);
    atomicMax(&s_hi, hi);
  }
  __syncthreads();  // keys staged, range known
  lo = s_lo;
  hi = s_hi;
  const int z = hi != lo ? __clz(hi - lo) - 16 : 0;  // normalised keys fill 16 bits
  uint32_t prefix = 0, mask = 0, remaining = (uint32_t)R;
  for (int level = 0; level < 2; ++level) {
    const int sh = 8 - 8 * level;
    for (int m = tid; m < S; m += kThrLongThreads) {
      const uint32_t nk = (((uint32_t)st[m] - lo) << z) & 0xFFFFu;
      if ((nk & mask) == prefix) atomicAdd(&hist[(nk >> sh) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns bins 255 - 8l - q, q = 0..7 (from the top)
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        c[q] = hist[255 - 8 * lane - q];
        sum += c[q];
      }
      const uint32_t incl = warp_incl_scan(sum);
      const unsigned own = __ballot_sync(0xFFFFFFFFu, incl - sum < remaining && remaining <= incl);
      const int o = __ffs(own) - 1;
      if (lane == o) {
        uint32_t above = incl - sum;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (above < remaining && remaining <= above + c[q]) {
            s_sel[0] = 255u - 8u * (uint32_t)lane - (uint32_t)q;
            s_sel[1] = remaining - above;
          }
          above += c[q];
        }
      }
    }
    __syncthreads();  // bin picked, histogram read
    prefix |= s_sel[0] << sh;
    mask |= 255u << sh;
    remaining = s_sel[1];
    for (int t = tid; t < 256; t += kThrLongThreads) hist[t] = 0;
    __syncthreads();  // histogram zeroed, s_sel read
  }
  if (tid == 0) {
    a.thr[i] = thr_key16_value(lo + (prefix >> z));
    a.khi[i] = topk_key(thr_key16_value(hi));
  }
}

}  // namespace dsa
