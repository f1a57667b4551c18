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
  // level 1: lane l owns the l-th block of PER bins counted from the top
  const int hi1 = NB - 1 - lane * PER;
  uint32_t sum = 0;
#pragma unroll
  for (int q = 0; q < PER; q += 4) {
    const uint4 u = *reinterpret_cast<const uint4*>(hist + hi1 - PER + 1 + q);
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

__global__ void __launch_bounds__(kTopkThreads, 2) topk_kernel(TopkArgs a) {
  extern __shared__ uint32_t dyn[];
  uint32_t* hA = dyn;            // 4096: sample, top 12 bits
  uint32_t* hB = hA + 4096;      // 1024: sample, next 10 bits
  uint32_t* hC = hB + 1024;      // 1024: sample, last 10 bits
  uint32_t* hD = hC + 1024;      // 4096: candidates / row, top 12 bits
  uint32_t* hE = hD + 4096;      // 1024
  uint32_t* hF = hE + 1024;      // 1024
  uint32_t* cand = dyn + kTopkHistWords;
  uint32_t* fk = cand;                 // fast path: candidate keys      [kTopkFastCap]
  uint32_t* fp = cand + kTopkFastCap;  // fast path: candidate positions [kTopkFastCap]
  __shared__ uint32_t s_tot[64];
  __shared__ uint32_t s_sel[3];
  __shared__ uint32_t s_ncand;

  const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;
  const int64_t i = a.q_count - 1 - (int64_t)blockIdx.x;  // rows late in a sequence first
  const int64_t r = a.q_begin + i;
  const int b = seq_of_row(a.q_offsets, a.batch, r);
  const int64_t qo = __ldg(a.q_offsets + b), qn = __ldg(a.q_offsets + b + 1);
  const int64_t L = (int64_t)__ldg(a.kv_offsets + b + 1) - __ldg(a.kv_offsets + b);
  const int64_t p = L - (qn - qo) + (r - qo);
  const int64_t n = p + 1 > 0 ? p + 1 : 0;
  const int K = a.K;
  int32_t* out = a.idx + i * a.ld_idx;

  if (n <= K) {
    for (int j = tid; j < K; j += kTopkThreads) out[j] = j < n ? j : -1;
    if (a.cnt && tid == 0) a.cnt[i] = (int32_t)n;
    return;
  }

  const float* row = a.scores + i * a.ld;
  const int nn = (int)n;  // rows are shorter than 2^31
  int bank = 0;
  {
    // pull the whole row towards L2 now, so that its DRAM latency overlaps the threshold
    // estimate below and the candidate pass reads from L2 (the row is 16-byte aligned and
    // its padded length round4(n) <= ld)
    const int64_t bytes = (((int64_t)nn + 3) & ~int64_t(3)) * 4;
    constexpr int64_t kPiece = 16384;
    for (int64_t off = (int64_t)tid * kPiece; off < bytes; off += (int64_t)kTopkThreads * kPiece)
      bulk_prefetch_l2(reinterpret_cast<const char*>(row) + off,
                       (uint32_t)(bytes - off < kPiece ? bytes - off : kPiece));
  }
  // four consecutive keys starting at j0 (a multiple of 4; 0 past the end)
  auto load4 = [&](int j0, uint32_t (&k4)[4]) {
    if (j0 + 3 < nn) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(row + j0));
      k4[0] = topk_key(f.x);
      k4[1] = topk_key(f.y);
      k4[2] = topk_key(f.z);
      k4[3] = topk_key(f.w);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) k4[q] = j0 + q < nn ? topk_key(__ldg(row + j0 + q)) : 0u;
    }
  };
  // radix select over keys held by the threads (`get(c)` for c in [0, count) strided by
  // thread), in hist12 / hist10a / hist10b (zeroed): returns the threshold key in *tau and
  // the count still needed from keys equal to it (0 when the threshold bin is kept whole).
  auto select = [&](uint32_t* h12, uint32_t* h10a, uint32_t* h10b, uint32_t want, auto&& get,
                    uint32_t count, int levels, uint32_t* tau, bool* whole) -> uint32_t {
    for (uint32_t c = tid; c < count; c += kTopkThreads) atomicAdd(&h12[get(c) >> 20], 1u);
    __syncthreads();
    if (warp == 0) warp_select<4096>(h12, want, s_sel);
    __syncthreads();
    uint32_t t = s_sel[0] << 20, need = s_sel[1];
    bool w = s_sel[2] != 0;
    if (!w) {
      for (uint32_t c = tid; c < count; c += kTopkThreads) {
        const uint32_t key = get(c);
        if ((key & 0xFFF00000u) == t) atomicAdd(&h10a[(key >> 10) & 1023u], 1u);
      }
      __syncthreads();
      if (warp == 0) warp_select<1024>(h10a, need, s_sel);
      __syncthreads();
      t |= s_sel[0] << 10;
      need = s_sel[1];
      w = s_sel[2] != 0;
      if (!w && levels > 2) {
        for (uint32_t c = tid; c < count; c += kTopkThreads) {
          const uint32_t key = get(c);
          if ((key & 0xFFFFFC00u) == t) atomicAdd(&h10b[key & 1023u], 1u);
        }
        __syncthreads();
        if (warp == 0) warp_select<1024>(h10b, need, s_sel);
        __syncthreads();
        t |= s_sel[0];
        need = s_sel[1];
        w = s_sel[2] != 0;
      }
    }
    *tau = t;
    *whole = w;
    return w ? 0u : need;
  };

  // ---- zero every histogram once
  for (int t = tid; t < kTopkHistWords; t += kTopkThreads) dyn[t] = 0;
  if (tid == 0) s_ncand = 0;
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
      for (int j = tid; j < nn; j += kTopkThreads) fk[j] = topk_key(__ldg(row + j));
    }
    __syncthreads();
    auto sget = [&](uint32_t c) -> uint32_t { return fk[c]; };
    uint32_t t_est;
    bool sw;
    // 22 bits of the estimate are plenty: every sample >= t_est counts towards m
    select(hA, hB, hC, (uint32_t)m, sget, (uint32_t)S, 2, &t_est, &sw);
    __syncthreads();  // samples read; the candidate pass may overwrite them

    // -- candidates: every key >= t_est, in position order.  The comparison is done on the
    // raw scores (key order = float order, -0.0 == +0.0); keys are formed only for the
    // candidates.
    const float t_val = topk_key_value(t_est);
    uint32_t run = 0;
    bool overflow = false;
    for (int cb = 0; cb < nn && !overflow; cb += kTopkRun) {
      float4 xb[kTopkBatch];
#pragma unroll
      for (int it = 0; it < kTopkBatch; ++it) {  // warp w owns positions cb + 1024 w .. + 1023
        const int j0 = cb + warp * 1024 + it * 128 + lane * 4;
        if (j0 + 3 < nn) {
          xb[it] = __ldg(reinterpret_cast<const float4*>(row + j0));
        } else {
          xb[it].x = j0 < nn ? __ldg(row + j0) : -INFINITY;
          xb[it].y = j0 + 1 < nn ? __ldg(row + j0 + 1) : -INFINITY;
          xb[it].z = j0 + 2 < nn ? __ldg(row + j0 + 2) : -INFINITY;
          xb[it].w = j0 + 3 < nn ? __ldg(row + j0 + 3) : -INFINITY;
        }
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
      const uint32_t wb = block_scan(lane == 31 ? wtot : 0u, s_tot, bank, chunk_total);
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
      // -- exact selection among the candidates
      const uint32_t C = run;
      auto cget = [&](uint32_t c) -> uint32_t { return fk[c]; };
      uint32_t tau;
      bool ge;
      const uint32_t ties_needed = select(hD, hE, hF, (uint32_t)K, cget, C, 3, &tau, &ge);
      // -- ordered output over the candidates (they are in position order)
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
        const uint32_t before = block_scan(packed, s_tot, bank, total);
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
      if (tid == 0 && a.cnt) a.cnt[i] = K;
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
  if (warp == 0) warp_select<4096>(hD, (uint32_t)K, s_sel);
  __syncthreads();
  const uint32_t b12 = s_sel[0];
  uint32_t remaining = s_sel[1];
  uint32_t prefix = b12 << 20;
  bool ge_mode = s_sel[2] != 0;
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
              if (lane == 0) slot = atomicAdd(&s_ncand, (uint32_t)__popc(bal));
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
      if (warp == 0) warp_select<1024>(h, remaining, s_sel);
      __syncthreads();
      prefix |= s_sel[0] << shift;
      remaining = s_sel[1];
      ge_mode = s_sel[2] != 0;
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
      const uint32_t before = block_scan(packed, s_tot, bank, total);
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
  if (tid == 0 && a.cnt) a.cnt[i] = K;
}

}  // namespace dsa
