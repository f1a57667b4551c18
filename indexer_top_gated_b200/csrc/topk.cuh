// topk.cuh - step 2 of the layer: per-row Top-K selection by radix select.
//
// For a score row s[0..n) (n = p+1 causal candidates) and K < n, every fp32 score becomes
// an order-preserving 32-bit key (-0.0 folded onto +0.0).
//
// Fast path (almost every row):
//  - 1024 evenly spaced samples give an estimate t of the K-th largest key: the sample of
//    rank S*K/n plus a margin of 4 sigma + 8 (radix select over the samples), so that with
//    overwhelming probability at least K keys of the row are >= t;
//  - one ordered pass keeps every key >= t, with its position, as a candidate in shared
//    memory (each warp owns a contiguous run of positions; packed warp scans and one block
//    scan per 32768 positions give the slots, so candidates stay in position order);
//  - an exact radix select (12 + 10 + 10 bits) over the candidates alone finds the
//    threshold key tau and how many keys equal to tau are still needed; an ordered pass
//    over the candidates writes the selected positions in ascending order, ties going to
//    the lower position.
// Exact path (if the estimate was off: fewer than K candidates, or more than fit):
//  - a 4096-bin histogram of the top 12 key bits over the whole row (staged in shared
//    memory when it fits), the threshold bin's keys refined by two 10-bit digits, then one
//    ordered pass over the whole row.
// No sort and no global scratch.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kTopkThreads = 1024;
constexpr int kTopkStageCap = 32768;  // scores staged in shared memory (128 KiB)
constexpr int kTopkCandCap = 16384;   // candidate keys of the threshold bin (64 KiB)
constexpr int kTopkHistBins = 4096;
constexpr int kTopkBatch = 8;         // row loads kept in flight per thread
constexpr int kTopkFastCap = kTopkCandCap / 2;  // fast-path candidates (key + position)

__host__ inline size_t topk_smem_bytes(int64_t max_kv_len) {
  const int64_t stage = max_kv_len + 4 < kTopkStageCap ? max_kv_len + 4 : kTopkStageCap;
  return (size_t)(kTopkHistBins + kTopkCandCap + stage) * sizeof(uint32_t);
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

// Block-wide exclusive scan of one 32-bit value per thread (1024 threads).
DSA_DEV uint32_t block_excl_scan(uint32_t v, uint32_t* warp_tot, uint32_t& total) {
  const int lane = lane_id(), warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = warp_tot[lane];
    uint32_t s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xFFFFFFFFu, s, o);
      if (lane >= o) s += y;
    }
    warp_tot[lane] = s - t;  // exclusive prefix of warp totals
    if (lane == 31) warp_tot[32] = s;
  }
  __syncthreads();
  const uint32_t res = warp_tot[warp] + x - v;
  total = warp_tot[32];
  __syncthreads();  // warp_tot reused by the next call
  return res;
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

// Pick, over hist[0 .. 1024*BPT) scanned from the top bin down, the bin in which the
// count of larger keys first reaches `remaining`.  s_sel = {bin, still needed from that
// bin, bin kept whole}.  All threads return after s_sel is visible.
template <int BPT>
DSA_DEV void select_bin(const uint32_t* hist, uint32_t remaining, uint32_t* warp_tot,
                        uint32_t* s_sel) {
  const int top = kTopkThreads * BPT - 1;
  const int tid = threadIdx.x;
  uint32_t c[BPT], sum = 0;
#pragma unroll
  for (int q = 0; q < BPT; ++q) {
    c[q] = hist[top - tid * BPT - q];
    sum += c[q];
  }
  uint32_t total;
  const uint32_t excl = block_excl_scan(sum, warp_tot, total);
  if (excl < remaining && remaining <= excl + sum) {
    uint32_t above = excl;
#pragma unroll
    for (int q = 0; q < BPT; ++q) {
      if (above < remaining && remaining <= above + c[q]) {
        s_sel[0] = (uint32_t)(top - tid * BPT - q);
        s_sel[1] = remaining - above;
        s_sel[2] = (remaining - above == c[q]) ? 1u : 0u;
      }
      above += c[q];
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(TopkArgs a) {
  extern __shared__ uint32_t dyn[];
  uint32_t* hist = dyn;                         // [kTopkHistBins]
  uint32_t* cand = dyn + kTopkHistBins;         // [kTopkCandCap]
  uint32_t* s_keys = cand + kTopkCandCap;       // [kTopkStageCap] when the row is staged
  __shared__ uint32_t warp_tot[33];
  __shared__ uint32_t s_sel[3];
  __shared__ uint32_t s_ncand;

  const int tid = threadIdx.x, lane = lane_id();
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
  const bool staged = nn <= kTopkStageCap;
  // four consecutive keys starting at j0 (a multiple of 4; 0 past the end)
  auto load4 = [&](int j0, uint32_t (&k4)[4], bool from_global) {
    if (j0 + 3 < nn) {
      if (from_global) {
        const float4 f = __ldg(reinterpret_cast<const float4*>(row + j0));
        k4[0] = topk_key(f.x);
        k4[1] = topk_key(f.y);
        k4[2] = topk_key(f.z);
        k4[3] = topk_key(f.w);
      } else {
        const uint4 u = *reinterpret_cast<const uint4*>(s_keys + j0);
        k4[0] = u.x;
        k4[1] = u.y;
        k4[2] = u.z;
        k4[3] = u.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        k4[q] = j0 + q < nn ? (from_global ? topk_key(__ldg(row + j0 + q)) : s_keys[j0 + q]) : 0u;
    }
  };

  // ================================================================ fast path
  uint32_t* fk = cand;                  // candidate keys      [kTopkFastCap]
  uint32_t* fp = cand + kTopkFastCap;   // candidate positions [kTopkFastCap]
  {
    // -- threshold estimate: the m-th largest of S evenly spaced samples
    const int S = nn < kTopkThreads ? nn : kTopkThreads;
    const bool sact = tid < S;
    const uint32_t skey = sact ? topk_key(__ldg(row + (int)(((int64_t)tid * nn) / S))) : 0u;
    const float m_exp = (float)S * (float)K / (float)nn;
    int m = (int)ceilf(m_exp + 4.f * sqrtf(m_exp) + 8.f);
    if (m > S) m = S;
    for (int t = tid; t < kTopkHistBins; t += kTopkThreads) hist[t] = 0;
    __syncthreads();
    if (sact) atomicAdd(&hist[skey >> 20], 1u);
    __syncthreads();
    select_bin<4>(hist, (uint32_t)m, warp_tot, s_sel);
    uint32_t t_est = s_sel[0] << 20;
    uint32_t rem = s_sel[1];
    bool whole = s_sel[2] != 0;
    for (int level = 0; level < 2 && !whole; ++level) {
      const int shift = level == 0 ? 10 : 0;
      const uint32_t mask = level == 0 ? 0xFFF00000u : 0xFFFFFC00u;
      for (int t = tid; t < 1024; t += kTopkThreads) hist[t] = 0;
      __syncthreads();
      if (sact && (skey & mask) == t_est) atomicAdd(&hist[(skey >> shift) & 1023u], 1u);
      __syncthreads();
      select_bin<1>(hist, rem, warp_tot, s_sel);
      t_est |= s_sel[0] << shift;
      rem = s_sel[1];
      whole = s_sel[2] != 0;
    }
    // -- candidates: every key >= t_est, in position order
    uint32_t run = 0;
    bool overflow = false;
    const int warp = tid >> 5;
    for (int cb = 0; cb < nn && !overflow; cb += 32 * kTopkThreads) {
      uint32_t kb[8][4];
#pragma unroll
      for (int it = 0; it < 8; ++it)  // warp w owns positions cb + 1024 w .. + 1023
        load4(cb + warp * 1024 + it * 128 + lane * 4, kb[it], true);
      uint32_t fl = 0;                  // bit 4*it + q: key q of iteration it is kept
      uint32_t cnt_lo = 0, cnt_hi = 0;  // per-iteration counts packed in bytes
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int j0 = cb + warp * 1024 + it * 128 + lane * 4;
        uint32_t f = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) f |= (uint32_t)(j0 + q < nn && kb[it][q] >= t_est) << q;
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
      const uint32_t wbase = block_excl_scan(lane == 31 ? wtot : 0u, warp_tot, chunk_total);
      // block_excl_scan sums one value per thread: only lane 31 contributes its warp's total,
      // so the exclusive prefix seen by lane 0 of warp w is the count of warps before w
      const uint32_t warp_base = __shfl_sync(0xFFFFFFFFu, wbase, 0);
      if (run + chunk_total > (uint32_t)kTopkFastCap) {
        overflow = true;  // uniform: chunk_total is the block total
        break;
      }
      uint32_t pre = run + warp_base;  // candidates before iteration `it` of this warp
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const uint32_t lo = it < 4 ? (exc_lo >> (8 * it)) & 255u : (exc_hi >> (8 * (it - 4))) & 255u;
        const uint32_t tt = it < 4 ? (tot_lo >> (8 * it)) & 255u : (tot_hi >> (8 * (it - 4))) & 255u;
        uint32_t slot = pre + lo;
        const int j0 = cb + warp * 1024 + it * 128 + lane * 4;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if ((fl >> (4 * it + q)) & 1u) {
            fk[slot] = kb[it][q];
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
      for (int t = tid; t < kTopkHistBins; t += kTopkThreads) hist[t] = 0;
      __syncthreads();
      for (uint32_t c = tid; c < C; c += kTopkThreads) atomicAdd(&hist[fk[c] >> 20], 1u);
      __syncthreads();
      select_bin<4>(hist, (uint32_t)K, warp_tot, s_sel);
      uint32_t tau = s_sel[0] << 20;
      uint32_t need = s_sel[1];
      bool ge = s_sel[2] != 0;
      for (int level = 0; level < 2 && !ge; ++level) {
        const int shift = level == 0 ? 10 : 0;
        const uint32_t mask = level == 0 ? 0xFFF00000u : 0xFFFFFC00u;
        for (int t = tid; t < 1024; t += kTopkThreads) hist[t] = 0;
        __syncthreads();
        for (uint32_t c = tid; c < C; c += kTopkThreads) {
          const uint32_t key = fk[c];
          if ((key & mask) == tau) atomicAdd(&hist[(key >> shift) & 1023u], 1u);
        }
        __syncthreads();
        select_bin<1>(hist, need, warp_tot, s_sel);
        tau |= s_sel[0] << shift;
        need = s_sel[1];
        ge = s_sel[2] != 0;
      }
      // -- ordered output over the candidates (they are in position order)
      const uint32_t ties_needed = ge ? 0u : need;
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
        const uint32_t before = block_excl_scan(packed, warp_tot, total);
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
  // ---- pass A: histogram of the top 12 bits (and staging)
  for (int t = tid; t < kTopkHistBins; t += kTopkThreads) hist[t] = 0;
  if (tid == 0) s_ncand = 0;
  __syncthreads();
  for (int base = 0; base < nn; base += 4 * kTopkThreads * kTopkBatch) {
    uint32_t kb[kTopkBatch][4];
#pragma unroll
    for (int bb = 0; bb < kTopkBatch; ++bb)  // all loads in flight before any is used
      load4(base + bb * 4 * kTopkThreads + 4 * tid, kb[bb], true);
#pragma unroll
    for (int bb = 0; bb < kTopkBatch; ++bb) {
      const int j0 = base + bb * 4 * kTopkThreads + 4 * tid;
      if (j0 + 3 < nn) {
        if (staged)
          *reinterpret_cast<uint4*>(s_keys + j0) = make_uint4(kb[bb][0], kb[bb][1], kb[bb][2], kb[bb][3]);
#pragma unroll
        for (int q = 0; q < 4; ++q) atomicAdd(&hist[kb[bb][q] >> 20], 1u);
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (j0 + q < nn) {
            if (staged) s_keys[j0 + q] = kb[bb][q];
            atomicAdd(&hist[kb[bb][q] >> 20], 1u);
          }
        }
      }
    }
  }
  __syncthreads();
  select_bin<4>(hist, (uint32_t)K, warp_tot, s_sel);
  const uint32_t b12 = s_sel[0];
  uint32_t remaining = s_sel[1];
  uint32_t prefix = b12 << 20;
  bool ge_mode = s_sel[2] != 0;  // true: keep every key >= prefix, no ties to split

  if (!ge_mode) {
    const uint32_t n_bin = hist[b12];
    const bool use_cand = n_bin <= (uint32_t)kTopkCandCap;
    __syncthreads();  // every thread has read hist[b12] before it is cleared below
    if (use_cand) {
      // candidates: low 20 bits of the keys in the threshold bin (order is irrelevant)
      for (int base = 0; base < nn; base += 4 * kTopkThreads * kTopkBatch) {
        uint32_t kb[kTopkBatch][4];
#pragma unroll
        for (int bb = 0; bb < kTopkBatch; ++bb)
          load4(base + bb * 4 * kTopkThreads + 4 * tid, kb[bb], !staged);
#pragma unroll
        for (int bb = 0; bb < kTopkBatch; ++bb) {
          const int j0 = base + bb * 4 * kTopkThreads + 4 * tid;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const bool m = (j0 + q < nn) && ((kb[bb][q] >> 20) == b12);
            const unsigned bal = __ballot_sync(0xFFFFFFFFu, m);
            if (bal) {
              uint32_t slot = 0;
              if (lane == 0) slot = atomicAdd(&s_ncand, (uint32_t)__popc(bal));
              slot = __shfl_sync(0xFFFFFFFFu, slot, 0);
              if (m) cand[slot + __popc(bal & ((1u << lane) - 1u))] = kb[bb][q] & 0xFFFFFu;
            }
          }
        }
      }
    }
    // two 10-bit digits below the 12-bit prefix
    for (int level = 0; level < 2 && !ge_mode; ++level) {
      const int shift = level == 0 ? 10 : 0;
      for (int t = tid; t < 1024; t += kTopkThreads) hist[t] = 0;
      __syncthreads();
      if (use_cand) {
        for (uint32_t c = tid; c < n_bin; c += kTopkThreads) {
          const uint32_t low = cand[c];
          if (level == 0 || (low >> 10) == ((prefix >> 10) & 1023u))
            atomicAdd(&hist[(low >> shift) & 1023u], 1u);
        }
      } else {
        const uint32_t want_mask = level == 0 ? 0xFFF00000u : 0xFFFFFC00u;
        for (int base = 0; base < nn; base += 4 * kTopkThreads * kTopkBatch) {
          uint32_t kb[kTopkBatch][4];
#pragma unroll
          for (int bb = 0; bb < kTopkBatch; ++bb)
            load4(base + bb * 4 * kTopkThreads + 4 * tid, kb[bb], !staged);
#pragma unroll
          for (int bb = 0; bb < kTopkBatch; ++bb) {
            const int j0 = base + bb * 4 * kTopkThreads + 4 * tid;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (j0 + q < nn && (kb[bb][q] & want_mask) == prefix)
                atomicAdd(&hist[(kb[bb][q] >> shift) & 1023u], 1u);
          }
        }
      }
      __syncthreads();
      select_bin<1>(hist, remaining, warp_tot, s_sel);
      prefix |= s_sel[0] << shift;
      remaining = s_sel[1];
      ge_mode = s_sel[2] != 0;
    }
  }

  // Ordered compaction.  Definite: key > tau (or >= prefix in ge_mode).  Ties: key == tau,
  // the first `remaining` of them in position order are kept.
  const uint32_t tau = prefix;
  const uint32_t ties_needed = ge_mode ? 0u : remaining;
  uint32_t run_def = 0, run_tie = 0;
  for (int base = 0; base < nn; base += 4 * kTopkThreads * kTopkBatch) {
    uint32_t kb[kTopkBatch][4];
#pragma unroll
    for (int bb = 0; bb < kTopkBatch; ++bb)
      load4(base + bb * 4 * kTopkThreads + 4 * tid, kb[bb], !staged);
#pragma unroll
    for (int bb = 0; bb < kTopkBatch; ++bb) {
      if (base + bb * 4 * kTopkThreads >= nn) continue;  // uniform across the block
      const int j0 = base + bb * 4 * kTopkThreads + 4 * tid;
      const uint32_t (&k4)[4] = kb[bb];
      uint32_t dflag = 0, tflag = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool valid = j0 + q < nn;
        const bool def = valid && (ge_mode ? k4[q] >= tau : k4[q] > tau);
        const bool tie = valid && !ge_mode && k4[q] == tau;
        dflag |= (uint32_t)def << q;
        tflag |= (uint32_t)tie << q;
      }
      // packed counts: low 16 bits definite, high 16 bits ties (each <= 4096 per block)
      const uint32_t packed = (uint32_t)__popc(dflag) | ((uint32_t)__popc(tflag) << 16);
      uint32_t total;
      const uint32_t before = block_excl_scan(packed, warp_tot, total);
      uint32_t d_before = run_def + (before & 0xFFFFu);
      uint32_t t_before = run_tie + (before >> 16);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool def = (dflag >> q) & 1u, tie = (tflag >> q) & 1u;
        if (def) {
          const uint32_t slot = d_before + (t_before < ties_needed ? t_before : ties_needed);
          out[slot] = (int32_t)(j0 + q);
          ++d_before;
        } else if (tie) {
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
