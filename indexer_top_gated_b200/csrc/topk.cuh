// topk.cuh - step 2 of the layer: per-row Top-K selection by radix select.
//
// For a score row s[0..n) (n = p+1 causal candidates) and K < n:
//  - every fp32 score becomes an order-preserving 32-bit key (-0.0 folded onto +0.0);
//  - pass A: a 4096-bin shared-memory histogram of the top 12 key bits over the whole row
//    (the row is staged in shared memory on the way when it fits) picks the bin that
//    holds the K-th largest key;
//  - the keys of that bin (at most kTopkCandCap of them) are compacted into a candidate
//    list, and two 1024-bin passes over the candidates alone settle the remaining 20 bits,
//    giving the exact threshold key tau and how many keys equal to tau are still needed;
//    a bin that is kept whole ends the search early;
//  - one ordered pass over positions keeps every key above tau plus the first needed keys
//    equal to it: a block-wide exclusive scan of packed (definite, tie) counts gives each
//    kept position its output slot, so the output is in ascending position order and
//    ties go to the lower position.
// Full-row passes: 3 (histogram, candidate compaction, output).  A threshold bin larger
// than the candidate list falls back to filtered passes over the whole row.  No sort and
// no global scratch.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kTopkThreads = 1024;
constexpr int kTopkStageCap = 32768;  // scores staged in shared memory (128 KiB)
constexpr int kTopkCandCap = 16384;   // candidate keys of the threshold bin (64 KiB)
constexpr int kTopkHistBins = 4096;

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
  const bool staged = n <= kTopkStageCap;
  // four consecutive keys starting at j0 (0 past the end)
  auto load4 = [&](int64_t j0, uint32_t (&k4)[4], bool from_global) {
    if (!from_global) {
#pragma unroll
      for (int q = 0; q < 4; ++q) k4[q] = j0 + q < n ? s_keys[j0 + q] : 0u;
    } else if (j0 + 3 < n) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(row + j0));
      k4[0] = topk_key(f.x);
      k4[1] = topk_key(f.y);
      k4[2] = topk_key(f.z);
      k4[3] = topk_key(f.w);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) k4[q] = j0 + q < n ? topk_key(__ldg(row + j0 + q)) : 0u;
    }
  };

  // ---- pass A: histogram of the top 12 bits (and staging)
  for (int t = tid; t < kTopkHistBins; t += kTopkThreads) hist[t] = 0;
  if (tid == 0) s_ncand = 0;
  __syncthreads();
  for (int64_t base = 0; base < n; base += 4 * kTopkThreads) {
    const int64_t j0 = base + 4 * tid;
    uint32_t k4[4];
    load4(j0, k4, true);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (j0 + q < n) {
        if (staged) s_keys[j0 + q] = k4[q];
        atomicAdd(&hist[k4[q] >> 20], 1u);
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
      for (int64_t base = 0; base < n; base += 4 * kTopkThreads) {
        const int64_t j0 = base + 4 * tid;
        uint32_t k4[4];
        load4(j0, k4, !staged);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const bool m = (j0 + q < n) && ((k4[q] >> 20) == b12);
          const unsigned bal = __ballot_sync(0xFFFFFFFFu, m);
          if (bal) {
            uint32_t slot = 0;
            if (lane == 0) slot = atomicAdd(&s_ncand, (uint32_t)__popc(bal));
            slot = __shfl_sync(0xFFFFFFFFu, slot, 0);
            if (m) cand[slot + __popc(bal & ((1u << lane) - 1u))] = k4[q] & 0xFFFFFu;
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
        for (int64_t base = 0; base < n; base += 4 * kTopkThreads) {
          const int64_t j0 = base + 4 * tid;
          uint32_t k4[4];
          load4(j0, k4, !staged);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (j0 + q < n && (k4[q] & want_mask) == prefix)
              atomicAdd(&hist[(k4[q] >> shift) & 1023u], 1u);
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
  for (int64_t base = 0; base < n; base += 4 * kTopkThreads) {
    const int64_t j0 = base + 4 * tid;
    uint32_t k4[4];
    if (staged) {
#pragma unroll
      for (int q = 0; q < 4; ++q) k4[q] = j0 + q < n ? s_keys[j0 + q] : 0u;
    } else if (j0 + 3 < n) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(row + j0));
      k4[0] = topk_key(f.x); k4[1] = topk_key(f.y);
      k4[2] = topk_key(f.z); k4[3] = topk_key(f.w);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) k4[q] = j0 + q < n ? topk_key(__ldg(row + j0 + q)) : 0u;
    }
    uint32_t dflag = 0, tflag = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const bool valid = j0 + q < n;
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
  if (tid == 0 && a.cnt) a.cnt[i] = K;
}

}  // namespace dsa
