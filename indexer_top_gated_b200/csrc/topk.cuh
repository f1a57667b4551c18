// topk.cuh - step 2 of the layer: per-row Top-K selection by radix select.
//
// For a score row s[0..n) (n = p+1 causal candidates) and K < n:
//  - every fp32 score becomes an order-preserving 32-bit key (-0.0 folded onto +0.0);
//  - up to four MSB-first 8-bit digit passes build a 256-bin shared-memory histogram of
//    the keys that still match the chosen prefix (warp-aggregated atomics: lanes with
//    the same digit add once), and pick the bin holding the K-th largest key;
//  - one ordered pass over positions then keeps every key above the threshold plus the
//    first (K - count above) keys equal to it: a block-wide exclusive scan of packed
//    (definite, tie) counts gives each kept position its output slot, so the output is
//    in ascending position order and ties go to the lower position.
// Rows of up to kTopkStageCap scores are staged in shared memory on the first pass, so
// the row is read from global memory once; longer rows are re-read (from L2).
// No sort, no global scratch.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kTopkThreads = 1024;
constexpr int kTopkStageCap = 32768;  // scores staged in shared memory (128 KiB)

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

// Add 1 to hist[bin] for every active lane; lanes sharing a bin add once together.
DSA_DEV void hist_add(uint32_t* hist, uint32_t bin, bool active) {
  const unsigned m = __ballot_sync(0xFFFFFFFFu, active);
  if (active) {
    const unsigned peers = __match_any_sync(m, bin);
    if ((int)(__ffs(peers) - 1) == lane_id()) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
  }
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

__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(TopkArgs a) {
  extern __shared__ uint32_t s_keys[];  // [kTopkStageCap] when the row is staged
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_tot[33];
  __shared__ uint32_t s_sel[3];  // chosen digit, remaining, early-exit flag

  const int tid = threadIdx.x;
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
  uint32_t prefix = 0, mask = 0, remaining = (uint32_t)K;
  bool ge_mode = false;  // true: keep every key >= prefix, no ties to split

  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int t = tid; t < 256; t += kTopkThreads) hist[t] = 0;
    __syncthreads();
    for (int64_t base = 0; base < n; base += 4 * kTopkThreads) {
      const int64_t j0 = base + 4 * tid;
      uint32_t k4[4];
      if (pass == 0 || !staged) {
        if (j0 + 3 < n) {
          const float4 f = __ldg(reinterpret_cast<const float4*>(row + j0));
          k4[0] = topk_key(f.x); k4[1] = topk_key(f.y);
          k4[2] = topk_key(f.z); k4[3] = topk_key(f.w);
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q) k4[q] = j0 + q < n ? topk_key(__ldg(row + j0 + q)) : 0u;
        }
        if (pass == 0 && staged) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (j0 + q < n) s_keys[j0 + q] = k4[q];
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) k4[q] = j0 + q < n ? s_keys[j0 + q] : 0u;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool act = (j0 + q < n) && ((k4[q] & mask) == prefix);
        hist_add(hist, (k4[q] >> shift) & 255u, act);
      }
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns bins 255-8l .. 248-8l (descending); find the bin where the count of
      // larger keys first reaches `remaining`
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        c[q] = hist[255 - 8 * tid - q];
        sum += c[q];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (tid >= o) incl += y;
      }
      const uint32_t excl = incl - sum;
      const bool mine = excl < remaining && remaining <= incl;
      if (mine) {
        uint32_t above = excl;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (above < remaining && remaining <= above + c[q]) {
            s_sel[0] = 255u - 8u * tid - q;
            s_sel[1] = remaining - above;
            s_sel[2] = (remaining - above == c[q]) ? 1u : 0u;
          }
          above += c[q];
        }
      }
    }
    __syncthreads();
    const uint32_t digit = s_sel[0];
    remaining = s_sel[1];
    prefix |= digit << shift;
    mask |= 255u << shift;
    if (s_sel[2]) {  // the whole bin is kept: threshold is "key >= prefix"
      ge_mode = true;
      break;
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
