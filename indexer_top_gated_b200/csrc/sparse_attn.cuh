// sparse_attn.cuh - steps 3-4 of the layer: exact softmax attention over the selected
// cache rows, with the sigmoid output gate fused into the epilogue.
//
// One CTA per (query row, pair of KV heads or one KV head), 4 warps, three CTAs per SM.  Each warp owns
// one KV head and 16 positions of every chunk of selected positions, and gathers exactly
// the bytes it consumes, so warps never synchronise with each other inside the main loop:
//  - gather: the warp's 16 positions x (K and V slices of its head, 256 B each) arrive
//    through 16-byte cp.async (32 lanes = 512 contiguous bytes per instruction) into the
//    warp's own 2-stage ring (XOR-swizzled 16-byte chunks, conflict-free for ldmatrix).
//    Index entries are read once per position, and the row's offset (32 bits: bytes or
//    16-byte units, or the row index for the largest caches) is shared across the warp by
//    shuffles; padding / out-of-range entries copy the sequence's first row (finite data)
//    and are masked (a ballot mask).
//  - logits are computed transposed, S^T = K_sel Q^T (mma.sync m16n8k16, keys on M, the
//    group's 8 query heads on N, two independent accumulation chains), so a group of 8
//    heads needs no padding and the query heads of a GQA group share the gather.
//  - online softmax in registers (log2 domain); P^T becomes the B operand of
//    O^T += V_sel^T P^T through movmatrix (8x8 transposes in registers) and V^T comes
//    from ldmatrix.trans.  P enters rounded to bf16 (2^-9 relative per weight; the row sum
//    l is taken from the fp32 weights).  Carrying P as P_hi + P_lo (two bf16 terms, ~2^-17)
//    was measured at 8 % more time for the whole kernel: the output is bf16 itself, so the
//    single rounding costs no more than the output's own.
//  - warps of the same KV head merge (m, l, O) through shared memory; the epilogue
//    divides by l, multiplies by sigmoid(gate) (and adds the second branch weighted by
//    1 - sigmoid(gate) when one is given) and stores bf16 (and the LSE).
// The work per row is bound by the gather bytes (K * Hkv * d * 2 * 2 per query), so the
// tensor-core path here only has to keep up with memory.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kHeadDim = 128;
constexpr float kLazyMax = 8.f;  // log2 units the running maximum may lag behind

// CTA shape: 4 warps with 2-stage rings (64 KiB), three CTAs per SM (12 warps, the most
// that the ~150-170 registers per thread and the rings allow).  A CTA holds two KV heads
// (two warps each, 32 positions per chunk) or one head (four warps, 64 positions per
// chunk): for a layer with a single KV head, and in decode, where one query per sequence
// gives too few rows to fill the GPU with two-head CTAs.  Several small CTAs per SM overlap one row's
// set-up (index scan, query loads, first gathers) and merge / epilogue with the main
// loops of the others, which one large CTA per SM left exposed.
template <int HKV_CTA>
struct AttnShape {
  static_assert(HKV_CTA == 1 || HKV_CTA == 2, "one or two KV heads per CTA");
  static constexpr int kWarps = 4;
  static constexpr int kStages = 2;
  static constexpr int kCtasPerSm = 3;
};

struct AttnArgs {
  const int32_t* q_offsets;
  const int32_t* kv_offsets;
  int batch;
  int64_t q_begin;
  int64_t q_count;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* idx;
  int64_t ld_idx;
  int K;
  const __nv_bfloat16* gate;
  const __nv_bfloat16* other;  // second branch to mix in (needs gate), or nullptr
  __nv_bfloat16* out;
  float* lse;
  int32_t* err_count;
  int* status;
  int Hq, Hkv, G;
  float scale_log2;  // softmax scale * log2(e)
  CachePages pages;  // paged k_cache / v_cache
};

template <int HKV_CTA>
struct AttnGeom {
  static constexpr int kWarps = AttnShape<HKV_CTA>::kWarps;
  static constexpr int kStages = AttnShape<HKV_CTA>::kStages;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kWPG = kWarps / HKV_CTA;      // warps per KV head
  static constexpr int kChunk = 16 * kWPG;           // positions per chunk (all warps)
  static constexpr int kWarpHalf = 16 * kHeadDim * 2;  // one warp's K (or V) slice: 4 KiB
  static constexpr int kWarpStage = 2 * kWarpHalf;     // K + V: 8 KiB
};

__host__ inline size_t attn_smem_bytes() {
  return (size_t)AttnGeom<1>::kWarps * AttnGeom<1>::kStages * AttnGeom<1>::kWarpStage +
         128 /*align*/;
}

// How a selected row's 16-byte pieces are addressed (AM): kAddrBytes32, each cache spans at
// most 4 GiB, so a piece is the cache's base plus a shuffled 32-bit byte offset;
// kAddrUnits32, at most 64 GiB, the same with the offset in 16-byte units; kAddrRows, any
// size: the shuffled 32-bit row index times the row's size in 16-byte units, widened to 64
// bits per piece and array.
constexpr int kAddrBytes32 = 1;
constexpr int kAddrUnits32 = 2;
constexpr int kAddrRows = 3;

template <int HKV_CTA, int NT, int AM>
__global__ void __launch_bounds__(AttnGeom<HKV_CTA>::kThreads, AttnShape<HKV_CTA>::kCtasPerSm)
    sparse_attn_kernel(AttnArgs a) {
  using Geo = AttnGeom<HKV_CTA>;
  constexpr int CH = Geo::kChunk;
  constexpr int kAttnThreads = Geo::kThreads;
  constexpr int kAttnWarps = Geo::kWarps;
  constexpr int kAttnStages = Geo::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ int s_last;
  __shared__ int s_err;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t i = a.q_count - 1 - (int64_t)blockIdx.x;
  const int64_t r = a.q_begin + i;
  const int g0 = (int)blockIdx.y * HKV_CTA;
  const int b = seq_of_row(a.q_offsets, a.batch, r);
  const int64_t qo = __ldg(a.q_offsets + b), qn = __ldg(a.q_offsets + b + 1);
  const int64_t kbase = __ldg(a.kv_offsets + b);
  const int64_t L = (int64_t)__ldg(a.kv_offsets + b + 1) - kbase;
  const int64_t p = L - (qn - qo) + (r - qo);
  const int32_t* irow = a.idx + i * a.ld_idx;
  const int K = a.K;

  // ---- scan the index row: last non-padding entry, and out-of-range entries
  if (tid == 0) {
    s_last = -1;
    s_err = 0;
  }
  __syncthreads();
  {
    int last = -1, err = 0;
    if ((K & 3) == 0 && (reinterpret_cast<uintptr_t>(irow) & 15) == 0) {
      // four entries per 16-byte load, all of a thread's loads in flight
      const int4* i4 = reinterpret_cast<const int4*>(irow);
      for (int e4 = tid; e4 < (K >> 2); e4 += kAttnThreads) {
        const int4 v = __ldg(i4 + e4);
        const int jj[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (jj[q] >= 0) {
            if ((int64_t)jj[q] <= p) last = 4 * e4 + q;
            else ++err;
          }
        }
      }
    } else {
      for (int e = tid; e < K; e += kAttnThreads) {
        const int j = __ldg(irow + e);
        if (j >= 0) {
          if ((int64_t)j <= p) last = e;
          else ++err;
        }
      }
    }
    if (last >= 0) atomicMax(&s_last, last);
    if (err) atomicAdd(&s_err, err);
  }
  __syncthreads();
  if (tid == 0 && s_err && a.err_count && blockIdx.y == 0) atomicAdd(a.err_count, s_err);
  const int n_chunks = (s_last + CH) / CH;  // 0 when nothing is selected

  // ---- per-warp state: one KV head (g) and positions sub*16 .. sub*16+15 of every chunk
  const int g = warp / Geo::kWPG;
  const int sub = warp % Geo::kWPG;
  const int hg = g0 + g;  // KV head
  uint8_t* wsm = smem + (size_t)warp * kAttnStages * Geo::kWarpStage;  // this warp's ring
  const uint32_t row_stride = (uint32_t)a.Hkv * kHeadDim;  // elements per cache row

  // gather chunk c into ring slot st; returns the validity mask of its 16 positions.
  // Lane t < 16 reads the index of position t; every cp.async step then moves two whole
  // 256-byte head slices (512 contiguous bytes per warp instruction), the row's offset
  // arriving by shuffle.  Padding and out-of-range entries copy the sequence's first row
  // (finite data) and are masked in the softmax, so the copies need no per-piece predicate.
  const int lt = lane & 15, lhi = lane >> 4;
  const uint32_t swz = (uint32_t)((lt ^ lhi) << 4);  // lt ^ ((2k + lhi) & 7) = (lt ^ lhi) ^ 2k&7
  // a cache row's size and this lane's piece within it, in bytes or in 16-byte units
  constexpr uint32_t kUnit = AM == kAddrBytes32 ? 1u : 16u;
  const uint32_t row_off = row_stride * 2u / kUnit;
  const uint32_t piece_off = (uint32_t)((hg * kHeadDim + lt * 8) * 2) / kUnit;
  const char* kb = reinterpret_cast<const char*>(a.k);
  const char* vb = reinterpret_cast<const char*>(a.v);
  auto load_chunk = [&](int c, int st) -> uint32_t {
    const int e = c * CH + sub * 16 + lt;
    const int j = e < K ? __ldg(irow + e) : -1;
    const bool valid = j >= 0 && (int64_t)j <= p;
    const uint32_t vmask = __ballot_sync(0xFFFFFFFFu, valid) & 0xFFFFu;
    // the cache row of the position (or of position 0 for padding)
    const int rowi = a.pages.table ? (int)cache_row(a.kv_offsets, a.pages, b, valid ? j : 0)
                                   : (int)kbase + (valid ? j : 0);
    const uint32_t kdst = smem_u32(wsm + st * Geo::kWarpStage) + lhi * 256;
    const uint32_t vdst = kdst + Geo::kWarpHalf;
    if (AM != kAddrRows) {
      const uint32_t myoff = (uint32_t)rowi * row_off;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t off = __shfl_sync(0xFFFFFFFFu, myoff, 2 * k + lhi) + piece_off;
        const uint32_t so = (uint32_t)(k * 512) + (swz ^ (uint32_t)(((2 * k) & 7) << 4));
        if (AM == kAddrUnits32) {
          cp_async_16(kdst + so, reinterpret_cast<const uint4*>(kb) + off, 16u);
          cp_async_16(vdst + so, reinterpret_cast<const uint4*>(vb) + off, 16u);
        } else {
          cp_async_16(kdst + so, kb + off, 16u);
          cp_async_16(vdst + so, vb + off, 16u);
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t rt = (uint32_t)__shfl_sync(0xFFFFFFFFu, rowi, 2 * k + lhi);
        const uint64_t off = (uint64_t)rt * row_off + piece_off;
        const uint32_t so = (uint32_t)(k * 512) + (swz ^ (uint32_t)(((2 * k) & 7) << 4));
        cp_async_16(kdst + so, reinterpret_cast<const uint4*>(kb) + off, 16u);
        cp_async_16(vdst + so, reinterpret_cast<const uint4*>(vb) + off, 16u);
      }
    }
    return vmask;
  };

  uint32_t bq[NT][8][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int hh = nt * 8 + (lane >> 2);
    const bool hv = hh < a.G;
    const __nv_bfloat16* qh = a.q + (r * a.Hq + (int64_t)hg * a.G + (hv ? hh : 0)) * kHeadDim;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int d0 = ks * 16 + 2 * (lane & 3);
      bq[nt][ks][0] = hv ? __ldg(reinterpret_cast<const uint32_t*>(qh + d0)) : 0u;
      bq[nt][ks][1] = hv ? __ldg(reinterpret_cast<const uint32_t*>(qh + d0 + 8)) : 0u;
    }
  }
  float o[NT][8][4];
  float m_run[NT][2], l_run[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int q = 0; q < 4; ++q) o[nt][mt][q] = 0.f;
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_run[nt][0] = l_run[nt][1] = 0.f;
  }

  // ldmatrix row of this lane within the warp's 16 positions (K: A rows; V: A^T rows)
  const int kt = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int vt = (lane & 7) + (lane >> 4) * 8;
  const int kch = lane >> 4, vch = (lane >> 3) & 1;

  uint64_t vmasks = 0;  // 16-bit validity mask of each ring slot
#pragma unroll
  for (int s = 0; s < kAttnStages - 1; ++s) {
    if (s < n_chunks) vmasks |= (uint64_t)load_chunk(s, s) << (16 * s);
    cp_async_commit();
  }

  for (int c = 0; c < n_chunks; ++c) {
    cp_async_wait<kAttnStages - 2>();
    __syncwarp();
    const int st = c % kAttnStages;
    const uint32_t vm = (uint32_t)(vmasks >> (16 * st)) & 0xFFFFu;
    {
      const int nxt = c + kAttnStages - 1;
      if (nxt < n_chunks) {
        const int ns = nxt % kAttnStages;
        vmasks = (vmasks & ~(0xFFFFull << (16 * ns))) | ((uint64_t)load_chunk(nxt, ns) << (16 * ns));
      }
      cp_async_commit();
    }
    const uint32_t kst = smem_u32(wsm + st * Geo::kWarpStage);
    const uint32_t vst = kst + Geo::kWarpHalf;

    // S^T[16 pos x 8 heads] = K_sel[16 x 128] * Q^T[128 x 8]; two accumulation chains
    float s[NT][4], s2[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) s[nt][q] = s2[nt][q] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t af[4];
      const int chk = ks * 2 + kch;
      ldmatrix_x4(kst + kt * 256 + ((chk ^ (kt & 7)) << 4), af);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (ks & 1) mma_bf16_16816(s2[nt], af, bq[nt][ks][0], bq[nt][ks][1]);
        else mma_bf16_16816(s[nt], af, bq[nt][ks][0], bq[nt][ks][1]);
      }
    }
    const bool v_lo = (vm >> (lane >> 2)) & 1u;
    const bool v_hi = (vm >> ((lane >> 2) + 8)) & 1u;
    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      s[nt][0] = v_lo ? (s[nt][0] + s2[nt][0]) * a.scale_log2 : -INFINITY;
      s[nt][1] = v_lo ? (s[nt][1] + s2[nt][1]) * a.scale_log2 : -INFINITY;
      s[nt][2] = v_hi ? (s[nt][2] + s2[nt][2]) * a.scale_log2 : -INFINITY;
      s[nt][3] = v_hi ? (s[nt][3] + s2[nt][3]) * a.scale_log2 : -INFINITY;
      // Lazy running maximum: the reference m_run only moves (with a warp-wide max and a
      // rescale of the partial sums) when some logit exceeds it by more than kLazyMax, so
      // every weight stays <= 2^kLazyMax, well inside bf16 / fp32 range.
      float mx[2] = {fmaxf(s[nt][0], s[nt][2]), fmaxf(s[nt][1], s[nt][3])};
      const bool need = !(mx[0] <= m_run[nt][0] + kLazyMax) || !(mx[1] <= m_run[nt][1] + kLazyMax) ||
                        m_run[nt][0] == -INFINITY || m_run[nt][1] == -INFINITY;
      float pr[4];
      if (__any_sync(0xFFFFFFFFu, need)) {
        float alpha[2];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          mx[cc] = fmaxf(mx[cc], __shfl_xor_sync(0xFFFFFFFFu, mx[cc], 4));
          mx[cc] = fmaxf(mx[cc], __shfl_xor_sync(0xFFFFFFFFu, mx[cc], 8));
          mx[cc] = fmaxf(mx[cc], __shfl_xor_sync(0xFFFFFFFFu, mx[cc], 16));
          const float m_new = fmaxf(m_run[nt][cc], mx[cc]);
          if (m_new == -INFINITY) {
            alpha[cc] = 1.f;
            pr[cc] = 0.f;
            pr[cc + 2] = 0.f;
          } else {
            alpha[cc] = ex2_approx(m_run[nt][cc] - m_new);
            pr[cc] = ex2_approx(s[nt][cc] - m_new);
            pr[cc + 2] = ex2_approx(s[nt][cc + 2] - m_new);
          }
          m_run[nt][cc] = m_new;
          l_run[nt][cc] = l_run[nt][cc] * alpha[cc] + pr[cc] + pr[cc + 2];
        }
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          o[nt][mt][0] *= alpha[0];
          o[nt][mt][1] *= alpha[1];
          o[nt][mt][2] *= alpha[0];
          o[nt][mt][3] *= alpha[1];
        }
      } else {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          pr[cc] = ex2_approx(s[nt][cc] - m_run[nt][cc]);
          pr[cc + 2] = ex2_approx(s[nt][cc + 2] - m_run[nt][cc]);
          l_run[nt][cc] += pr[cc] + pr[cc + 2];
        }
      }
      pb[nt][0] = movmatrix_trans(pack_bf16x2(pr[0], pr[1]));  // positions 0-7
      pb[nt][1] = movmatrix_trans(pack_bf16x2(pr[2], pr[3]));  // positions 8-15
    }
    // O^T[128 dims x 8 heads] += V_sel^T[128 x 16] * P^T[16 x 8]
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t vf[4];
      const int chv = mt * 2 + vch;
      ldmatrix_x4_trans(vst + vt * 256 + ((chv ^ (vt & 7)) << 4), vf);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(o[nt][mt], vf, pb[nt][0], pb[nt][1]);
    }
    __syncwarp();  // the slot is refilled by the next iteration's loads
  }
  cp_async_wait<0>();

  __syncthreads();  // all warps are done with their rings: the memory is reused below

  // ---- merge the warps of each KV head through shared memory
  constexpr int HPW = NT * 8;  // head slots per warp
  float* red_o = reinterpret_cast<float*>(smem);       // [warps][HPW][128]
  float* red_m = red_o + kAttnWarps * HPW * kHeadDim;  // [warps][HPW]
  float* red_l = red_m + kAttnWarps * HPW;             // [warps][HPW]
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      float l = l_run[nt][cc];
      l += __shfl_xor_sync(0xFFFFFFFFu, l, 4);
      l += __shfl_xor_sync(0xFFFFFFFFu, l, 8);
      l += __shfl_xor_sync(0xFFFFFFFFu, l, 16);
      if (lane < 4) {
        const int hh = nt * 8 + 2 * lane + cc;
        red_m[warp * HPW + hh] = m_run[nt][cc];
        red_l[warp * HPW + hh] = l;
      }
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      const int d = mt * 16 + (lane >> 2);
      const int hh = nt * 8 + 2 * (lane & 3);
      float* w0 = red_o + ((size_t)warp * HPW + hh) * kHeadDim;
      w0[d] = o[nt][mt][0];
      w0[kHeadDim + d] = o[nt][mt][1];
      w0[d + 8] = o[nt][mt][2];
      w0[kHeadDim + d + 8] = o[nt][mt][3];
    }
  }
  __syncthreads();

  // ---- epilogue: normalise, gate, store (8 dims per thread per item)
  const int items = HKV_CTA * a.G * (kHeadDim / 8);
  for (int it = tid; it < items; it += kAttnThreads) {
    const int gg = it / (a.G * 16);
    const int rem = it % (a.G * 16);
    const int hh = rem / 16;
    const int d0 = (rem % 16) * 8;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < Geo::kWPG; ++w) M = fmaxf(M, red_m[(gg * Geo::kWPG + w) * HPW + hh]);
    float Lsum = 0.f, acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < Geo::kWPG; ++w) {
        const int ww = gg * Geo::kWPG + w;
        const float f = exp2f(red_m[ww * HPW + hh] - M);
        Lsum += red_l[ww * HPW + hh] * f;
        const float* src = red_o + ((size_t)ww * HPW + hh) * kHeadDim + d0;
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] += src[k] * f;
      }
    }
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    const int64_t h = (int64_t)(g0 + gg) * a.G + hh;
    const int64_t off = (r * a.Hq + h) * kHeadDim + d0;
    float gv[8];
    if (a.gate) {
      const uint4 graw = __ldg(reinterpret_cast<const uint4*>(a.gate + off));
      const __nv_bfloat16* gb = reinterpret_cast<const __nv_bfloat16*>(&graw);
#pragma unroll
      for (int k = 0; k < 8; ++k) gv[k] = 1.f / (1.f + __expf(-__bfloat162float(gb[k])));
      if (a.other) {
        // the second branch enters with weight 1 - sigmoid(g) = sigmoid(-g), formed
        // directly so that it keeps its relative precision when sigmoid(g) is near 1
        const uint4 oraw = __ldg(reinterpret_cast<const uint4*>(a.other + off));
        const __nv_bfloat16* ob = reinterpret_cast<const __nv_bfloat16*>(&oraw);
        float mix[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mix[k] = __bfloat162float(ob[k]) / (1.f + __expf(__bfloat162float(gb[k])));
        uint4 packed;
        uint32_t* pw = reinterpret_cast<uint32_t*>(&packed);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          pw[k] = pack_bf16x2(acc[2 * k] * inv * gv[2 * k] + mix[2 * k],
                              acc[2 * k + 1] * inv * gv[2 * k + 1] + mix[2 * k + 1]);
        *reinterpret_cast<uint4*>(a.out + off) = packed;
        if (a.lse && d0 == 0)
          a.lse[i * a.Hq + h] = Lsum > 0.f ? (M + __log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
        continue;
      }
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) gv[k] = 1.f;
    }
    uint4 packed;
    uint32_t* pw = reinterpret_cast<uint32_t*>(&packed);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      pw[k] = pack_bf16x2(acc[2 * k] * inv * gv[2 * k], acc[2 * k + 1] * inv * gv[2 * k + 1]);
    *reinterpret_cast<uint4*>(a.out + off) = packed;
    if (a.lse && d0 == 0)
      a.lse[i * a.Hq + h] = Lsum > 0.f ? (M + __log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
  }
}

}  // namespace dsa
