// sparse_attn.cuh - steps 3-4 of the layer: exact softmax attention over the selected
// cache rows, with the sigmoid output gate fused into the epilogue.
//
// One CTA per (query row, block of up to 8 KV heads).  Per chunk of selected positions:
//  - gather: all KV heads of a selected position are one contiguous run in the cache
//    ([pos][Hkv][d]), so the CTA copies K and V rows with 16-byte cp.async into a
//    3-stage ring in shared memory (XOR-swizzled 16-byte chunks, conflict-free for
//    ldmatrix).  Padding / out-of-range entries are zero-filled and masked.
//  - each warp owns one KV head and 16 positions of the chunk; the query heads of the
//    GQA group share that gather.  Logits are computed transposed, S^T = K_sel Q^T
//    (mma.sync m16n8k16, keys on M, the group's 8 query heads on N), so a group of 8
//    heads needs no padding.
//  - online softmax in registers (log2 domain); P^T becomes the B operand of
//    O^T += V_sel^T P^T through movmatrix (8x8 transposes in registers) and V^T comes
//    from ldmatrix.trans.  P enters as two bf16 terms (P_hi + P_lo), so rounding P
//    costs ~2^-17 relative instead of 2^-9: the error no longer scales with
//    sum_j p_j |v_j| (which dominates outputs that nearly cancel).
//  - warps of the same KV head merge (m, l, O) through shared memory; the epilogue
//    divides by l, multiplies by sigmoid(gate) and stores bf16 (and the LSE).
// The work per row is bound by the gather bytes (K * Hkv * d * 2 * 2 per query), so
// the tensor-core path here only has to keep up with memory.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kAttnThreads = 256;
constexpr int kAttnStages = 3;
constexpr int kHeadDim = 128;

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
  __nv_bfloat16* out;
  float* lse;
  int32_t* err_count;
  int Hq, Hkv, G;
  float scale_log2;  // softmax scale * log2(e)
};

template <int HKV_CTA>
struct AttnGeom {
  static constexpr int kWPG = 8 / HKV_CTA;            // warps per KV head
  static constexpr int kChunk = 16 * kWPG;            // positions per stage
  static constexpr int kRowBytes = HKV_CTA * kHeadDim * 2;
  static constexpr int kHalfBytes = kChunk * kRowBytes;  // K (or V) part of a stage
  static constexpr int kStageBytes = 2 * kHalfBytes;     // 64 KiB
  static constexpr int kPieces = kStageBytes / 16;       // 16-byte copies per stage
};

__host__ inline size_t attn_smem_bytes() {
  return (size_t)kAttnStages * AttnGeom<1>::kStageBytes + 128 /*align*/;
}

template <int HKV_CTA, int NT>
__global__ void __launch_bounds__(kAttnThreads, 1) sparse_attn_kernel(AttnArgs a) {
  using Geo = AttnGeom<HKV_CTA>;
  constexpr int CH = Geo::kChunk;
  constexpr int ROWB = Geo::kRowBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ uint8_t s_valid[kAttnStages][CH];
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
    for (int e = tid; e < K; e += kAttnThreads) {
      const int j = __ldg(irow + e);
      if (j >= 0) {
        if ((int64_t)j <= p) last = e;
        else ++err;
      }
    }
    if (last >= 0) atomicMax(&s_last, last);
    if (err) atomicAdd(&s_err, err);
  }
  __syncthreads();
  if (tid == 0 && s_err && a.err_count && blockIdx.y == 0) atomicAdd(a.err_count, s_err);
  const int n_chunks = (s_last + CH) / CH;  // 0 when nothing is selected

  // ---- gather of one chunk of selected positions into stage st.  Each warp copies whole
  // position rows: one (broadcast) index load per position, then every cp.async of the
  // warp covers a contiguous 512-byte run of the row (K and V rows alike).
  auto load_chunk = [&](int c, int st) {
    constexpr int CPR = HKV_CTA * 16;             // 16-byte pieces per position row
    constexpr int LPP = CPR < 32 ? CPR : 32;      // lanes per position
    constexpr int PPI = 32 / LPP;                 // positions per warp iteration
    constexpr int PIECES = CPR / LPP;             // pieces per lane per position row
    constexpr int PPW = CH / 8;                   // positions per warp per chunk
    uint8_t* base = smem + (size_t)st * Geo::kStageBytes;
    const int sub_lane = lane % LPP;
#pragma unroll
    for (int it = 0; it < PPW / PPI; ++it) {
      const int pos = warp * PPW + it * PPI + lane / LPP;
      const int e = c * CH + pos;
      const int j = e < K ? __ldg(irow + e) : -1;
      const bool valid = j >= 0 && (int64_t)j <= p;
      const int64_t row_elem = ((kbase + (valid ? j : 0)) * a.Hkv + g0) * kHeadDim;
      const __nv_bfloat16* ksrc = a.k + row_elem;
      const __nv_bfloat16* vsrc = a.v + row_elem;
      uint8_t* kdst = base + pos * ROWB;
      uint8_t* vdst = kdst + Geo::kHalfBytes;
#pragma unroll
      for (int q = 0; q < PIECES; ++q) {
        const int ch = sub_lane + q * LPP;
        const uint32_t off = (uint32_t)((ch ^ (pos & 7)) << 4);
        cp_async_16(smem_u32(kdst + off), valid ? (const void*)(ksrc + ch * 8) : (const void*)a.k,
                    valid ? 16u : 0u);
        cp_async_16(smem_u32(vdst + off), valid ? (const void*)(vsrc + ch * 8) : (const void*)a.k,
                    valid ? 16u : 0u);
      }
      if (sub_lane == 0) s_valid[st][pos] = valid ? 1 : 0;
    }
  };

  // ---- per-warp state: one KV head (g) and 16 positions (sub) of every chunk
  const int g = warp / Geo::kWPG;
  const int sub = warp % Geo::kWPG;
  const int hg = g0 + g;  // KV head
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

#pragma unroll
  for (int s = 0; s < kAttnStages - 1; ++s) {
    if (s < n_chunks) load_chunk(s, s);
    cp_async_commit();
  }

  for (int c = 0; c < n_chunks; ++c) {
    cp_async_wait<kAttnStages - 2>();
    __syncthreads();
    {
      const int nxt = c + kAttnStages - 1;
      if (nxt < n_chunks) load_chunk(nxt, nxt % kAttnStages);
      cp_async_commit();
    }
    const int st = c % kAttnStages;
    const uint8_t* kst = smem + (size_t)st * Geo::kStageBytes;
    const uint8_t* vst = kst + Geo::kHalfBytes;

    // S^T[16 pos x 8 heads] = K_sel[16 x 128] * Q^T[128 x 8]
    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    {
      const int pos = sub * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const uint8_t* rowp = kst + pos * ROWB;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int ch = g * 16 + ks * 2 + (lane >> 4);
        uint32_t af[4];
        ldmatrix_x4(smem_u32(rowp + ((ch ^ (pos & 7)) << 4)), af);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(s[nt], af, bq[nt][ks][0], bq[nt][ks][1]);
      }
    }
    const bool v_lo = s_valid[st][sub * 16 + (lane >> 2)] != 0;
    const bool v_hi = s_valid[st][sub * 16 + (lane >> 2) + 8] != 0;
    uint32_t pb[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      s[nt][0] = v_lo ? s[nt][0] * a.scale_log2 : -INFINITY;
      s[nt][1] = v_lo ? s[nt][1] * a.scale_log2 : -INFINITY;
      s[nt][2] = v_hi ? s[nt][2] * a.scale_log2 : -INFINITY;
      s[nt][3] = v_hi ? s[nt][3] * a.scale_log2 : -INFINITY;
      float mx[2] = {fmaxf(s[nt][0], s[nt][2]), fmaxf(s[nt][1], s[nt][3])};
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        mx[cc] = fmaxf(mx[cc], __shfl_xor_sync(0xFFFFFFFFu, mx[cc], 4));
        mx[cc] = fmaxf(mx[cc], __shfl_xor_sync(0xFFFFFFFFu, mx[cc], 8));
        mx[cc] = fmaxf(mx[cc], __shfl_xor_sync(0xFFFFFFFFu, mx[cc], 16));
      }
      float alpha[2], pr[4];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const float m_new = fmaxf(m_run[nt][cc], mx[cc]);
        if (m_new == -INFINITY) {
          alpha[cc] = 1.f;
          pr[cc] = 0.f;
          pr[cc + 2] = 0.f;
        } else {
          alpha[cc] = exp2f(m_run[nt][cc] - m_new);
          pr[cc] = exp2f(s[nt][cc] - m_new);
          pr[cc + 2] = exp2f(s[nt][cc + 2] - m_new);
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
      // P = P_hi + P_lo, both bf16: the P.V product keeps ~16 significant bits of P
      const uint32_t h01 = pack_bf16x2(pr[0], pr[1]), h23 = pack_bf16x2(pr[2], pr[3]);
      const uint32_t l01 = pack_bf16x2(pr[0] - bf16_lo(h01), pr[1] - bf16_hi(h01));
      const uint32_t l23 = pack_bf16x2(pr[2] - bf16_lo(h23), pr[3] - bf16_hi(h23));
      pb[nt][0] = movmatrix_trans(h01);  // positions 0-7
      pb[nt][1] = movmatrix_trans(h23);  // positions 8-15
      pb[nt][2] = movmatrix_trans(l01);
      pb[nt][3] = movmatrix_trans(l23);
    }
    // O^T[128 dims x 8 heads] += V_sel^T[128 x 16] * P^T[16 x 8]
    {
      const int pos = sub * 16 + (lane & 7) + (lane >> 4) * 8;
      const uint8_t* rowp = vst + pos * ROWB;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int ch = g * 16 + mt * 2 + ((lane >> 3) & 1);
        uint32_t vf[4];
        ldmatrix_x4_trans(smem_u32(rowp + ((ch ^ (pos & 7)) << 4)), vf);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_bf16_16816(o[nt][mt], vf, pb[nt][0], pb[nt][1]);
          mma_bf16_16816(o[nt][mt], vf, pb[nt][2], pb[nt][3]);
        }
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- merge the warps of each KV head through shared memory
  constexpr int HPW = NT * 8;  // head slots per warp
  float* red_o = reinterpret_cast<float*>(smem);               // [8 warps][HPW][128]
  float* red_m = red_o + 8 * HPW * kHeadDim;                    // [8][HPW]
  float* red_l = red_m + 8 * HPW;                               // [8][HPW]
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
