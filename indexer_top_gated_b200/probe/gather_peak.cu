// gather_peak.cu - measurement kernels for the roofline of the sparse attention's gather.
//
// The attention reads, per selected position, one 256-byte slice (one KV head of one cache
// row) of the K cache and one of the V cache, at positions that are effectively random.
// The rate at which SMs can pull such rows depends on where they live: from L2 when the
// cache fits there (a 64 MiB K+V cache at T = 32768), from HBM otherwise.  These kernels
// read random 256-byte rows of one buffer with the attention's access shape and nothing
// else: a warp takes 32 row indices with one coalesced load, shares them by shuffle, and
// moves two rows (512 contiguous bytes) per instruction in 16-byte pieces per lane.  Their
// rate is the ceiling the attention's gather can reach on that buffer.  Two ways of moving
// the bytes are measured; the better one is the ceiling:
//   - registers: ld.global.nc 16-byte loads, all 16 row pairs of a chunk in flight;
//   - shared memory: cp.async 16-byte copies into a per-warp ring of 2 chunks (8 KiB).
// Row indices are a counter-based hash (splitmix64 finaliser) masked to the buffer's row
// count (a power of two), so every access stays inside the buffer.
#include <cuda_runtime.h>
#include <stdint.h>

#include "dsa_probe.h"

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void fill_rows_kernel(int32_t* idx, uint32_t n_idx, uint32_t row_mask, uint64_t seed) {
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n_idx; i += gridDim.x * blockDim.x)
    idx[i] = (int32_t)(mix64(seed ^ i) & row_mask);
}

// Address of piece lt of row r: 64-bit arithmetic, or (IDX32) a 32-bit index of 16-byte
// units (buffers up to 64 GiB) added to the base.
template <bool IDX32>
__device__ __forceinline__ const uint4* piece(const uint4* buf, int r, int lt) {
  if (IDX32) return buf + ((uint32_t)r * 16u + (uint32_t)lt);
  return buf + (int64_t)r * 16 + lt;
}

// Warp w handles chunks c = 0 .. chunks_per_warp-1, each 32 row indices starting at
// ((w * chunks_per_warp + c) * 32) & idx_mask of idx.
template <bool IDX32>
__global__ void __launch_bounds__(256) gather_regs_kernel(const uint4* __restrict__ buf,
                                                          const int32_t* __restrict__ idx,
                                                          uint32_t idx_mask, int chunks_per_warp,
                                                          uint4* sink) {
  const int lane = threadIdx.x & 31;
  const uint32_t gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lt = lane & 15, lhi = lane >> 4;
  uint4 acc = make_uint4(0u, 0u, 0u, 0u);
  for (int c = 0; c < chunks_per_warp; ++c) {
    const int row = __ldg(idx + (((gw * (uint32_t)chunks_per_warp + c) * 32u + lane) & idx_mask));
    uint4 v[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int r = __shfl_sync(0xFFFFFFFFu, row, 2 * k + lhi);
      v[k] = __ldg(piece<IDX32>(buf, r, lt));
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      acc.x ^= v[k].x;
      acc.y ^= v[k].y;
      acc.z ^= v[k].z;
      acc.w ^= v[k].w;
    }
  }
  if ((acc.x & acc.y & acc.z & acc.w) == 0xFFFFFFFFu) sink[gw * 32 + lane] = acc;  // keeps the loads
}

template <bool IDX32>
__global__ void __launch_bounds__(256) gather_smem_kernel(const uint4* __restrict__ buf,
                                                          const int32_t* __restrict__ idx,
                                                          uint32_t idx_mask, int chunks_per_warp,
                                                          uint4* sink) {
  extern __shared__ uint4 ring[];  // [8 warps][2 chunks][16 row pairs][32 lanes]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t gw = blockIdx.x * (blockDim.x >> 5) + warp;
  const int lt = lane & 15, lhi = lane >> 4;
  uint4* my = ring + (size_t)warp * 2 * 16 * 32;
  auto issue = [&](int c) {
    const int row = __ldg(idx + (((gw * (uint32_t)chunks_per_warp + c) * 32u + lane) & idx_mask));
    uint4* slot = my + (c & 1) * 16 * 32;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int r = __shfl_sync(0xFFFFFFFFu, row, 2 * k + lhi);
      const uint32_t dst = (uint32_t)__cvta_generic_to_shared(slot + k * 32 + lane);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst),
                   "l"(piece<IDX32>(buf, r, lt))
                   : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  uint4 acc = make_uint4(0u, 0u, 0u, 0u);
  issue(0);
  for (int c = 0; c < chunks_per_warp; ++c) {
    if (c + 1 < chunks_per_warp) {
      issue(c + 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncwarp();
    const uint4 v = my[(c & 1) * 16 * 32 + lane];  // one piece per chunk keeps the copies live
    acc.x ^= v.x;
    acc.y ^= v.y;
    acc.z ^= v.z;
    acc.w ^= v.w;
    __syncwarp();
  }
  if ((acc.x & acc.y & acc.z & acc.w) == 0xFFFFFFFFu) sink[gw * 32 + lane] = acc;
}

constexpr size_t kSmemRing = 8 * 2 * 16 * 32 * 16;  // 128 KiB per CTA

}  // namespace

extern "C" {

// Declared and documented in include/dsa_probe.h.
double dsa_probe_gather(const void* buf, uint32_t n_rows, int32_t* idx, uint32_t n_idx,
                        int variant, int blocks, int chunks_per_warp, int reps, void* sink) {
  if (!buf || !idx || !sink || n_rows == 0 || (n_rows & (n_rows - 1)) || n_idx < 32 ||
      (n_idx & (n_idx - 1)) || blocks < 1 || chunks_per_warp < 1 || reps < 1 ||
      variant < 0 || variant > 3 || (variant >= 2 && n_rows > (1u << 28)))
    return 0.0;
  if ((reinterpret_cast<uintptr_t>(buf) & 15) || (reinterpret_cast<uintptr_t>(sink) & 15))
    return 0.0;
  fill_rows_kernel<<<256, 256>>>(idx, n_idx, n_rows - 1, 0x5EEDull);
  if ((variant & 1) &&
      (cudaFuncSetAttribute(gather_smem_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                            (int)kSmemRing) != cudaSuccess ||
       cudaFuncSetAttribute(gather_smem_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                            (int)kSmemRing) != cudaSuccess))
    return 0.0;
  const uint4* b = static_cast<const uint4*>(buf);
  uint4* s = static_cast<uint4*>(sink);
  auto launch = [&]() {
    if (variant == 0)
      gather_regs_kernel<false><<<blocks, 256>>>(b, idx, n_idx - 1, chunks_per_warp, s);
    else if (variant == 1)
      gather_smem_kernel<false><<<blocks, 256, kSmemRing>>>(b, idx, n_idx - 1, chunks_per_warp, s);
    else if (variant == 2)
      gather_regs_kernel<true><<<blocks, 256>>>(b, idx, n_idx - 1, chunks_per_warp, s);
    else
      gather_smem_kernel<true><<<blocks, 256, kSmemRing>>>(b, idx, n_idx - 1, chunks_per_warp, s);
  };
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  double result = 0.0;
  if (cudaEventCreate(&e0) == cudaSuccess && cudaEventCreate(&e1) == cudaSuccess) {
    launch();  // untimed (fills L2 when the buffer fits)
    cudaEventRecord(e0);
    for (int r = 0; r < reps; ++r) launch();
    cudaEventRecord(e1);
    if (cudaEventSynchronize(e1) == cudaSuccess && cudaGetLastError() == cudaSuccess) {
      float ms = 0.f;
      cudaEventElapsedTime(&ms, e0, e1);
      const double bytes = (double)reps * blocks * 8.0 * chunks_per_warp * 32.0 * 256.0;
      if (ms > 0.f) result = bytes / (ms * 1e-3);
    }
  }
  if (e0) cudaEventDestroy(e0);
  if (e1) cudaEventDestroy(e1);
  return result;
}

}  // extern "C"
