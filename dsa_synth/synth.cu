/*
 * synth.cu - host and device fills of the counter-based generator in synth.h.
 *
 * Every fill writes dst[k] = value(seed, tensor, start + k) for k < count, so a
 * host fill of any sub-range reproduces exactly what a device fill of the
 * whole tensor wrote there.  These are input makers for tests and benchmarks;
 * they carry none of the sparse-attention layer's arithmetic.
 */
#include <cuda_runtime.h>
#include <stdint.h>

#include "synth.h"

namespace {

__global__ void fill_bf16_kernel(uint16_t* dst, int64_t count, int family, uint64_t seed,
                                 uint32_t tensor, uint64_t start, float scale) {
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < count; k += stride)
    dst[k] = synth_bf16_elem(family, seed, tensor, start + (uint64_t)k, scale);
}

__global__ void fill_e4m3_grid_kernel(uint8_t* dst, int64_t count, uint64_t seed, uint32_t tensor,
                                      uint64_t start) {
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < count; k += stride)
    dst[k] = synth_grid_e4m3(synth_hash(seed, tensor, start + (uint64_t)k));
}

__global__ void fill_f32_kernel(float* dst, int64_t count, int family, uint64_t seed,
                                uint32_t tensor, uint64_t start, float scale) {
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < count; k += stride) {
    uint64_t i = start + (uint64_t)k;
    float v = 0.f;
    if (family == SYNTH_WEIGHT) v = synth_weight(synth_hash(seed, tensor, i));
    else if (family == SYNTH_GRID) v = synth_grid_value(synth_hash(seed, tensor, i));
    else if (family == SYNTH_NORMAL) v = synth_normal(seed, tensor, i, scale);
    else if (family == SYNTH_ONE) v = scale;
    dst[k] = v;
  }
}

int grid_for(int64_t count) {
  int64_t blocks = (count + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  if (blocks < 1) blocks = 1;
  return (int)blocks;
}

}  // namespace

extern "C" {

/* ---- device fills (asynchronous on stream; return cudaError_t as int) ---- */

int synth_fill_bf16_device(void* dst, int64_t count, int family, uint64_t seed, uint32_t tensor,
                           uint64_t start, float scale, void* stream) {
  if (count <= 0) return 0;
  fill_bf16_kernel<<<grid_for(count), 256, 0, (cudaStream_t)stream>>>(
      (uint16_t*)dst, count, family, seed, tensor, start, scale);
  return (int)cudaGetLastError();
}

int synth_fill_e4m3_grid_device(void* dst, int64_t count, uint64_t seed, uint32_t tensor,
                                uint64_t start, void* stream) {
  if (count <= 0) return 0;
  fill_e4m3_grid_kernel<<<grid_for(count), 256, 0, (cudaStream_t)stream>>>(
      (uint8_t*)dst, count, seed, tensor, start);
  return (int)cudaGetLastError();
}

int synth_fill_f32_device(float* dst, int64_t count, int family, uint64_t seed, uint32_t tensor,
                          uint64_t start, float scale, void* stream) {
  if (count <= 0) return 0;
  fill_f32_kernel<<<grid_for(count), 256, 0, (cudaStream_t)stream>>>(dst, count, family, seed,
                                                                      tensor, start, scale);
  return (int)cudaGetLastError();
}

/* ---- host fills (same values, host memory) ---- */

void synth_fill_bf16_host(uint16_t* dst, int64_t count, int family, uint64_t seed,
                          uint32_t tensor, uint64_t start, float scale) {
  for (int64_t k = 0; k < count; ++k)
    dst[k] = synth_bf16_elem(family, seed, tensor, start + (uint64_t)k, scale);
}

void synth_fill_e4m3_grid_host(uint8_t* dst, int64_t count, uint64_t seed, uint32_t tensor,
                               uint64_t start) {
  for (int64_t k = 0; k < count; ++k)
    dst[k] = synth_grid_e4m3(synth_hash(seed, tensor, start + (uint64_t)k));
}

void synth_fill_f32_host(float* dst, int64_t count, int family, uint64_t seed, uint32_t tensor,
                         uint64_t start, float scale) {
  for (int64_t k = 0; k < count; ++k) {
    uint64_t i = start + (uint64_t)k;
    float v = 0.f;
    if (family == SYNTH_WEIGHT) v = synth_weight(synth_hash(seed, tensor, i));
    else if (family == SYNTH_GRID) v = synth_grid_value(synth_hash(seed, tensor, i));
    else if (family == SYNTH_NORMAL) v = synth_normal(seed, tensor, i, scale);
    else if (family == SYNTH_ONE) v = scale;
    dst[k] = v;
  }
}

/* raw 64-bit draws, for layout decisions (ragged lengths, needle positions) */
void synth_u64_host(uint64_t* dst, int64_t count, uint64_t seed, uint32_t tensor, uint64_t start) {
  for (int64_t k = 0; k < count; ++k) dst[k] = synth_hash(seed, tensor, start + (uint64_t)k);
}

}  // extern "C"
