/*
 * moe_synth/synth.cu -- host and device fills for the synthetic inputs defined
 * in synth.h. The host fills run on the CPU (OpenMP); the device fills are one
 * grid-stride kernel each. Both evaluate the same per-element function, so a
 * tensor filled on the GPU equals, bit for bit, the same tensor filled on the
 * host. Test and benchmark infrastructure: no MoE arithmetic lives here.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>
#include "synth.h"

/* element value of a "normal" tensor: float(ih4) * c, rounded to bf16 */
static __host__ __device__ __forceinline__ uint16_t synth_normal_bf16(uint64_t key, uint64_t i, float c) {
  const float s = (float)synth_ih4(synth_bits(key, i));
#if defined(__CUDA_ARCH__)
  return synth_f32_to_bf16(__fmul_rn(s, c));
#else
  return synth_f32_to_bf16(s * c);
#endif
}

static __host__ __device__ __forceinline__ float synth_logit(uint64_t key, uint64_t i, float c, float bias) {
  const float s = (float)synth_ih4(synth_bits(key, i));
#if defined(__CUDA_ARCH__)
  return __fadd_rn(__fmul_rn(s, c), bias);
#else
  volatile float prod = s * c; /* keep the multiply and the add as two roundings */
  return prod + bias;
#endif
}

__global__ void synth_normal_bf16_kernel(uint16_t* out, uint64_t n, uint64_t key, uint64_t offset, float c) {
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = synth_normal_bf16(key, offset + i, c);
}

__global__ void synth_logits_kernel(float* out, uint64_t rows, uint32_t cols, uint64_t key, uint64_t row0, float c,
                                    const float* bias) {
  const uint64_t n = rows * cols;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const uint32_t col = (uint32_t)(i % cols);
    out[i] = synth_logit(key, row0 * cols + i, c, bias ? bias[col] : 0.0f);
  }
}

static int synth_grid(uint64_t n) {
  uint64_t blocks = (n + 255) / 256;
  if (blocks > 148ull * 32ull) blocks = 148ull * 32ull;
  if (blocks < 1) blocks = 1;
  return (int)blocks;
}

extern "C" {

uint64_t synth_bits_at(uint64_t seed, uint32_t tensor_id, uint64_t i) {
  return synth_bits(synth_key(seed, tensor_id), i);
}

/* out[i] = bf16(float(ih4(seed, tensor_id, offset + i)) * c), i < n, on the host */
int synth_fill_normal_bf16_host(uint16_t* out, uint64_t n, uint64_t seed, uint32_t tensor_id, uint64_t offset,
                                float c) {
  if (!out && n) return 1;
  const uint64_t key = synth_key(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < (int64_t)n; ++i) out[i] = synth_normal_bf16(key, offset + (uint64_t)i, c);
  return 0;
}

/* out[r, e] = float(ih4(seed, tensor_id, (row0 + r) * cols + e)) * c + bias[e], on the host */
int synth_fill_logits_host(float* out, uint64_t rows, uint32_t cols, uint64_t seed, uint32_t tensor_id,
                           uint64_t row0, float c, const float* bias) {
  if ((!out && rows) || cols == 0) return 1;
  const uint64_t key = synth_key(seed, tensor_id);
  const int64_t n = (int64_t)(rows * cols);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    const uint32_t col = (uint32_t)((uint64_t)i % cols);
    out[i] = synth_logit(key, row0 * cols + (uint64_t)i, c, bias ? bias[col] : 0.0f);
  }
  return 0;
}

/* device versions: same values, written by a kernel on `stream` (a cudaStream_t) */
int synth_fill_normal_bf16_device(uint16_t* out, uint64_t n, uint64_t seed, uint32_t tensor_id, uint64_t offset,
                                  float c, void* stream) {
  if (n == 0) return 0;
  if (!out) return 1;
  synth_normal_bf16_kernel<<<synth_grid(n), 256, 0, (cudaStream_t)stream>>>(out, n, synth_key(seed, tensor_id),
                                                                            offset, c);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

int synth_fill_logits_device(float* out, uint64_t rows, uint32_t cols, uint64_t seed, uint32_t tensor_id,
                             uint64_t row0, float c, const float* bias_device, void* stream) {
  if (rows == 0) return 0;
  if (!out || cols == 0) return 1;
  synth_logits_kernel<<<synth_grid(rows * cols), 256, 0, (cudaStream_t)stream>>>(
      out, rows, cols, synth_key(seed, tensor_id), row0, c, bias_device);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

} /* extern "C" */
