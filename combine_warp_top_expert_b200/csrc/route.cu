/*
 * route.cu -- router top-k and gates.
 *
 * Page "Expert Parallelism" (learning-materials IX.05) §1: each token is routed
 * to k of the E experts; §4: the router's output names, per token, the experts
 * it goes to. One warp per token: lane l holds the logits of experts l, l+32, ...
 * (coalesced 128-byte loads), k rounds of a warp-shuffle arg-max select the
 * experts in descending logit order with ties to the lower index, and the gates
 * are the softmax over the k selected logits.
 *
 * Bytes per token: E*4 read + k*8 written; bandwidth-bound at large T.
 */
#include <math.h>

#include "moe_device.cuh"

namespace moe {

namespace {

/* (v, e) ranks before (bv, be): larger logit, or equal logit and lower index.
 * IEEE compare, so -0.0 and +0.0 tie. */
__device__ __forceinline__ bool ranks_before(float v, int e, float bv, int be) {
  return v > bv || (v == bv && e < be);
}

template <int NV>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits, int32_t* __restrict__ topk_idx,
                                                    float* __restrict__ topk_gate, int64_t T, int E, int k,
                                                    uint32_t* status) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  bool saw_nan = false;
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
    const float* row = logits + t * E;
    float v[NV];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      if (e < E) {
        float l = __ldg(row + e);
        if (isnan(l)) {
          saw_nan = true;
          l = -INFINITY;
        }
        v[i] = l;
      } else {
        v[i] = -INFINITY;
        taken |= 1u << i; /* not an expert: never selectable */
      }
    }
    float my_v = -INFINITY;
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int be = 0x7FFFFFFF;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        if (!((taken >> i) & 1u) && ranks_before(v[i], e, bv, be)) {
          bv = v[i];
          be = e;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
        const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, off);
        if (ranks_before(ov, oe, bv, be)) {
          bv = ov;
          be = oe;
        }
      }
      if (lane == (be & 31)) taken |= 1u << (be >> 5);
      if (lane == j) {
        my_v = bv;
        my_e = be;
      }
    }
    /* gates: softmax over the selected logits, relative to the largest */
    const float l0 = __shfl_sync(0xFFFFFFFFu, my_v, 0);
    float ex = 0.0f;
    if (lane < k) ex = (l0 == -INFINITY) ? 1.0f : expf(my_v - l0);
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
    if (lane < k) {
      topk_idx[t * k + lane] = my_e;
      topk_gate[t * k + lane] = ex / sum;
    }
  }
  if (saw_nan) raise_status(status, MOE_DEV_NAN_LOGIT);
}

}  // namespace

cudaError_t launch_route(const float* logits, int32_t* topk_idx, float* topk_gate, int64_t T, int E, int k,
                         uint32_t* status, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t warps_needed = T;
  int64_t blocks = (warps_needed + (threads / 32) - 1) / (threads / 32);
  const int64_t cap = (int64_t)num_sms() * 16;
  if (blocks > cap) blocks = cap;
  const int nv = (E + 31) / 32;
  switch (nv) {
#define MOE_ROUTE_CASE(N) \
  case N:                 \
    route_kernel<N><<<(int)blocks, threads, 0, stream>>>(logits, topk_idx, topk_gate, T, E, k, status); break;
    MOE_ROUTE_CASE(1)
    MOE_ROUTE_CASE(2)
    MOE_ROUTE_CASE(3)
    MOE_ROUTE_CASE(4)
    MOE_ROUTE_CASE(5)
    MOE_ROUTE_CASE(6)
    MOE_ROUTE_CASE(7)
    MOE_ROUTE_CASE(8)
#undef MOE_ROUTE_CASE
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace moe
