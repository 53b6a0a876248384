/*
 * route.cu -- router top-k and gates.
 *
 * Page "Expert Parallelism" (learning-materials IX.05) §1: each token is routed
 * to k of the E experts; §4: the router's output names, per token, the experts
 * it goes to. One warp per token: lane l holds the logits of experts l, l+32, ...
 * (coalesced 128-byte loads) as order-preserving 32-bit keys; each of k rounds
 * takes the warp's largest key with one redux.sync max and the lowest expert
 * holding it with one redux.sync min, so the experts come out in descending
 * logit order with ties to the lower index. The gates are the softmax over the
 * k selected logits.
 *
 * Bytes per token: E*4 read + k*8 written; bandwidth-bound at large T.
 */
#include <math.h>

#include "moe_device.cuh"

namespace moe {

namespace {

/* Unsigned key of a (non-NaN) logit: key(a) > key(b) iff a > b, and key(a) ==
 * key(b) iff a == b under IEEE compare (-0.0 is folded onto +0.0 first). Sign-
 * magnitude floats become monotone unsigned integers by flipping every bit of a
 * negative value and only the sign bit of a positive one. The smallest key a
 * logit can take is key(-inf) = 0x007FFFFF, so 0 marks a slot that cannot be
 * selected (already taken, or past the last expert). */
__device__ __forceinline__ uint32_t logit_key(float l) {
  uint32_t u = __float_as_uint(l);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

/* The logit of a key (inverse of logit_key; -0.0 comes back as +0.0). */
__device__ __forceinline__ float key_logit(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

template <int NV>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits, int32_t* __restrict__ topk_idx,
                                                    float* __restrict__ topk_gate, int64_t T, int E, int k,
                                                    uint32_t* status) {
  pdl_wait(); /* the logits may come from the kernel just before this one */
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  bool saw_nan = false;
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
    const float* row = logits + t * E;
    uint32_t key[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      key[i] = 0u; /* not an expert: never selectable */
      if (e < E) {
        float l = __ldg(row + e);
        if (isnan(l)) {
          saw_nan = true;
          l = -INFINITY;
        }
        key[i] = logit_key(l);
      }
    }
    uint32_t my_key = 0u;
    uint32_t my_e = 0u;
    for (int j = 0; j < k; ++j) {
      uint32_t m = key[0];
#pragma unroll
      for (int i = 1; i < NV; ++i) m = max(m, key[i]);
      const uint32_t best = __reduce_max_sync(0xFFFFFFFFu, m);
      /* this lane's lowest expert holding the best key (slots ascend in expert) */
      uint32_t cand = 0xFFFFFFFFu;
#pragma unroll
      for (int i = NV - 1; i >= 0; --i)
        if (key[i] == best) cand = (uint32_t)(lane + 32 * i);
      const uint32_t be = __reduce_min_sync(0xFFFFFFFFu, cand);
#pragma unroll
      for (int i = 0; i < NV; ++i)
        if ((uint32_t)(lane + 32 * i) == be) key[i] = 0u;
      if (lane == j) {
        my_key = best;
        my_e = be;
      }
    }
    const float my_v = key_logit(my_key); /* meaningful on lanes < k only */
    /* gates: softmax over the selected logits, relative to the largest */
    const float l0 = __shfl_sync(0xFFFFFFFFu, my_v, 0);
    float ex = 0.0f;
    if (lane < k) ex = (l0 == -INFINITY) ? 1.0f : expf(my_v - l0);
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
    if (lane < k) {
      topk_idx[t * k + lane] = (int32_t)my_e;
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
#define MOE_ROUTE_CASE(N)                                                                                      \
  case N:                                                                                                      \
    return launch_kernel(route_kernel<N>, dim3((unsigned)blocks), dim3(threads), 0, stream, 1, logits, topk_idx, \
                         topk_gate, T, E, k, status);
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
}

}  // namespace moe
