/*
 * combine.cu -- un-permute and top-k gate-weighted sum.
 *
 * Page "Expert Parallelism" (learning-materials IX.05) §4 COMBINE: "Send the
 * results back to the originating GPUs, in the original order. Weighted-sum the
 * k expert outputs per token." One warp per token: the k row indices and gates
 * are loaded once by lanes 0..k-1 and broadcast by shuffle; each lane then
 * streams 16-byte vectors of the k expert rows (+ the shared-expert row),
 * accumulates in fp32 in j order and stores one bf16 vector.
 *
 * Bytes per token: k*d*2 + (shared) d*2 read, d*2 written, k*8 of indices.
 */
#include "moe_device.cuh"

namespace moe {

namespace {

template <int U>
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ y_perm,
                                                      const int32_t* __restrict__ assign_row,
                                                      const float* __restrict__ topk_gate,
                                                      const uint16_t* __restrict__ y_shared,
                                                      uint16_t* __restrict__ out, int64_t T, int d, int k,
                                                      int64_t A, uint32_t* status) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int nv = d >> 3;
  bool bad = false;
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
    int row = -1;
    float g = 0.0f;
    if (lane < k) {
      row = __ldg(assign_row + t * k + lane);
      g = __ldg(topk_gate + t * k + lane);
      if (row >= A) {
        bad = true;
        row = -1;
      }
    }
    int64_t src[kMaxK];
    float gs[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      const int r = __shfl_sync(0xFFFFFFFFu, row, j);
      gs[j] = __shfl_sync(0xFFFFFFFFu, g, j);
      src[j] = (j < k && r >= 0) ? (int64_t)r * d : -1;
    }
    const uint16_t* ysh = y_shared ? y_shared + t * d : nullptr;
    uint16_t* o = out + t * d;
    for (int v0 = lane; v0 < nv; v0 += 32 * U) {
      float acc[U][8];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[u][q] = 0.0f;
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        if (src[j] < 0) continue;
        uint4 w[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + 32 * u;
          if (v < nv) w[u] = ld_nc_v4(y_perm + src[j] + (int64_t)v * 8);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const uint32_t ww[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[u][2 * q] = fmaf(gs[j], bf16lo(ww[q]), acc[u][2 * q]);
            acc[u][2 * q + 1] = fmaf(gs[j], bf16hi(ww[q]), acc[u][2 * q + 1]);
          }
        }
      }
      if (ysh) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + 32 * u;
          if (v < nv) {
            const uint4 w = ld_nc_v4(ysh + (int64_t)v * 8);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              acc[u][2 * q] += bf16lo(ww[q]);
              acc[u][2 * q + 1] += bf16hi(ww[q]);
            }
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + 32 * u;
        if (v < nv) {
          uint4 r;
          r.x = pack_bf16x2(acc[u][0], acc[u][1]);
          r.y = pack_bf16x2(acc[u][2], acc[u][3]);
          r.z = pack_bf16x2(acc[u][4], acc[u][5]);
          r.w = pack_bf16x2(acc[u][6], acc[u][7]);
          st_v4(o + (int64_t)v * 8, r);
        }
      }
    }
  }
  if (bad) raise_status(status, MOE_DEV_BOUNDS);
}

}  // namespace

cudaError_t launch_combine(const moe_shape_t& s, const uint16_t* y_perm, const int32_t* assign_row,
                           const float* topk_gate, const uint16_t* y_shared, uint16_t* out, uint32_t* status,
                           cudaStream_t stream) {
  if (s.T == 0) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = ((int64_t)s.T + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  combine_kernel<2><<<(unsigned)blocks, threads, 0, stream>>>(y_perm, assign_row, topk_gate, y_shared, out, s.T,
                                                              s.d, s.k, (int64_t)s.T * s.k, status);
  return cudaGetLastError();
}

}  // namespace moe
