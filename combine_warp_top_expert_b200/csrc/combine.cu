/*
 * combine.cu -- un-permute and top-k gate-weighted sum.
 *
 * Page "Expert Parallelism" (learning-materials IX.05) §4 COMBINE: expert
 * outputs go back to where their tokens came from, in the original token order,
 * and each token's k outputs are summed with its gate weights. One warp per (token, column slice): the k row
 * indices and gates are loaded by lanes 0..k-1 and broadcast by shuffle; each
 * lane then streams 16-byte vectors of the k expert rows (+ the shared-expert
 * row), accumulates in fp32 in j order and stores one bf16 vector. Slices keep
 * every SM busy when T is small. The expert-parallel form reads each expert row
 * from the GPU that computed it (peer loads over NVLink): the return trip of the
 * page's COMBINE step fused into the weighted sum.
 *
 * Bytes per token: k*d*2 + (shared) d*2 read, d*2 written, k*8 of indices.
 */
#include <algorithm>

#include "moe_device.cuh"

namespace moe {

namespace {

/* Where the expert-parallel combine reads rows (EP form): the output buffers of the
 * R ranks (peer-mapped device pointers); a token's row j sits in the buffer of the
 * rank owning expert topk_idx[t, j] (experts_per_rank per rank), at assign_row. */
struct EpSource {
  uint16_t* const* y_rows = nullptr;
  const int32_t* topk_idx = nullptr;
  int experts_per_rank = 1;
};

/* U vectors per lane per step, rows of up to KMAX experts in flight together.
 * Local form: rows come from y_perm (A rows). EP form: from the owners' buffers
 * (ep; A is then the rows each of them holds). SH: a shared-expert row is added
 * (y_shared non-null); without it the kernel holds fewer registers. */
template <int U, int KMAX, bool EP, bool SH>
__global__ void __launch_bounds__(256, 2) combine_kernel(const uint16_t* __restrict__ y_perm,
                                                      const int32_t* __restrict__ assign_row,
                                                      const float* __restrict__ topk_gate,
                                                      const uint16_t* __restrict__ y_shared,
                                                      uint16_t* __restrict__ out, int64_t T, int d, int k,
                                                      int64_t A, int slices, int vps, uint32_t* status,
                                                      int early_index_reads, const EpSource ep) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int nv = d >> 3;
  const int64_t items = T * slices;
  bool bad = false;
  const int64_t w0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  int row = -1, owner = 0;
  float g = 0.0f;
  auto load_index = [&](int64_t w) {
    const int64_t t = w / slices;
    row = -1;
    g = 0.0f;
    if (lane < k) {
      row = __ldg(assign_row + t * k + lane);
      g = __ldg(topk_gate + t * k + lane);
      if (EP) owner = __ldg(ep.topk_idx + t * k + lane) / ep.experts_per_rank;
    }
  };
  /* inside the whole-layer call the indices and gates come from kernels before the
   * down GEMM that this kernel follows: the first item's are read before pdl_wait */
  if (early_index_reads && w0 < items) load_index(w0);
  pdl_wait(); /* y_perm and y_shared come from the down GEMM */
  pdl_trigger();
  for (int64_t w = w0; w < items; w += warps) {
    const int64_t t = w / slices;
    const int sl = (int)(w - t * slices);
    const int v_end = min(nv, (sl + 1) * vps);
    if (!(early_index_reads && w == w0)) load_index(w);
    if (lane < k && row >= A) {
      bad = true;
      row = -1;
    }
    const uint16_t* src[KMAX];
    float gs[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      const int r = __shfl_sync(0xFFFFFFFFu, row, j);
      const int o = __shfl_sync(0xFFFFFFFFu, owner, j);
      gs[j] = __shfl_sync(0xFFFFFFFFu, g, j);
      const uint16_t* base = EP ? ep.y_rows[o] : y_perm;
      src[j] = (j < k && r >= 0) ? base + (int64_t)r * d : nullptr;
    }
    const uint16_t* ysh = SH ? y_shared + t * d : nullptr;
    uint16_t* o = out + t * d;
    for (int v0 = sl * vps + lane; v0 < v_end; v0 += 32 * U) {
      uint4 wv[KMAX][U];
      uint4 sv[SH ? U : 1];
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + 32 * u;
          wv[j][u] = (src[j] != nullptr && v < v_end) ? ld_nc_v4(src[j] + (int64_t)v * 8) : make_uint4(0, 0, 0, 0);
        }
      if (SH) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + 32 * u;
          sv[SH ? u : 0] = v < v_end ? ld_nc_v4(ysh + (int64_t)v * 8) : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          if (src[j] == nullptr) continue;
          const uint32_t ww[4] = {wv[j][u].x, wv[j][u].y, wv[j][u].z, wv[j][u].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[2 * q] = fmaf(gs[j], bf16lo(ww[q]), acc[2 * q]);
            acc[2 * q + 1] = fmaf(gs[j], bf16hi(ww[q]), acc[2 * q + 1]);
          }
        }
        if (SH) {
          const uint4 q4 = sv[SH ? u : 0];
          const uint32_t ss[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[2 * q] += bf16lo(ss[q]);
            acc[2 * q + 1] += bf16hi(ss[q]);
          }
        }
        const int v = v0 + 32 * u;
        if (v < v_end)
          st_v4(o + (int64_t)v * 8, make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                               pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7])));
      }
    }
  }
  if (bad) raise_status(status, MOE_DEV_BOUNDS);
}

}  // namespace

cudaError_t launch_combine(const moe_shape_t& s, const uint16_t* y_perm, const int32_t* assign_row,
                           const float* topk_gate, const uint16_t* y_shared, uint16_t* out, uint32_t* status,
                           cudaStream_t stream, bool early_index_reads) {
  if (s.T == 0) return cudaSuccess;
  const RowSlices rs = row_slices(s.T, s.d);
  const int64_t A = (int64_t)s.T * s.k;
  auto kernel = y_shared ? (s.k <= 2 ? combine_kernel<4, 2, false, true>
                                     : (s.k <= 4 ? combine_kernel<2, 4, false, true> : combine_kernel<1, 8, false, true>))
                         : (s.k <= 2 ? combine_kernel<4, 2, false, false>
                                     : (s.k <= 4 ? combine_kernel<2, 4, false, false> : combine_kernel<1, 8, false, false>));
  /* one wave of CTAs (the warps loop over their items) */
  const int blocks = std::min(rs.blocks, resident_blocks(reinterpret_cast<const void*>(kernel), 256));
  return launch_kernel(kernel, dim3((unsigned)blocks), dim3(256), 0, stream, 1, y_perm, assign_row, topk_gate,
                       y_shared, out, (int64_t)s.T, s.d, s.k, A, rs.slices, rs.vps, status,
                       early_index_reads ? 1 : 0, EpSource{});
}

cudaError_t launch_ep_combine(const moe_shape_t& s, uint16_t* const* y_rows, int experts_per_rank, int64_t rows_cap,
                              const int32_t* send_row, const int32_t* topk_idx, const float* topk_gate,
                              const uint16_t* y_shared, uint16_t* out, uint32_t* status, cudaStream_t stream) {
  if (s.T == 0) return cudaSuccess;
  const RowSlices rs = row_slices(s.T, s.d);
  EpSource ep;
  ep.y_rows = y_rows;
  ep.topk_idx = topk_idx;
  ep.experts_per_rank = experts_per_rank;
  auto kernel = y_shared ? (s.k <= 2 ? combine_kernel<4, 2, true, true>
                                     : (s.k <= 4 ? combine_kernel<2, 4, true, true> : combine_kernel<1, 8, true, true>))
                         : (s.k <= 2 ? combine_kernel<4, 2, true, false>
                                     : (s.k <= 4 ? combine_kernel<2, 4, true, false> : combine_kernel<1, 8, true, false>));
  return launch_kernel(kernel, dim3((unsigned)rs.blocks), dim3(256), 0, stream, 1, (const uint16_t*)nullptr, send_row,
                       topk_gate, y_shared, out, (int64_t)s.T, s.d, s.k, rows_cap, rs.slices, rs.vps, status, 0, ep);
}

}  // namespace moe
