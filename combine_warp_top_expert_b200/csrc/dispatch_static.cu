/*
 * dispatch_static.cu -- moe_dispatch_static: the dispatch step for callers that
 * cannot allocate device memory.
 *
 * Some callers have no way to hand this library a workspace: an inference-engine
 * plugin or a serving runtime whose device memory is planned up front and owned
 * by its own arena, or a C/FFI caller with no CUDA allocator of its own. For
 * them cudaMalloc on the hot path is either not permitted or too costly (it can
 * synchronise the device). This entry point runs exactly the same kernels as
 * moe_dispatch, but the kernels' scratch memory (the status word, per-chunk
 * expert counts and in-chunk ranks) lives in one fixed array compiled into the
 * library instead of in a caller-provided workspace.
 *
 * The array is a file-scope __device__ variable of kStaticScratchBytes (1 MiB):
 * every GPU on which the library is loaded holds it until the process exits.
 * Its device address is looked up once per device (cudaGetSymbolAddress, with
 * that device current) on the first call made on that device; host code must
 * not use the variable's name as a device address.
 */
#include <mutex>

#include "moe_internal.h"

namespace moe {

namespace {

constexpr size_t kStaticScratchBytes = size_t(1) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_dispatch_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

/* Device address of the scratch array on the current device (looked up once per device). */
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dispatch_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_dispatch_static(const moe_shape_t* shape, const moe_bf16_t* x, const int32_t* topk_idx,
                                            int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                                            int32_t* rank_offsets, int32_t* row_src, int32_t* assign_row,
                                            moe_bf16_t* x_perm, float* imbalance, uint32_t* status, void* stream) {
  const moe_status_t st = validate_shape(shape);
  if (st != MOE_OK) return st;
  if (!expert_counts || !expert_offsets || !rank_counts || !rank_offsets || !imbalance) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!x || !topk_idx || !row_src || !assign_row || !x_perm)) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(x_perm) & 15)))
    return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*shape);
  /* the dispatch kernels use the layout's prefix [0, L.h): status, chunk counts, local ranks */
  if (L.h > kStaticScratchBytes) return MOE_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e == cudaSuccess) e = cudaMemsetAsync(static_cast<uint8_t*>(scratch) + L.status, 0, sizeof(uint32_t),
                                            (cudaStream_t)stream);
  if (e == cudaSuccess)
    e = launch_dispatch(*shape, L, static_cast<uint8_t*>(scratch), x, topk_idx, expert_counts, expert_offsets,
                        rank_counts, rank_offsets, row_src, assign_row, x_perm, imbalance, (cudaStream_t)stream);
  if (e == cudaSuccess && status)
    e = cudaMemcpyAsync(status, static_cast<uint8_t*>(scratch) + L.status, sizeof(uint32_t),
                        cudaMemcpyDeviceToDevice, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}
