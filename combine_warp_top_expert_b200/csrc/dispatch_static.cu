/*
 * dispatch_static.cu -- moe_dispatch_static: the dispatch step for callers that
 * cannot allocate device memory.
 *
 * Some callers have no way to hand this library a workspace: an inference-engine
 * plugin or a serving runtime whose device memory is planned up front and owned
 * by its own arena, or a C/FFI caller with no CUDA allocator of its own. For
 * them cudaMalloc on the hot path is either not permitted or too costly (it can
 * synchronise the device). This entry point runs exactly the same kernels as
 * moe_dispatch, but the kernels' scratch memory (the status word, the last-chunk
 * ticket, per-chunk expert counts and in-chunk ranks) lives in one fixed array
 * compiled into the library instead of in a caller-provided workspace.
 *
 * The array is a file-scope __device__ variable of kStaticScratchBytes (1 MiB):
 * every GPU on which the library is loaded holds it until the process exits.
 * Host code must not use the variable's name as a device address: its device
 * address is looked up with cudaGetSymbolAddress, with the device current, the
 * first time a call runs in a CUDA context, and looked up again if that device's
 * context changes (cudaDeviceReset, or a released and re-created primary
 * context, may load the module at a new address). Contexts are told apart by
 * their unique id (cuCtxGetId), not by their handle, which can be reused.
 * Every call zeroes the array's 256-byte header (status word and ticket) before
 * its kernels run, so a call that was interrupted or raced cannot leave state
 * that a later, properly ordered call would read.
 */
#include <cudaTypedefs.h>

#include <mutex>

#include "moe_internal.h"

namespace moe {

namespace {

constexpr size_t kStaticScratchBytes = size_t(1) << 20;
constexpr size_t kHeaderBytes = 256;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_dispatch_scratch[kStaticScratchBytes];

struct ScratchSlot {
  unsigned long long ctx_id = 0; /* 0: not looked up yet */
  void* addr = nullptr;
};

std::mutex g_scratch_mu;
ScratchSlot g_scratch[kMaxDevices];

PFN_cuCtxGetId_v12000 ctx_id_fn() {
  static PFN_cuCtxGetId_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  return fn;
}

/* Unique id of the CUDA context current on this thread (0 if none is current yet). */
unsigned long long current_ctx_id() {
  auto fn = ctx_id_fn();
  if (!fn) return 0;
  unsigned long long id = 0;
  if (fn(nullptr, &id) != CUDA_SUCCESS) return 0; /* NULL: the current context */
  return id;
}

/* Device address of the scratch array in the current device's context. */
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& slot = g_scratch[dev];
  const unsigned long long id = current_ctx_id();
  if (id == 0 || id != slot.ctx_id || !slot.addr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dispatch_scratch); /* also makes the device's primary context current */
    if (e != cudaSuccess) return e;
    slot.addr = p;
    slot.ctx_id = current_ctx_id();
  }
  *out = slot.addr;
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
  if (shape->T > 0 && (!topk_idx || !row_src || !assign_row)) return MOE_ERR_INVALID_ARG;
  /* x_perm NULL: indices only (x may then be NULL too), as for moe_dispatch */
  if (shape->T > 0 && x_perm &&
      (!x || (reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(x_perm) & 15)))
    return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*shape);
  /* the dispatch kernels use the layout's prefix [0, L.dispatch_end): header, chunk counts, local ranks */
  if (L.dispatch_end > kStaticScratchBytes) return MOE_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e == cudaSuccess) e = cudaMemsetAsync(scratch, 0, kHeaderBytes, (cudaStream_t)stream);
  if (e == cudaSuccess)
    e = launch_dispatch(*shape, L, static_cast<uint8_t*>(scratch), x, topk_idx, expert_counts, expert_offsets,
                        rank_counts, rank_offsets, row_src, assign_row, x_perm, imbalance, (cudaStream_t)stream);
  if (e == cudaSuccess && status)
    e = cudaMemcpyAsync(status, static_cast<uint8_t*>(scratch) + L.status, sizeof(uint32_t),
                        cudaMemcpyDeviceToDevice, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

extern "C" moe_status_t moe_dispatch_static_scratch(void** scratch, size_t* bytes) {
  if (!scratch || !bytes) return MOE_ERR_INVALID_ARG;
  void* p = nullptr;
  const cudaError_t e = scratch_address(&p);
  if (e != cudaSuccess) return cuda_fail(e);
  *scratch = p;
  *bytes = kStaticScratchBytes;
  return MOE_OK;
}
