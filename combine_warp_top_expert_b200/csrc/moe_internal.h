/*
 * moe_internal.h -- host-side internals shared by the translation units of
 * libmoe_b200.so: workspace layout and kernel launchers. Not part of the ABI.
 */
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "moe.h" /* include/ is on the include path */

namespace moe {

constexpr int kMaxE = 256;
constexpr int kMaxK = 8;
constexpr int kHPadRows = 256;        /* h rows of each expert group are padded to a multiple of this */
constexpr int kGemmAuto = 0;          /* grouped GEMM: tile shape chosen per GEMM from the shape */
constexpr int kGemmSingle = 1;        /* grouped GEMM: single-CTA 128-row tiles only */
constexpr int kGemmPair = 2;          /* grouped GEMM: CTA-pair 256-row tiles wherever they apply */
constexpr int kChunkAssign = 2048;    /* assignments per dispatch histogram chunk */
constexpr uint64_t kDefaultWaitNs = 2000000000ull; /* bounded-wait limit of the GEMM pipeline */
constexpr size_t kTicketOffset = 64; /* uint32 in the workspace header: dispatch's last-chunk ticket */
constexpr size_t kGemm1CtrOffset = 128; /* 2 x uint32 in the header: gate/up tile counter, finished CTAs */
constexpr size_t kGemm2CtrOffset = 136; /* 2 x uint32 in the header: down tile counter, finished CTAs */
/* expert-parallel signal slots (flag arrays of MOE_EP_SLOTS x R per rank) */
constexpr int kEpSlotCounts = 0, kEpSlotRows = 1, kEpSlotOutputs = 2, kEpSlotDone = 3, kEpSlots = 4;

/* Work split of the row-copy kernels (permute, combine): one warp per (token,
 * slice of `vps` 16-byte vectors), `blocks` CTAs of 8 warps (grid-stride). */
struct RowSlices {
  int slices = 1;
  int vps = 32;
  int blocks = 1;
};
RowSlices row_slices(int64_t T, int d);

/* CTAs of `kernel` (block of `threads`, no dynamic shared memory) that fit on the
 * current device at once: SMs x resident blocks per SM (cached per device and kernel). */
int resident_blocks(const void* kernel, int threads);

/* Dispatch path (see moe_set_dispatch_path). */
constexpr int kDispatchAuto = 0;     /* one pass when A <= kOnePassAutoMaxA, else two kernels */
constexpr int kDispatchTwoPass = 1;  /* histogram/scan kernel, then the permute kernel */
constexpr int kDispatchOnePass = 2;  /* one kernel wherever a CTA's assignments fit its shared memory */
constexpr int64_t kOnePassAutoMaxA = 16384;
int dispatch_path();

/* Launch shape of the one-pass dispatch (use = false: the two-kernel path runs). */
struct OnePass {
  bool use = false;
  int blocks = 0;
  int64_t ipc = 0; /* (token, slice) items per CTA, contiguous */
  int slices = 1;
  int vps = 32;
};
OnePass onepass_plan(const moe_shape_t& s, bool index_only);

/* Byte offsets into the caller's workspace (all 256-byte aligned). */
struct WsLayout {
  size_t status = 0;      /* uint32 device status word (first 256 bytes) */
  size_t chunk = 0;       /* int32 [C][E]: per-chunk expert counts, then chunk base rows */
  size_t local_rank = 0;  /* int32 [A]: rank of an assignment among its chunk's same-expert ones */
  size_t dispatch_end = 0; /* end of what the dispatch kernels use: header, chunk counts, local ranks */
  size_t ep = 0;          /* int32 scratch of the expert-parallel calls (plan, local scan outputs) */
  size_t fc_cnt = 0;      /* uint32 [T][d/64]: combine counters of GEMM2 with the combine folded in */
  size_t h = 0;           /* bf16 [h_rows][f]: SwiGLU hidden rows, 128-row padded per expert */
  size_t total = 0;
  int64_t A = 0;          /* T * k */
  int64_t tok_per_chunk = 1;
  int64_t n_chunks = 0;
  int64_t mt_routed_max = 0; /* upper bound of sum_e ceil(count_e / 256) */
  int64_t h_rows = 0;
};

WsLayout ws_layout(const moe_shape_t& s);

/* Where the expert-parallel dispatch stores rows (see ep.cu). */
struct EpTarget {
  uint16_t* const* dst_rows = nullptr; /* [R] receive buffers (device pointers, peer-mapped) */
  const int32_t* row_base = nullptr;   /* [E] first row, on the owner, of this rank's rows of expert e */
  const int32_t* keep = nullptr;       /* [E] this rank's assignments to e that are kept */
  int experts_per_rank = 1;
  int64_t rows_cap = 0;                /* rows each receive buffer holds */
};

/* Host-side shape validation shared by every entry point. */
moe_status_t validate_shape(const moe_shape_t* s);

/* Record a CUDA error for moe_last_cuda_error() and return MOE_ERR_CUDA. */
moe_status_t cuda_fail(cudaError_t e);

/* Device SM count of the current device (cached). */
int num_sms();

uint64_t wait_timeout_ns();

/* Tile-shape policy of the grouped GEMM (kGemmAuto, kGemmSingle or kGemmPair). */
int gemm_policy();

/* Test hook: grouped-GEMM producers leave their first stage unloaded (see moe_set_test_stall). */
bool test_stall();

/* MOE_DEBUG set in the environment: launch configuration notes on stderr. */
bool debug_log();

/* Launches carry programmatic stream serialization (see moe_set_pdl). */
bool pdl_enabled();

/* Count one successful kernel launch (see moe_kernel_launches). */
void count_launch();

/* Launch `kernel` on `stream`, with programmatic stream serialization when
 * pdl_enabled() (the kernel keeps the pdl_wait / pdl_trigger protocol of
 * moe_device.cuh), and an optional cluster of `cluster_x` CTAs. */
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e == cudaSuccess) count_launch();
  return e;
}

cudaError_t launch_route(const float* logits, int32_t* topk_idx, float* topk_gate, int64_t T, int E, int k,
                         uint32_t* status, cudaStream_t stream);

/* fc_out non-null: a GEMM2 with the combine folded in follows (zero its counters, and
 * the output rows of tokens none of whose rows will arrive). early_x: x is written by
 * nothing after the kernel before this call's first one (inside moe_layer: the router
 * follows x's producer), so the one-pass kernel may load rows of x before its pdl_wait. */
cudaError_t launch_dispatch(const moe_shape_t& s, const WsLayout& L, uint8_t* ws, const uint16_t* x,
                            const int32_t* topk_idx, int32_t* expert_counts, int32_t* expert_offsets,
                            int32_t* rank_counts, int32_t* rank_offsets, int32_t* row_src, int32_t* assign_row,
                            uint16_t* x_perm, float* imbalance, cudaStream_t stream, uint16_t* fc_out = nullptr,
                            bool early_x = false);

/* The combine folded into GEMM2's epilogue for moe_layer (see moe_set_fused_combine). */
bool fused_combine_enabled();

/* Histogram and scan of dispatch only (no permute), with or without the capacity. */
cudaError_t launch_dispatch_count(const moe_shape_t& s, const WsLayout& L, uint8_t* ws, const int32_t* topk_idx,
                                  int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                                  int32_t* rank_offsets, float* imbalance, bool apply_capacity, cudaStream_t stream);

/* Expert-parallel dispatch: rows of x to the owners' receive buffers (after
 * launch_dispatch_count without capacity and launch_ep_plan). send_row[a] = row on
 * the owner, -1 if dropped. */
cudaError_t launch_ep_scatter(const moe_shape_t& s, const WsLayout& L, uint8_t* ws, const uint16_t* x,
                              const int32_t* topk_idx, const EpTarget& ep, int32_t* send_row, cudaStream_t stream);

cudaError_t launch_ep_counts(const int32_t* counts, int32_t* const* tables, uint64_t* const* peer_flags, int R, int E,
                             int me, uint64_t epoch, cudaStream_t stream);
cudaError_t launch_ep_plan(int32_t* const* tables, int R, int E, int me, int32_t cap, int32_t* row_base,
                           int32_t* keep, int32_t* recv_offsets, uint32_t* status, cudaStream_t stream);
cudaError_t launch_ep_signal(uint64_t* const* peer_flags, int R, int me, int slot, uint64_t epoch,
                             cudaStream_t stream);
cudaError_t launch_ep_wait(uint64_t* const* peer_flags, int R, int me, int slot, uint64_t epoch, uint32_t* status,
                           cudaStream_t stream);

/* Expert-parallel combine: the k rows of each token are read from the owners'
 * output buffers (y_rows[R], peer-mapped) at send_row. */
cudaError_t launch_ep_combine(const moe_shape_t& s, uint16_t* const* y_rows, int experts_per_rank, int64_t rows_cap,
                              const int32_t* send_row, const int32_t* topk_idx, const float* topk_gate,
                              const uint16_t* y_shared, uint16_t* out, uint32_t* status, cudaStream_t stream);

/* GEMM1: h (workspace) = silu(A W_gate^T) * (A W_up^T) per expert group; A is
 * x_perm, or (x_perm null) the rows of x gathered through row_src */
cudaError_t launch_gate_up(const moe_shape_t& s, const WsLayout& L, uint8_t* ws, const uint16_t* x_perm,
                           const int32_t* row_src, const int32_t* expert_offsets, const uint16_t* w13,
                           const uint16_t* x, const uint16_t* w13s, cudaStream_t stream);

/* The combine folded into GEMM2's epilogue (see launch_down). */
struct FusedCombine {
  const int32_t* row_src;
  const int32_t* assign_row;
  const float* topk_gate;
  uint16_t* out;
};

/* GEMM2: y_perm / y_shared = h W2^T per expert group; with fc, also out = the combine
 * of those rows (the workspace's combine counters must be zero: the dispatch of the
 * whole-layer call zeroes them) */
cudaError_t launch_down(const moe_shape_t& s, const WsLayout& L, uint8_t* ws, const int32_t* expert_offsets,
                        const uint16_t* w2, const uint16_t* w2s, uint16_t* y_perm, uint16_t* y_shared,
                        cudaStream_t stream, const FusedCombine* fc = nullptr);

/* early_index_reads: the combine kernel may read assign_row and topk_gate before
 * its pdl_wait (only when they come from kernels before its predecessor, as inside
 * moe_layer; a standalone call waits first). */
cudaError_t launch_combine(const moe_shape_t& s, const uint16_t* y_perm, const int32_t* assign_row,
                           const float* topk_gate, const uint16_t* y_shared, uint16_t* out, uint32_t* status,
                           cudaStream_t stream, bool early_index_reads = false);

}  // namespace moe
