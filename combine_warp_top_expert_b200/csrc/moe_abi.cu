/*
 * moe_abi.cu -- the C ABI of libmoe_b200.so (declared in include/moe.h):
 * argument validation, workspace layout, and the launch sequence of each entry
 * point. Every check runs on the host before anything is launched; the library
 * allocates no memory and holds no per-call state.
 */
#include <atomic>
#include <mutex>
#include <vector>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include <nvtx3/nvToolsExt.h>

#include "moe_internal.h"

namespace moe {

/* NVTX range around one ABI call on the host, so that Nsight timelines show which
 * entry point issued which kernels (header-only NVTX: a no-op unless a tool is
 * attached). */
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

namespace {

thread_local char g_last_cuda_error[256] = "";
std::atomic<uint64_t> g_wait_timeout_ns{kDefaultWaitNs};
std::atomic<int> g_gemm_policy{kGemmAuto};
std::atomic<int> g_test_stall{0};
std::atomic<int> g_pdl{1};
std::atomic<int> g_fused_combine{0};
std::atomic<int> g_dispatch_path{kDispatchAuto};
std::atomic<uint64_t> g_launches{0};

}  // namespace

moe_status_t cuda_fail(cudaError_t e) {
  std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return MOE_ERR_CUDA;
}

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

/* GEMM1 gathering rows of x keeps each row's byte offset into x in 32 bits. */
bool gather_fits(const moe_shape_t& s) { return (uint64_t)s.T * (uint64_t)s.d * 2u <= 0xFFFFFFFFull; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

moe_status_t validate_shape(const moe_shape_t* s) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->d < 1 || s->f < 1 || s->E < 1 || s->k < 1 || s->R < 1) return MOE_ERR_INVALID_ARG;
  if (s->k > s->E || s->E % s->R != 0 || (s->n_shared != 0 && s->n_shared != 1)) return MOE_ERR_INVALID_ARG;
  if (s->capacity < 0) return MOE_ERR_INVALID_ARG;
  if (s->E > kMaxE || s->k > kMaxK) return MOE_ERR_UNSUPPORTED;
  if ((int64_t)s->T * s->k > (int64_t(1) << 27)) return MOE_ERR_UNSUPPORTED;
  if (s->d % 128 != 0 || s->f % 128 != 0 || s->d > 65536 || s->f > 65536) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

namespace {

moe_status_t check_ws(const moe_shape_t& s, const void* ws, size_t ws_bytes) {
  if (!ws || !aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < ws_layout(s).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

}  // namespace

WsLayout ws_layout(const moe_shape_t& s) {
  WsLayout L;
  L.A = (int64_t)s.T * s.k;
  L.tok_per_chunk = s.k > 0 ? (kChunkAssign / s.k > 0 ? kChunkAssign / s.k : 1) : 1;
  L.n_chunks = (s.T + L.tok_per_chunk - 1) / L.tok_per_chunk;
  /* sum_e ceil(n_e / 256) <= floor(A / 256) + (number of non-empty experts) */
  L.mt_routed_max = L.A / kHPadRows + (L.A < s.E ? L.A : s.E);
  L.h_rows = (int64_t)kHPadRows * (L.mt_routed_max + (s.n_shared ? (s.T + kHPadRows - 1) / kHPadRows : 0));
  size_t off = 256;
  L.status = 0;
  L.chunk = off;
  off = round_up(off + (size_t)L.n_chunks * s.E * sizeof(int32_t), 256);
  L.local_rank = off;
  off = round_up(off + (size_t)L.A * sizeof(int32_t), 256);
  L.dispatch_end = off;
  L.ep = off; /* row_base[256], keep[256], offsets[257], rank counts[256], rank offsets[257], imbalance[2] */
  off = round_up(off + (size_t)(6 * kMaxE + 4) * sizeof(int32_t), 256);
  L.fc_cnt = off;
  off = round_up(off + (size_t)s.T * (size_t)(s.d / 64) * sizeof(uint32_t), 256);
  L.h = off;
  off = round_up(off + (size_t)L.h_rows * s.f * sizeof(uint16_t), 256);
  L.total = off;
  return L;
}

int num_sms() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) dev = 0;
  const int slot = dev < 64 ? dev : 63;
  int n = cache[slot].load(std::memory_order_relaxed);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[slot].store(n, std::memory_order_relaxed);
  }
  return n;
}

int resident_blocks(const void* kernel, int threads) {
  struct Entry {
    int dev;
    const void* kernel;
    int threads;
    int blocks;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& e : cache)
    if (e.dev == dev && e.kernel == kernel && e.threads == threads) return e.blocks;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int blocks = per_sm * num_sms();
  cache.push_back(Entry{dev, kernel, threads, blocks});
  return blocks;
}

uint64_t wait_timeout_ns() { return g_wait_timeout_ns.load(std::memory_order_relaxed); }

int gemm_policy() { return g_gemm_policy.load(std::memory_order_relaxed); }

bool test_stall() { return g_test_stall.load(std::memory_order_relaxed) != 0; }

bool pdl_enabled() { return g_pdl.load(std::memory_order_relaxed) != 0; }

bool fused_combine_enabled() { return g_fused_combine.load(std::memory_order_relaxed) != 0; }

int dispatch_path() { return g_dispatch_path.load(std::memory_order_relaxed); }

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

bool debug_log() {
  static const bool on = [] {
    const char* v = std::getenv("MOE_DEBUG");
    return v && *v && *v != '0';
  }();
  return on;
}

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_bytes(const moe_shape_t* shape) {
  if (validate_shape(shape) != MOE_OK) return 0;
  return ws_layout(*shape).total;
}

moe_status_t moe_clear_status(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || !aligned(ws, 256) || ws_bytes < 256) return MOE_ERR_WORKSPACE;
  const cudaError_t e = cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream); /* status word and dispatch ticket */
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status_t moe_get_status(const void* ws, size_t ws_bytes, uint32_t* bits, void* stream) {
  if (!bits) return MOE_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < 256) return MOE_ERR_WORKSPACE;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaMemcpy(bits, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status_t moe_route(const moe_shape_t* shape, const float* logits, int32_t* topk_idx, float* topk_gate, void* ws,
                       size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_range("moe_route");
  moe_status_t st = validate_shape(shape);
  if (st != MOE_OK) return st;
  if (shape->T > 0 && (!logits || !topk_idx || !topk_gate)) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(*shape, ws, ws_bytes)) != MOE_OK) return st;
  const WsLayout L = ws_layout(*shape);
  const cudaError_t e = launch_route(logits, topk_idx, topk_gate, shape->T, shape->E, shape->k,
                                     reinterpret_cast<uint32_t*>((uint8_t*)ws + L.status), (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status_t moe_dispatch(const moe_shape_t* shape, const moe_bf16_t* x, const int32_t* topk_idx,
                          int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                          int32_t* rank_offsets, int32_t* row_src, int32_t* assign_row, moe_bf16_t* x_perm,
                          float* imbalance, void* ws, size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_range("moe_dispatch");
  moe_status_t st = validate_shape(shape);
  if (st != MOE_OK) return st;
  if (!expert_counts || !expert_offsets || !rank_counts || !rank_offsets || !imbalance) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!topk_idx || !row_src || !assign_row)) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && x_perm && (!x || !aligned(x, 16) || !aligned(x_perm, 16))) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(*shape, ws, ws_bytes)) != MOE_OK) return st;
  const WsLayout L = ws_layout(*shape);
  const cudaError_t e = launch_dispatch(*shape, L, (uint8_t*)ws, x, topk_idx, expert_counts, expert_offsets,
                                        rank_counts, rank_offsets, row_src, assign_row, x_perm, imbalance,
                                        (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status_t moe_expert_ffn(const moe_shape_t* shape, const moe_bf16_t* x_perm, const int32_t* expert_offsets,
                            const moe_bf16_t* w13, const moe_bf16_t* w2, const moe_bf16_t* x,
                            const moe_bf16_t* w13s, const moe_bf16_t* w2s, moe_bf16_t* y_perm,
                            moe_bf16_t* y_shared, void* ws, size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_range("moe_expert_ffn");
  moe_status_t st = validate_shape(shape);
  if (st != MOE_OK) return st;
  if (!expert_offsets || !w13 || !w2) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!x_perm || !y_perm)) return MOE_ERR_INVALID_ARG;
  if (shape->n_shared && shape->T > 0 && (!x || !w13s || !w2s || !y_shared)) return MOE_ERR_INVALID_ARG;
  if (!aligned(w13, 16) || !aligned(w2, 16) || (x_perm && !aligned(x_perm, 16)) || (y_perm && !aligned(y_perm, 16)))
    return MOE_ERR_INVALID_ARG;
  if (shape->n_shared && ((x && !aligned(x, 16)) || (w13s && !aligned(w13s, 16)) || (w2s && !aligned(w2s, 16)) ||
                          (y_shared && !aligned(y_shared, 16))))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(*shape, ws, ws_bytes)) != MOE_OK) return st;
  const WsLayout L = ws_layout(*shape);
  cudaError_t e =
      launch_gate_up(*shape, L, (uint8_t*)ws, x_perm, nullptr, expert_offsets, w13, x, w13s, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e);
  e = launch_down(*shape, L, (uint8_t*)ws, expert_offsets, w2, w2s, y_perm, shape->n_shared ? y_shared : nullptr,
                  (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status_t moe_expert_gate_up(const moe_shape_t* shape, const moe_bf16_t* x_perm, const int32_t* expert_offsets,
                                const moe_bf16_t* w13, const moe_bf16_t* x, const moe_bf16_t* w13s, void* ws,
                                size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_range("moe_expert_gate_up");
  moe_status_t st = validate_shape(shape);
  if (st != MOE_OK) return st;
  if (!expert_offsets || !w13 || !aligned(w13, 16)) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!x_perm || !aligned(x_perm, 16))) return MOE_ERR_INVALID_ARG;
  if (shape->n_shared && shape->T > 0 && (!x || !w13s || !aligned(x, 16) || !aligned(w13s, 16)))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(*shape, ws, ws_bytes)) != MOE_OK) return st;
  const cudaError_t e = launch_gate_up(*shape, ws_layout(*shape), (uint8_t*)ws, x_perm, nullptr, expert_offsets, w13, x,
                                       w13s, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status_t moe_expert_gate_up_gather(const moe_shape_t* shape, const moe_bf16_t* x, const int32_t* row_src,
                                       const int32_t* expert_offsets, const moe_bf16_t* w13, const moe_bf16_t* w13s,
                                       void* ws, size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_range("moe_expert_gate_up_gather");
  moe_status_t st = validate_shape(shape);
  if (st != MOE_OK) return st;
  if (!expert_offsets || !w13 || !aligned(w13, 16)) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!x || !row_src || !aligned(x, 16))) return MOE_ERR_INVALID_ARG;
  if (shape->n_shared && shape->T > 0 && (!w13s || !aligned(w13s, 16))) return MOE_ERR_INVALID_ARG;
  if (!gather_fits(*shape)) return MOE_ERR_UNSUPPORTED;
  if ((st = check_ws(*shape, ws, ws_bytes)) != MOE_OK) return st;
  const cudaError_t e = launch_gate_up(*shape, ws_layout(*shape), (uint8_t*)ws, nullptr, row_src, expert_offsets, w13,
                                       x, w13s, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status_t moe_expert_down(const moe_shape_t* shape, const int32_t* expert_offsets, const moe_bf16_t* w2,
                             const moe_bf16_t* w2s, moe_bf16_t* y_perm, moe_bf16_t* y_shared, void* ws,
                             size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_range("moe_expert_down");
  moe_status_t st = validate_shape(shape);
  if (st != MOE_OK) return st;
  if (!expert_offsets || !w2 || !aligned(w2, 16)) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!y_perm || !aligned(y_perm, 16))) return MOE_ERR_INVALID_ARG;
  if (shape->n_shared && shape->T > 0 && (!w2s || !y_shared || !aligned(w2s, 16) || !aligned(y_shared, 16)))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(*shape, ws, ws_bytes)) != MOE_OK) return st;
  const cudaError_t e = launch_down(*shape, ws_layout(*shape), (uint8_t*)ws, expert_offsets, w2, w2s, y_perm,
                                    shape->n_shared ? y_shared : nullptr, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status_t moe_combine(const moe_shape_t* shape, const moe_bf16_t* y_perm, const int32_t* assign_row,
                         const float* topk_gate, const moe_bf16_t* y_shared, moe_bf16_t* out, void* ws,
                         size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_range("moe_combine");
  moe_status_t st = validate_shape(shape);
  if (st != MOE_OK) return st;
  if (shape->T > 0 && (!y_perm || !assign_row || !topk_gate || !out)) return MOE_ERR_INVALID_ARG;
  if ((y_perm && !aligned(y_perm, 16)) || (out && !aligned(out, 16)) || (y_shared && !aligned(y_shared, 16)))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(*shape, ws, ws_bytes)) != MOE_OK) return st;
  const WsLayout L = ws_layout(*shape);
  const cudaError_t e = launch_combine(*shape, y_perm, assign_row, topk_gate, y_shared, out,
                                       reinterpret_cast<uint32_t*>((uint8_t*)ws + L.status), (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status_t moe_layer(const moe_shape_t* shape, const moe_layer_buffers_t* b, void* ws, size_t ws_bytes,
                       void* stream) {
  const NvtxRange nvtx_range("moe_layer");
  moe_status_t st = validate_shape(shape);
  if (st != MOE_OK) return st;
  if (!b) return MOE_ERR_INVALID_ARG;
  if (!b->w13 || !b->w2 || !b->expert_counts || !b->expert_offsets || !b->rank_counts || !b->rank_offsets ||
      !b->imbalance)
    return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!b->logits || !b->x || !b->topk_idx || !b->topk_gate || !b->row_src || !b->assign_row ||
                       !b->y_perm || !b->out))
    return MOE_ERR_INVALID_ARG;
  if (shape->n_shared && shape->T > 0 && (!b->w13s || !b->w2s || !b->y_shared)) return MOE_ERR_INVALID_ARG;
  if (!b->x_perm && !gather_fits(*shape)) return MOE_ERR_UNSUPPORTED;
  const void* al[] = {b->x, b->w13, b->w2, b->w13s, b->w2s, b->x_perm, b->y_perm, b->y_shared, b->out};
  for (const void* p : al)
    if (p && !aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(*shape, ws, ws_bytes)) != MOE_OK) return st;
  const WsLayout L = ws_layout(*shape);
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* w = (uint8_t*)ws;
  uint32_t* status = reinterpret_cast<uint32_t*>(w + L.status);
  cudaError_t e = launch_route(b->logits, b->topk_idx, b->topk_gate, shape->T, shape->E, shape->k, status, s);
  if (e != cudaSuccess) return cuda_fail(e);
  const bool fused = fused_combine_enabled();
  e = launch_dispatch(*shape, L, w, b->x, b->topk_idx, b->expert_counts, b->expert_offsets, b->rank_counts,
                      b->rank_offsets, b->row_src, b->assign_row, b->x_perm, b->imbalance, s,
                      fused ? b->out : nullptr, /*early_x=*/true);
  if (e != cudaSuccess) return cuda_fail(e);
  const uint16_t* ysh_in = shape->n_shared ? b->y_shared : nullptr;
  /* x_perm null: dispatch writes indices only and GEMM1 gathers the rows of x itself */
  e = launch_gate_up(*shape, L, w, b->x_perm, b->row_src, b->expert_offsets, b->w13, b->x, b->w13s, s);
  if (e != cudaSuccess) return cuda_fail(e);
  const FusedCombine fc{b->row_src, b->assign_row, b->topk_gate, b->out};
  e = launch_down(*shape, L, w, b->expert_offsets, b->w2, b->w2s, b->y_perm, shape->n_shared ? b->y_shared : nullptr,
                  s, fused ? &fc : nullptr);
  if (e != cudaSuccess) return cuda_fail(e);
  if (fused) return MOE_OK; /* out was written by the down GEMM's epilogue */
  /* combine's predecessor is the down GEMM: assign_row and topk_gate come from earlier kernels */
  e = launch_combine(*shape, b->y_perm, b->assign_row, b->topk_gate, ysh_in, b->out, status, s, true);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

const char* moe_status_string(moe_status_t status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
  }
  return "MOE_ERR_UNKNOWN";
}

const char* moe_last_cuda_error(void) { return g_last_cuda_error; }

int32_t moe_capacity_for(int64_t c_num, int64_t c_den, int32_t T, int32_t k, int32_t E) {
  if (c_num < 1 || c_den < 1 || T < 0 || k < 1 || E < 1) return -1;
  /* ceil(c_num * T * k / (c_den * E)) with no rounding: 128-bit products */
  const unsigned __int128 num = (unsigned __int128)(uint64_t)c_num * (uint64_t)T * (uint64_t)k;
  const unsigned __int128 den = (unsigned __int128)(uint64_t)c_den * (uint64_t)E;
  const unsigned __int128 q = (num + den - 1) / den;
  return q > (unsigned __int128)INT32_MAX ? -1 : (int32_t)q;
}

int moe_set_gemm_policy(int policy) {
  if (policy != kGemmAuto && policy != kGemmSingle && policy != kGemmPair) return -1;
  return g_gemm_policy.exchange(policy, std::memory_order_relaxed);
}

int moe_set_fused_combine(int enable) {
  return g_fused_combine.exchange(enable ? 1 : 0, std::memory_order_relaxed);
}

moe_status_t moe_expert_down_combine(const moe_shape_t* shape, const int32_t* expert_offsets, const moe_bf16_t* w2,
                                     const moe_bf16_t* w2s, const int32_t* row_src, const int32_t* assign_row,
                                     const float* topk_gate, moe_bf16_t* y_perm, moe_bf16_t* y_shared,
                                     moe_bf16_t* out, void* ws, size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_range("moe_expert_down_combine");
  moe_status_t st = validate_shape(shape);
  if (st != MOE_OK) return st;
  if (!expert_offsets || !w2 || !aligned(w2, 16)) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!y_perm || !aligned(y_perm, 16) || !row_src || !assign_row || !topk_gate || !out ||
                       !aligned(out, 16)))
    return MOE_ERR_INVALID_ARG;
  if (shape->n_shared && shape->T > 0 && (!w2s || !y_shared || !aligned(w2s, 16) || !aligned(y_shared, 16)))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(*shape, ws, ws_bytes)) != MOE_OK) return st;
  if (shape->T == 0) return MOE_OK;
  const WsLayout L = ws_layout(*shape);
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* w = (uint8_t*)ws;
  cudaError_t e = cudaMemsetAsync(w + L.fc_cnt, 0, (size_t)shape->T * (shape->d / 64) * sizeof(uint32_t), s);
  /* with a capacity and no shared expert a token may get no row at all: its output is zero */
  if (e == cudaSuccess && shape->capacity > 0 && !shape->n_shared)
    e = cudaMemsetAsync(out, 0, (size_t)shape->T * shape->d * sizeof(uint16_t), s);
  const FusedCombine fc{row_src, assign_row, topk_gate, out};
  if (e == cudaSuccess)
    e = launch_down(*shape, L, w, expert_offsets, w2, w2s, y_perm, shape->n_shared ? y_shared : nullptr, s, &fc);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

int moe_set_pdl(int enable) { return g_pdl.exchange(enable ? 1 : 0, std::memory_order_relaxed); }

uint64_t moe_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

int moe_set_dispatch_path(int path) {
  if (path != kDispatchAuto && path != kDispatchTwoPass && path != kDispatchOnePass) return -1;
  return g_dispatch_path.exchange(path, std::memory_order_relaxed);
}

int moe_set_test_stall(int enable) { return g_test_stall.exchange(enable ? 1 : 0, std::memory_order_relaxed); }

uint64_t moe_set_wait_timeout_ns(uint64_t ns) {
  return g_wait_timeout_ns.exchange(ns ? ns : kDefaultWaitNs, std::memory_order_relaxed);
}

}  // extern "C"
