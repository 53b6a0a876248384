/*
 * ep.cu -- expert parallelism across GPUs: the exchange plan, the cross-GPU
 * signals, and the entry points of the expert-parallel layer.
 *
 * Page "Expert Parallelism" (learning-materials IX.05) §1: experts sit on GPUs in
 * contiguous blocks (GPU r holds experts [r*E/R, (r+1)*E/R)); §4 "The All-to-All":
 * DISPATCH counts the tokens per GPU, exchanges the counts and then the token data,
 * so that each GPU holds one contiguous run of rows per expert it owns; COMBINE sends
 * the results back to the GPU each token came from, in the original order; §4 "The
 * communication volume": k * d * bytes per token and direction.
 *
 * On B200 the token exchange is part of the kernels that touch the rows anyway:
 * the dispatch permute stores each row straight into the owning GPU's receive
 * buffer over NVLink (peer stores), and the combine loads each expert output row
 * straight from the owning GPU (peer loads), so the rows cross NVLink once each way
 * and are never staged in a separate send buffer. The per-expert counts go the same
 * way: each rank stores its row of the R x E count table into every rank's copy.
 *
 * Plan (from the all-gathered counts C[s][e] = assignments of source rank s to
 * expert e, before any capacity):
 *   demand D[e] = sum_s C[s][e]; kept K[e] = min(D[e], capacity) (capacity 0 = none);
 *   on the owner o of e, the rows of e start at recv_off_o[e] = sum of K over o's
 *   experts before e, and inside them come source 0's rows, then source 1's, ...,
 *   each in its source's assignment order (so the first `capacity` rows of an
 *   expert in that order are the ones kept);
 *   for source me: P[e] = sum_{s < me} C[s][e]; my p-th assignment to e has global
 *   rank P[e] + p, is kept iff P[e] + p < K[e], and goes to row recv_off_o[e] + P[e] + p
 *   of the owner's receive buffer: row_base[e] = recv_off_o[e] + P[e], and
 *   keep[e] = max(0, K[e] - P[e]) of my assignments to e are kept.
 * The result is exactly the single-GPU layout of the R ranks' batches taken as one
 * batch (rank-major): owner o's receive buffer equals that layout's rows of logical
 * rank o.
 *
 * Signals: each rank owns a flag array in peer-mapped memory, R flags per slot;
 * rank `me` announces a step of call `epoch` to every rank by storing epoch into
 * flag [slot * R + me] of each (release, system scope), and waits until its own
 * flags [slot * R + s] reach epoch for every s (acquire, system scope; bounded).
 */
#include "moe_device.cuh"

namespace moe {

namespace {

constexpr int kPlanThreads = 256;

/* One CTA: the plan of source rank `me` (see the file comment). */
__global__ void __launch_bounds__(kPlanThreads) ep_plan_kernel(int32_t* const* tables, int R, int E, int me,
                                                              int32_t cap, int32_t* __restrict__ row_base,
                                                              int32_t* __restrict__ keep, int32_t* recv_offsets,
                                                              uint32_t* status) {
  __shared__ int32_t s_k[kMaxE];
  pdl_wait(); /* every rank's counts are in the table once the wait kernel before has returned */
  pdl_trigger();
  const int32_t* counts_all = tables[me];
  const int Er = E / R;
  bool bad = false;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int64_t d = 0, p = 0;
    for (int s = 0; s < R; ++s) {
      const int32_t c = __ldg(counts_all + (int64_t)s * E + e);
      if (c < 0) bad = true;
      d += c;
      if (s < me) p += c;
    }
    const int64_t k = d < cap ? d : cap;
    s_k[e] = (int32_t)k;
    keep[e] = (int32_t)(k > p ? k - p : 0);
    row_base[e] = (int32_t)p; /* + the expert's start on its owner, below */
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int first = (e / Er) * Er;
    int32_t off = 0;
    for (int e2 = first; e2 < e; ++e2) off += s_k[e2];
    row_base[e] += off;
    if (e / Er == me) recv_offsets[e - first] = off;
    if (e == first + Er - 1 && e / Er == me) recv_offsets[Er] = off + s_k[e];
  }
  if (bad) raise_status(status, MOE_DEV_COUNT_MISMATCH);
}

/* Store `epoch` into flag [slot * R + me] of every rank (thread r: rank r). The
 * rows this rank's earlier kernels stored into peers' memory were fenced at system
 * scope by the threads that stored them; the release store orders the rest. */
__global__ void ep_signal_kernel(uint64_t* const* __restrict__ peer_flags, int R, int me, int slot, uint64_t epoch) {
  pdl_wait();
  pdl_trigger();
  const int r = threadIdx.x;
  if (r >= R) return;
  uint64_t* f = peer_flags[r] + (int64_t)slot * R + me;
  __threadfence_system();
  asm volatile("st.release.sys.global.u64 [%0], %1;" ::"l"(f), "l"(epoch) : "memory");
}

/* Wait until flags [slot * R + s] >= epoch for every rank s (thread s), bounded by
 * timeout_ns; on expiry raise MOE_DEV_TIMEOUT and return. */
__global__ void ep_wait_kernel(uint64_t* const* peer_flags, int R, int me, int slot, uint64_t epoch,
                               uint64_t timeout_ns, uint32_t* status) {
  pdl_wait();
  pdl_trigger();
  const int s = threadIdx.x;
  if (s < R) {
    const uint64_t* f = peer_flags[me] + (int64_t)slot * R + s;
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
      uint64_t v;
      asm volatile("ld.acquire.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(f) : "memory");
      if (v >= epoch) break;
      if ((it & 63u) == 63u) {
        const uint64_t now = global_ns();
        if (t0 == 0) {
          t0 = now;
        } else if (now - t0 > timeout_ns) {
          raise_status(status, MOE_DEV_TIMEOUT);
          break;
        }
      }
      __nanosleep(64);
    }
  }
  __syncthreads();
}

/* Store this rank's expert counts (demand, no capacity) into row `me` of every
 * rank's count table, then announce them (slot kEpSlotCounts). One CTA. */
__global__ void __launch_bounds__(kPlanThreads) ep_counts_kernel(const int32_t* __restrict__ counts, int32_t* const* tables,
                                                                uint64_t* const* peer_flags, int R, int E, int me,
                                                                uint64_t epoch) {
  pdl_wait(); /* the counts come from the histogram kernel just before this one */
  pdl_trigger();
  for (int i = threadIdx.x; i < R * E; i += blockDim.x) {
    const int r = i / E, e = i - r * E;
    tables[r][(int64_t)me * E + e] = __ldg(counts + e);
  }
  __threadfence_system();
  __syncthreads();
  if (threadIdx.x < R) {
    uint64_t* f = peer_flags[threadIdx.x] + (int64_t)kEpSlotCounts * R + me;
    asm volatile("st.release.sys.global.u64 [%0], %1;" ::"l"(f), "l"(epoch) : "memory");
  }
}

}  // namespace

cudaError_t launch_ep_counts(const int32_t* counts, int32_t* const* tables, uint64_t* const* peer_flags, int R, int E,
                             int me, uint64_t epoch, cudaStream_t stream) {
  return launch_kernel(ep_counts_kernel, dim3(1), dim3(kPlanThreads), 0, stream, 1, counts, tables, peer_flags, R, E, me,
                       epoch);
}

cudaError_t launch_ep_plan(int32_t* const* tables, int R, int E, int me, int32_t cap, int32_t* row_base,
                           int32_t* keep, int32_t* recv_offsets, uint32_t* status, cudaStream_t stream) {
  return launch_kernel(ep_plan_kernel, dim3(1), dim3(kPlanThreads), 0, stream, 1, tables, R, E, me, cap, row_base, keep,
                       recv_offsets, status);
}

cudaError_t launch_ep_signal(uint64_t* const* peer_flags, int R, int me, int slot, uint64_t epoch,
                             cudaStream_t stream) {
  return launch_kernel(ep_signal_kernel, dim3(1), dim3(((unsigned)R + 31) / 32 * 32), 0, stream, 1, peer_flags, R, me,
                       slot, epoch);
}

cudaError_t launch_ep_wait(uint64_t* const* peer_flags, int R, int me, int slot, uint64_t epoch, uint32_t* status,
                           cudaStream_t stream) {
  return launch_kernel(ep_wait_kernel, dim3(1), dim3(((unsigned)R + 31) / 32 * 32), 0, stream, 1, peer_flags, R, me,
                       slot, epoch, wait_timeout_ns(), status);
}

}  // namespace moe

using namespace moe;

namespace {

/* The workspace's expert-parallel scratch (int32 units). */
struct EpScratch {
  int32_t* row_base;
  int32_t* keep;
  int32_t* offsets;
  int32_t* rank_counts;
  int32_t* rank_offsets;
  float* imbalance;
};

EpScratch ep_scratch(uint8_t* ws, const WsLayout& L) {
  int32_t* b = reinterpret_cast<int32_t*>(ws + L.ep);
  EpScratch x;
  x.row_base = b;
  x.keep = b + kMaxE;
  x.offsets = b + 2 * kMaxE;
  x.rank_counts = b + 3 * kMaxE + 1;
  x.rank_offsets = b + 4 * kMaxE + 1;
  x.imbalance = reinterpret_cast<float*>(b + 5 * kMaxE + 2);
  return x;
}

bool peers_ok(const moe_ep_peers_t* p) {
  return p && p->counts && p->recv_rows && p->y_rows && p->flags && p->rows_cap > 0;
}

moe_status_t ep_common(const moe_shape_t* shape, int32_t rank, const moe_ep_peers_t* peers, const void* ws,
                       size_t ws_bytes) {
  moe_status_t st = validate_shape(shape);
  if (st != MOE_OK) return st;
  if (rank < 0 || rank >= shape->R || !peers_ok(peers)) return MOE_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255) || ws_bytes < ws_layout(*shape).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

extern "C" {

moe_status_t moe_ep_exchange_counts(const moe_shape_t* shape, int32_t rank, uint64_t epoch, const int32_t* topk_idx,
                                    int32_t* expert_counts, const moe_ep_peers_t* peers, void* ws, size_t ws_bytes,
                                    void* stream) {
  moe_status_t st = ep_common(shape, rank, peers, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (!expert_counts || (shape->T > 0 && !topk_idx) || epoch == 0) return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*shape);
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* w = (uint8_t*)ws;
  const EpScratch x = ep_scratch(w, L);
  /* demand per expert: the capacity applies to the ranks' rows together, in the plan */
  cudaError_t e = launch_dispatch_count(*shape, L, w, topk_idx, expert_counts, x.offsets, x.rank_counts,
                                        x.rank_offsets, x.imbalance, false, s);
  if (e == cudaSuccess) e = launch_ep_counts(expert_counts, peers->counts, peers->flags, shape->R, shape->E, rank, epoch, s);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status_t moe_ep_dispatch(const moe_shape_t* shape, int32_t rank, uint64_t epoch, const moe_bf16_t* x,
                             const int32_t* topk_idx, int32_t* send_row, int32_t* recv_offsets,
                             const moe_ep_peers_t* peers, void* ws, size_t ws_bytes, void* stream) {
  moe_status_t st = ep_common(shape, rank, peers, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (!recv_offsets || epoch == 0) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!x || !aligned16(x) || !topk_idx || !send_row)) return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*shape);
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* w = (uint8_t*)ws;
  uint32_t* status = reinterpret_cast<uint32_t*>(w + L.status);
  const EpScratch sc = ep_scratch(w, L);
  const int32_t cap = shape->capacity > 0 ? shape->capacity : 0x7FFFFFFF;
  cudaError_t e = launch_ep_wait(peers->flags, shape->R, rank, kEpSlotCounts, epoch, status, s);
  if (e == cudaSuccess)
    e = launch_ep_plan(peers->counts, shape->R, shape->E, rank, cap, sc.row_base, sc.keep, recv_offsets, status, s);
  if (e == cudaSuccess) {
    EpTarget t;
    t.dst_rows = reinterpret_cast<uint16_t* const*>(peers->recv_rows);
    t.row_base = sc.row_base;
    t.keep = sc.keep;
    t.experts_per_rank = shape->E / shape->R;
    t.rows_cap = peers->rows_cap;
    e = launch_ep_scatter(*shape, L, w, x, topk_idx, t, send_row, s);
  }
  if (e == cudaSuccess) e = launch_ep_signal(peers->flags, shape->R, rank, kEpSlotRows, epoch, s);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status_t moe_ep_signal(int32_t R, int32_t rank, int32_t slot, uint64_t epoch, const moe_ep_peers_t* peers,
                           void* stream) {
  if (R < 1 || R > kMaxE || rank < 0 || rank >= R || slot < 0 || slot >= kEpSlots || epoch == 0 || !peers_ok(peers))
    return MOE_ERR_INVALID_ARG;
  const cudaError_t e = launch_ep_signal(peers->flags, R, rank, slot, epoch, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status_t moe_ep_wait(int32_t R, int32_t rank, int32_t slot, uint64_t epoch, const moe_ep_peers_t* peers, void* ws,
                         size_t ws_bytes, void* stream) {
  if (R < 1 || R > kMaxE || rank < 0 || rank >= R || slot < 0 || slot >= kEpSlots || epoch == 0 || !peers_ok(peers))
    return MOE_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255) || ws_bytes < 256) return MOE_ERR_WORKSPACE;
  const cudaError_t e =
      launch_ep_wait(peers->flags, R, rank, slot, epoch, reinterpret_cast<uint32_t*>(ws), (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status_t moe_ep_combine(const moe_shape_t* shape, int32_t rank, uint64_t epoch, const int32_t* send_row,
                            const int32_t* topk_idx, const float* topk_gate, const moe_bf16_t* y_shared,
                            moe_bf16_t* out, const moe_ep_peers_t* peers, void* ws, size_t ws_bytes, void* stream) {
  moe_status_t st = ep_common(shape, rank, peers, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (epoch == 0) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!send_row || !topk_idx || !topk_gate || !out || !aligned16(out))) return MOE_ERR_INVALID_ARG;
  if (y_shared && !aligned16(y_shared)) return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*shape);
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t* status = reinterpret_cast<uint32_t*>((uint8_t*)ws + L.status);
  cudaError_t e = launch_ep_wait(peers->flags, shape->R, rank, kEpSlotOutputs, epoch, status, s);
  if (e == cudaSuccess)
    e = launch_ep_combine(*shape, reinterpret_cast<uint16_t* const*>(peers->y_rows), shape->E / shape->R,
                          peers->rows_cap, send_row, topk_idx, topk_gate, y_shared, out, status, s);
  if (e == cudaSuccess) e = launch_ep_signal(peers->flags, shape->R, rank, kEpSlotDone, epoch, s);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

int32_t moe_ep_plan_host(int32_t R, int32_t E, int32_t rank, int32_t capacity, const int32_t* counts_all,
                         int32_t* row_base, int32_t* keep, int32_t* recv_offsets) {
  if (R < 1 || E < 1 || E > kMaxE || E % R != 0 || rank < 0 || rank >= R || capacity < 0 || !counts_all ||
      !row_base || !keep || !recv_offsets)
    return -1;
  const int Er = E / R;
  const int64_t cap = capacity > 0 ? capacity : INT64_MAX;
  int64_t kept[kMaxE];
  for (int e = 0; e < E; ++e) {
    int64_t d = 0, p = 0;
    for (int s = 0; s < R; ++s) {
      if (counts_all[(int64_t)s * E + e] < 0) return -1;
      d += counts_all[(int64_t)s * E + e];
      if (s < rank) p += counts_all[(int64_t)s * E + e];
    }
    kept[e] = d < cap ? d : cap;
    keep[e] = (int32_t)(kept[e] > p ? kept[e] - p : 0);
    row_base[e] = (int32_t)p;
  }
  for (int o = 0; o < R; ++o) {
    int64_t off = 0;
    for (int e = o * Er; e < (o + 1) * Er; ++e) {
      row_base[e] += (int32_t)off;
      if (o == rank) recv_offsets[e - o * Er] = (int32_t)off;
      off += kept[e];
    }
    if (o == rank) recv_offsets[Er] = (int32_t)off;
  }
  return 0;
}

}  // extern "C"
