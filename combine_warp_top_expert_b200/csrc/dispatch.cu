/*
 * dispatch.cu -- per-expert histogram, exclusive scan and stable permute.
 *
 * Page "Expert Parallelism" (learning-materials IX.05) §4 DISPATCH: tokens are
 * ordered by the expert they go to (which orders them by GPU too), the tokens per
 * GPU are counted, and afterwards every GPU holds one contiguous run of tokens
 * per expert it owns; §5: the load of the busiest GPU against the ideal.
 *
 * Assignment a = t*k + j goes to row offsets[e] + (number of earlier
 * assignments to e): a stable counting sort, bit-exact and deterministic (no
 * atomic decides a position). Two kernels:
 *   count   one CTA per chunk of ~2048 assignments: per-warp histograms with
 *           __match_any_sync give each assignment its rank inside the chunk;
 *           the CTA that finishes last (atomic ticket) runs the scan: expert
 *           demand, kept counts (capacity), exclusive scan, per-(chunk, expert)
 *           rank bases, logical-rank counts/offsets and the imbalance ratios;
 *   permute one warp per (token, column slice): writes row_src/assign_row and
 *           copies its slice of the token's row (16-byte vectors, read once)
 *           to the k destinations; slices keep every SM busy at small T.
 * Bytes: T*d*2 read + T*k*d*2 written by the permute, plus ~T*k*16 of indices.
 */
#include "moe_device.cuh"

namespace moe {

namespace {

constexpr int kHistThreads = 512;
constexpr int kHistWarps = kHistThreads / 32;
constexpr int kScanThreads = 512;
constexpr int kOnePassThreads = 512;
constexpr int kOnePassWarps = kOnePassThreads / 32;
constexpr int kOnePassMaxLocal = 1024; /* assignments of one CTA's tokens (rows kept in shared memory) */

/* Exclusive scan of cnt[0..E) into off[0..E] (off[E] = total), run by warp 0 alone:
 * each lane owns a contiguous slice of the experts. */
__device__ void expert_offsets_warp0(const int32_t* cnt, int32_t* off, int E) {
  const int lane = threadIdx.x & 31;
  const int per = (E + 31) / 32;
  const int b = min(E, lane * per), en = min(E, b + per);
  int local = 0;
  for (int i = b; i < en; ++i) local += cnt[i];
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  int run = incl - local;
  for (int i = b; i < en; ++i) {
    off[i] = run;
    run += cnt[i];
  }
  if (lane == 31) off[E] = incl;
}

/* The per-expert and per-rank outputs of dispatch from the kept counts cnt[E] and
 * their offsets off[E+1] (shared memory, complete): expert counts/offsets, logical-rank
 * counts/offsets and the imbalance ratios. Called by every thread of the CTA. */
__device__ void write_dispatch_totals(const int32_t* cnt, const int32_t* off, int E, int R, int32_t* expert_counts,
                                      int32_t* expert_offsets, int32_t* rank_counts, int32_t* rank_offsets,
                                      float* imbalance) {
  __shared__ int32_t s_max[2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int total = off[E];
  for (int e = tid; e < E; e += blockDim.x) {
    expert_counts[e] = cnt[e];
    expert_offsets[e] = off[e];
  }
  if (tid == 0) expert_offsets[E] = total;
  const int per_rank = E / R;
  for (int r = tid; r < R; r += blockDim.x) {
    rank_offsets[r] = off[r * per_rank];
    rank_counts[r] = off[(r + 1) * per_rank] - off[r * per_rank];
  }
  if (tid == 0) rank_offsets[R] = total;
  /* maxima over ranks and experts (warp 0) */
  if (warp == 0) {
    int me = 0, mr = 0;
    for (int i = lane; i < E; i += 32) me = max(me, cnt[i]);
    for (int r = lane; r < R; r += 32) mr = max(mr, off[(r + 1) * per_rank] - off[r * per_rank]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      me = max(me, __shfl_xor_sync(0xFFFFFFFFu, me, o));
      mr = max(mr, __shfl_xor_sync(0xFFFFFFFFu, mr, o));
    }
    if (lane == 0) {
      s_max[0] = mr;
      s_max[1] = me;
    }
  }
  __syncthreads();
  if (tid == 0) {
    /* max / mean = (max * R) / total: exact integers, one correctly rounded
     * double quotient, rounded once to fp32 (exact result for total < 2^28) */
    if (total == 0) {
      imbalance[0] = 1.0f;
      imbalance[1] = 1.0f;
    } else {
      imbalance[0] = (float)((double)((int64_t)s_max[0] * R) / (double)total);
      imbalance[1] = (float)((double)((int64_t)s_max[1] * E) / (double)total);
    }
  }
}

/* Scan over the per-chunk counts (run by one whole CTA of kScanThreads threads):
 * each expert keeps min(demand, cap) rows; offsets over the kept counts; chunk
 * counts -> rank bases (the expert-local rank of each chunk's first assignment,
 * in place); rank counts/offsets, imbalance; row_src beyond the kept total = -1. */
__device__ void scan_chunks(int32_t* chunk, int64_t C, int E, int R, int64_t A, int32_t cap, int32_t* expert_counts,
                            int32_t* expert_offsets, int32_t* rank_counts, int32_t* rank_offsets, float* imbalance,
                            int32_t* row_src) {
  __shared__ int32_t part[kScanThreads]; /* [G][E] partial sums over chunk ranges */
  __shared__ int32_t cnt[kMaxE];
  __shared__ int32_t off[kMaxE + 1];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int G = max(1, kScanThreads / E);
  const int e = tid % E, g = tid / E;
  const bool active = g < G;
  const int64_t c_begin = active ? (C * g) / G : 0, c_end = active ? (C * (g + 1)) / G : 0;
  int32_t s = 0;
  for (int64_t c = c_begin; c < c_end; ++c) s += __ldcg(chunk + c * E + e);
  if (active) part[g * E + e] = s;
  __syncthreads();
  if (tid < E) {
    int run = 0;
    for (int q = 0; q < G; ++q) {
      const int v = part[q * E + tid];
      part[q * E + tid] = run;
      run += v;
    }
    cnt[tid] = min(run, cap); /* kept rows */
  }
  __syncthreads();
  if (warp == 0) expert_offsets_warp0(cnt, off, E);
  __syncthreads();
  const int total = off[E];
  /* chunk rank bases, in place */
  if (active) {
    int32_t base = part[g * E + e];
    for (int64_t c = c_begin; c < c_end; ++c) {
      const int32_t v = __ldcg(chunk + c * E + e);
      chunk[c * E + e] = base;
      base += v;
    }
  }
  write_dispatch_totals(cnt, off, E, R, expert_counts, expert_offsets, rank_counts, rank_offsets, imbalance);
  if (row_src)
    for (int64_t p = total + tid; p < A; p += blockDim.x) row_src[p] = -1;
}

__global__ void __launch_bounds__(kHistThreads) dispatch_count_kernel(
    const int32_t* __restrict__ topk_idx, int64_t A, int E, int R, int32_t cap, int64_t chunk_assign, int64_t n_chunks,
    int32_t* __restrict__ chunk_cnt, int32_t* __restrict__ local_rank, uint32_t* status, uint32_t* ticket,
    int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts, int32_t* rank_offsets, float* imbalance,
    int32_t* row_src) {
  extern __shared__ int32_t sh[];
  __shared__ int s_last;
  int32_t* hist = sh; /* [kHistWarps][E] */
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t a0 = (int64_t)blockIdx.x * chunk_assign;
  const int64_t rem = A - a0;
  const int n = (int)(rem < chunk_assign ? rem : chunk_assign);
  const int per_warp = (n + kHistWarps - 1) / kHistWarps;
  const int w_begin = warp * per_warp, w_end = min(n, (warp + 1) * per_warp);
  for (int i = threadIdx.x; i < kHistWarps * E; i += blockDim.x) hist[i] = 0;
  pdl_wait(); /* topk_idx may come from the kernel just before this one */
  pdl_trigger();
  /* all of this warp's expert ids in flight at once, before the histogram needs them */
  constexpr int kIters = kChunkAssign / (kHistWarps * 32);
  static_assert(kIters * kHistWarps * 32 == kChunkAssign, "a chunk is whole 32-wide steps of every warp");
  int ev[kIters];
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int i = w_begin + it * 32 + lane;
    ev[it] = i < w_end ? __ldg(topk_idx + a0 + i) : -1;
  }
  __syncthreads();

  bool bad = false;
  int rv[kIters]; /* rank of each of this lane's assignments among the warp's earlier ones */
#pragma unroll
  for (int it = 0; it < kIters; ++it) rv[it] = -1;
  int32_t* my_hist = hist + warp * E;
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int i = w_begin + it * 32 + lane;
    if (w_begin + it * 32 >= w_end) break; /* warp-uniform */
    const bool valid = i < w_end;
    int e = valid ? ev[it] : -1;
    if (valid && (e < 0 || e >= E)) {
      bad = true;
      e = -1;
    }
    ev[it] = e; /* -1 for lanes past the end and for skipped entries */
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    int r = -1;
    if (e >= 0) r = my_hist[e] + __popc(peers & ((1u << lane) - 1u));
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) my_hist[e] += __popc(peers);
    __syncwarp();
    rv[it] = r;
  }
  __syncthreads();
  /* per expert: exclusive scan over the warps; chunk total to global */
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kHistWarps; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = run;
      run += c;
    }
    chunk_cnt[(int64_t)blockIdx.x * E + e] = run;
  }
  __syncthreads();
  /* each lane finishes its own assignments: rank inside the chunk = the warp's base
   * for the expert (exclusive scan over the warps) + the rank inside the warp */
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int i = w_begin + it * 32 + lane;
    if (i < w_end) local_rank[a0 + i] = rv[it] >= 0 ? hist[warp * E + ev[it]] + rv[it] : -1;
  }
  if (bad) raise_status(status, MOE_DEV_BOUNDS);

  /* the last chunk to finish scans all chunk counts (a single chunk is its own last one:
   * its counts are visible to the whole CTA after the barrier) */
  if (n_chunks > 1) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(ticket, 1u) == (uint32_t)(n_chunks - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
  } else {
    __syncthreads();
  }
  scan_chunks(chunk_cnt, n_chunks, E, R, A, cap, expert_counts, expert_offsets, rank_counts, rank_offsets, imbalance,
              row_src);
  if (threadIdx.x == 0) *ticket = 0; /* ready for the next call on this workspace */
}

/* Empty batch: zero counts, imbalance {1, 1}. */
__global__ void __launch_bounds__(kScanThreads) dispatch_empty_kernel(int E, int R, int32_t* expert_counts,
                                                                      int32_t* expert_offsets, int32_t* rank_counts,
                                                                      int32_t* rank_offsets, float* imbalance) {
  pdl_wait();
  pdl_trigger();
  scan_chunks(nullptr, 0, E, R, 0, 0x7FFFFFFF, expert_counts, expert_offsets, rank_counts, rank_offsets, imbalance,
              nullptr);
}

/* One-pass dispatch (small batches): histogram, scan and permute in one launch, with
 * no CTA waiting on another. Each CTA owns a contiguous range of (token, slice) items
 * and counts all A expert ids itself (A is small: they are L2-resident after the
 * router), split at its first token: the totals give every expert's kept count and
 * offset, the counts before its range the rank of its first assignment to each
 * expert; warp 0 then ranks the CTA's own assignments in order (the same stable
 * order as the two-kernel path, so the same rows). Every CTA derives the same totals
 * from the same ids; CTA 0 writes them out. The first item's row vectors (U per lane:
 * a whole 256-vector slice at U = 8) are loaded before the counting (before pdl_wait
 * when early_x: x then comes from before the kernel this one follows), so that part
 * of the read overlaps the count. */
template <int U>
__global__ void __launch_bounds__(kOnePassThreads, 1) dispatch_onepass_kernel(
    const uint16_t* __restrict__ x, const int32_t* __restrict__ topk_idx, int64_t T, int d, int E, int R, int k,
    int32_t cap, int64_t ipc, int slices, int vps, int32_t* expert_counts, int32_t* expert_offsets,
    int32_t* rank_counts, int32_t* rank_offsets, float* imbalance, int32_t* __restrict__ row_src,
    int32_t* __restrict__ assign_row, uint16_t* __restrict__ x_perm, uint32_t* status, int early_x) {
  extern __shared__ int32_t sh[];
  int32_t* hpre = sh;                           /* [warps][E]: ids before the CTA's first assignment */
  int32_t* htot = sh + kOnePassWarps * E;       /* [warps][E]: all ids */
  int32_t* s_pos = htot + kOnePassWarps * E;    /* [kOnePassMaxLocal]: rows of the CTA's assignments */
  __shared__ int32_t s_run[kMaxE];
  __shared__ int32_t s_cnt[kMaxE];
  __shared__ int32_t s_off[kMaxE + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t A = T * k;
  const int64_t items = T * slices;
  const int64_t i_lo = (int64_t)blockIdx.x * ipc;
  const int64_t i_hi = min(items, i_lo + ipc);
  const int64_t t_lo = i_lo / slices, t_hi = (i_hi - 1) / slices + 1;
  const int64_t a_lo = t_lo * k, a_hi = t_hi * k;
  const bool move = x_perm != nullptr;
  const int nv = d >> 3;
  for (int i = tid; i < 2 * kOnePassWarps * E; i += blockDim.x) sh[i] = 0;

  uint4 buf[U];
  auto load_item = [&](int64_t w) {
    const int64_t t = w / slices;
    const int sl = (int)(w - t * slices);
    const uint16_t* src = x + t * d;
    const int v_begin = sl * vps + lane, v_end = min(nv, (sl + 1) * vps);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v_begin + 32 * u;
      if (v < v_end) buf[u] = ld_nc_v4(src + (int64_t)v * 8);
    }
  };
  const int64_t w0 = i_lo + warp;
  if (early_x && move && w0 < i_hi) load_item(w0);
  pdl_wait(); /* topk_idx comes from the kernel before */
  pdl_trigger();
  if (!early_x && move && w0 < i_hi) load_item(w0);
  __syncthreads();

  /* 1. per-warp histograms of all ids and of the ids before a_lo (4 loads in flight) */
  bool bad = false;
  int32_t* my_pre = hpre + warp * E;
  int32_t* my_tot = htot + warp * E;
  constexpr int kStep = kOnePassThreads; /* ids per CTA-wide step */
  for (int64_t base = (int64_t)warp * 32; base < A; base += 4 * kStep) {
    int ev[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t a = base + (int64_t)u * kStep + lane;
      ev[u] = a < A ? __ldg(topk_idx + a) : -1;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t a = base + (int64_t)u * kStep + lane;
      int e = ev[u];
      if (a < A && (e < 0 || e >= E)) {
        bad = true;
        e = -1;
      }
      const unsigned before = __ballot_sync(0xFFFFFFFFu, a < a_lo);
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
      if (e >= 0 && lane == __ffs(peers) - 1) {
        my_tot[e] += __popc(peers);
        my_pre[e] += __popc(peers & before);
      }
    }
  }
  __syncthreads();
  /* 2. totals, kept counts, offsets; the rank bases of this CTA */
  for (int e = tid; e < E; e += blockDim.x) {
    int p = 0, t = 0;
#pragma unroll
    for (int w = 0; w < kOnePassWarps; ++w) {
      p += hpre[w * E + e];
      t += htot[w * E + e];
    }
    s_run[e] = p;
    s_cnt[e] = min(t, cap);
  }
  __syncthreads();
  if (warp == 0) expert_offsets_warp0(s_cnt, s_off, E);
  __syncthreads();
  const int total = s_off[E];
  /* 3. warp 0 ranks the CTA's own assignments in order; the CTA holding a token's
   * slice 0 writes its row_src / assign_row entries */
  if (warp == 0) {
    for (int64_t b = a_lo; b < a_hi; b += 32) {
      const int64_t a = b + lane;
      int e = a < a_hi ? __ldg(topk_idx + a) : -1;
      if (e >= E) e = -1;
      if (e < 0) e = -1;
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
      int pos = -1;
      if (e >= 0) {
        const int rank = s_run[e] + __popc(peers & ((1u << lane) - 1u));
        if (rank < cap) {
          const int64_t q = (int64_t)s_off[e] + rank;
          if (q >= 0 && q < A)
            pos = (int)q;
          else
            bad = true;
        }
      }
      __syncwarp();
      if (e >= 0 && lane == __ffs(peers) - 1) s_run[e] += __popc(peers);
      __syncwarp();
      if (a < a_hi) {
        s_pos[a - a_lo] = pos;
        if ((a / k) * slices >= i_lo) {
          assign_row[a] = pos;
          if (pos >= 0) row_src[pos] = (int32_t)a;
        }
      }
    }
  }
  for (int64_t p = total + (int64_t)blockIdx.x * blockDim.x + tid; p < A; p += (int64_t)gridDim.x * blockDim.x)
    row_src[p] = -1;
  if (blockIdx.x == 0)
    write_dispatch_totals(s_cnt, s_off, E, R, expert_counts, expert_offsets, rank_counts, rank_offsets, imbalance);
  __syncthreads();
  /* 4. the permute of this CTA's items */
  if (move) {
    for (int64_t w = w0; w < i_hi; w += kOnePassWarps) {
      const int64_t t = w / slices;
      const int sl = (int)(w - t * slices);
      const uint16_t* src = x + t * d;
      const int v_begin = sl * vps + lane, v_end = min(nv, (sl + 1) * vps);
      if (w != w0) load_item(w);
      const int pos = lane < k ? s_pos[t * k + lane - a_lo] : -1;
      uint16_t* dst[kMaxK];
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        const int p = __shfl_sync(0xFFFFFFFFu, pos, j);
        dst[j] = (j < k && p >= 0) ? x_perm + (int64_t)p * d : nullptr;
      }
      for (int v0 = v_begin; v0 < v_end; v0 += 32 * U) {
        if (v0 != v_begin) {
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int v = v0 + 32 * u;
            if (v < v_end) buf[u] = ld_nc_v4(src + (int64_t)v * 8);
          }
        }
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
          if (dst[j] == nullptr) continue;
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int v = v0 + 32 * u;
            if (v < v_end) st_v4(dst[j] + (int64_t)v * 8, buf[u]);
          }
        }
      }
    }
  }
  if (bad) raise_status(status, MOE_DEV_BOUNDS);
}

/* EP form: rows go to the receive buffer of the rank that owns their expert, at the
 * rows the exchange plan gives (ep.cu); x_perm, row_src and `cap` are not used. */
template <int U, bool EP>
__global__ void __launch_bounds__(256) dispatch_permute_kernel(
    const uint16_t* __restrict__ x, const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ chunk_base,
    const int32_t* __restrict__ local_rank, const int32_t* __restrict__ expert_offsets, int64_t T, int d, int E,
    int k, int32_t cap, int64_t tok_per_chunk, int slices, int vps, int32_t* __restrict__ row_src,
    int32_t* __restrict__ assign_row, uint16_t* __restrict__ x_perm, uint32_t* status, const EpTarget ep,
    uint32_t* __restrict__ fc_cnt, uint16_t* __restrict__ fc_out, int n_shared) {
  const int lane = threadIdx.x & 31;
  const int64_t A = T * k;
  const bool move = EP || x_perm != nullptr; /* false: index-only dispatch */
  bool bad = false;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int nv = d >> 3; /* 16-byte vectors per row */
  const int64_t items = T * slices;
  const int64_t w0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  /* the first row vectors need no index: their loads go out before the index chain.
   * The first item's go out even before pdl_wait: x predates the count kernel that
   * this kernel follows, and that kernel has passed its own wait when this one starts. */
  uint4 buf[U];
  auto load_first = [&](int64_t w) {
    const int64_t t = w / slices;
    const int sl = (int)(w - t * slices);
    const uint16_t* src = x + t * d;
    const int v_begin = sl * vps + lane, v_end = min(nv, (sl + 1) * vps);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v_begin + 32 * u;
      if (v < v_end) buf[u] = ld_nc_v4(src + (int64_t)v * 8);
    }
  };
  if (move && w0 < items) load_first(w0);
  pdl_wait(); /* chunk counts, ranks and offsets (EP: the plan) come from the kernel before */
  pdl_trigger();
  for (int64_t w = w0; w < items; w += warps) {
    const int64_t t = w / slices;
    const int sl = (int)(w - t * slices);
    const uint16_t* src = move ? x + t * d : nullptr;
    const int v_begin = sl * vps + lane, v_end = min(nv, (sl + 1) * vps);
    if (move && w != w0) load_first(w);
    int pos = -1, owner = 0;
    if (lane < k) {
      const int64_t a = t * k + lane;
      const int e = __ldg(topk_idx + a);
      const int lr = __ldg(local_rank + a);
      if (e >= 0 && e < E && lr >= 0) {
        const int rank = __ldg(chunk_base + (t / tok_per_chunk) * E + e) + lr; /* among e's assignments */
        if (EP) {
          if (rank < __ldg(ep.keep + e)) { /* else dropped by the capacity */
            const int64_t q = (int64_t)__ldg(ep.row_base + e) + rank;
            if (rank >= 0 && q >= 0 && q < ep.rows_cap) {
              pos = (int)q;
              owner = e / ep.experts_per_rank;
            } else {
              bad = true;
            }
          }
        } else if (rank < cap) { /* else dropped */
          const int64_t q = (int64_t)__ldg(expert_offsets + e) + rank;
          /* a row outside [0, A) can only come from inconsistent scratch: skip it, report it */
          if (rank >= 0 && q >= 0 && q < A)
            pos = (int)q;
          else
            bad = true;
        }
      }
      if (sl == 0) {
        if (!EP && pos >= 0) row_src[pos] = (int32_t)a;
        assign_row[a] = pos;
      }
    }
    if (fc_cnt != nullptr) {
      /* the combine folded into GEMM2 follows: zero the token's counters of this slice's
       * 64-column blocks, and, if none of its rows will arrive (all dropped, no shared
       * expert), its output */
      const int nb = d >> 6;
      for (int cb = (sl * vps >> 3) + lane; cb < (v_end >> 3); cb += 32) fc_cnt[t * nb + cb] = 0u;
      const unsigned kept = __ballot_sync(0xFFFFFFFFu, lane < k && pos >= 0);
      if (kept == 0u && n_shared == 0)
        for (int v = v_begin; v < v_end; v += 32) st_v4(fc_out + t * d + (int64_t)v * 8, make_uint4(0, 0, 0, 0));
    }
    if (!move) continue; /* index-only dispatch */
    uint16_t* dst[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      const int p = __shfl_sync(0xFFFFFFFFu, pos, j);
      const int o = __shfl_sync(0xFFFFFFFFu, owner, j);
      uint16_t* base = EP ? ep.dst_rows[o] : x_perm;
      dst[j] = (j < k && p >= 0) ? base + (int64_t)p * d : nullptr;
    }
    for (int v0 = v_begin; v0 < v_end; v0 += 32 * U) {
      if (v0 != v_begin) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + 32 * u;
          if (v < v_end) buf[u] = ld_nc_v4(src + (int64_t)v * 8);
        }
      }
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        if (dst[j] == nullptr) continue;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + 32 * u;
          if (v < v_end) st_v4(dst[j] + (int64_t)v * 8, buf[u]);
        }
      }
    }
  }
  if (bad) raise_status(status, MOE_DEV_BOUNDS);
  /* EP: the rows went to other GPUs; make them visible there before the rank's signal */
  if (EP) __threadfence_system();
}

}  // namespace

RowSlices row_slices(int64_t T, int d) {
  const int nv = d / 8;
  const int64_t target = (int64_t)num_sms() * 32; /* warps: 4 CTAs of 8 warps per SM */
  int64_t s = T > 0 ? (target + T - 1) / T : 1;
  const int max_s = (nv + 31) / 32;
  if (s > max_s) s = max_s;
  if (s < 1) s = 1;
  int vps = (int)((nv + s - 1) / s);
  vps = (vps + 31) / 32 * 32;
  RowSlices r;
  r.vps = vps;
  r.slices = (nv + vps - 1) / vps;
  const int64_t items = T * r.slices;
  int64_t blocks = (items + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 8;
  r.blocks = (int)(blocks > cap ? cap : (blocks < 1 ? 1 : blocks));
  return r;
}

OnePass onepass_plan(const moe_shape_t& s, bool index_only) {
  OnePass op;
  const int path = dispatch_path();
  const int64_t A = (int64_t)s.T * s.k;
  if (s.T <= 0 || path == kDispatchTwoPass || (path == kDispatchAuto && A > kOnePassAutoMaxA)) return op;
  RowSlices rs = row_slices(s.T, s.d);
  if (index_only) {
    rs.slices = 1;
    rs.vps = s.d / 8;
  }
  const int64_t items = (int64_t)s.T * rs.slices;
  /* one CTA per SM: every CTA counts all A ids, so fewer CTAs do less of that; 16
   * warps per SM keep enough row copies in flight (two CTAs per SM measured ~1 us slower
   * per call on 100 MB) */
  const int64_t max_blocks = (int64_t)num_sms();
  int64_t blocks = (items + kOnePassWarps - 1) / kOnePassWarps;
  if (blocks > max_blocks) blocks = max_blocks;
  if (blocks < 1) blocks = 1;
  const int64_t ipc = (items + blocks - 1) / blocks;
  blocks = (items + ipc - 1) / ipc;
  /* tokens one CTA touches: at most ceil(ipc / slices) + 1 */
  const int64_t local = ((ipc + rs.slices - 1) / rs.slices + 1) * s.k;
  if (local > kOnePassMaxLocal) return op;
  op.use = true;
  op.blocks = (int)blocks;
  op.ipc = ipc;
  op.slices = rs.slices;
  op.vps = rs.vps;
  return op;
}

cudaError_t launch_dispatch(const moe_shape_t& s, const WsLayout& L, uint8_t* ws, const uint16_t* x,
                            const int32_t* topk_idx, int32_t* expert_counts, int32_t* expert_offsets,
                            int32_t* rank_counts, int32_t* rank_offsets, int32_t* row_src, int32_t* assign_row,
                            uint16_t* x_perm, float* imbalance, cudaStream_t stream, uint16_t* fc_out,
                            bool early_x) {
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  uint32_t* ticket = reinterpret_cast<uint32_t*>(ws + L.status + kTicketOffset);
  int32_t* chunk = reinterpret_cast<int32_t*>(ws + L.chunk);
  int32_t* lrank = reinterpret_cast<int32_t*>(ws + L.local_rank);
  const int64_t chunk_assign = L.tok_per_chunk * s.k;
  if (L.n_chunks == 0) {
    return launch_kernel(dispatch_empty_kernel, dim3(1), dim3(kScanThreads), 0, stream, 1, s.E, s.R, expert_counts,
                         expert_offsets, rank_counts, rank_offsets, imbalance);
  }
  const int32_t cap = s.capacity > 0 ? s.capacity : 0x7FFFFFFF;
  if (fc_out == nullptr) {
    const OnePass op = onepass_plan(s, x_perm == nullptr);
    if (op.use) {
      const size_t osmem = (size_t)(2 * kOnePassWarps * s.E + kOnePassMaxLocal) * sizeof(int32_t);
      return launch_kernel(dispatch_onepass_kernel<8>, dim3((unsigned)op.blocks), dim3(kOnePassThreads), osmem,
                           stream, 1, x, topk_idx, (int64_t)s.T, s.d, s.E, s.R, s.k, cap, op.ipc, op.slices, op.vps,
                           expert_counts, expert_offsets, rank_counts, rank_offsets, imbalance, row_src, assign_row,
                           x_perm, status, early_x ? 1 : 0);
    }
  }
  const size_t smem = (size_t)kHistWarps * s.E * sizeof(int32_t);
  cudaError_t e = launch_kernel(dispatch_count_kernel, dim3((unsigned)L.n_chunks), dim3(kHistThreads), smem, stream,
                                1, topk_idx, L.A, s.E, s.R, cap, chunk_assign, L.n_chunks, chunk, lrank, status,
                                ticket, expert_counts, expert_offsets, rank_counts, rank_offsets, imbalance, row_src);
  if (e != cudaSuccess) return e;
  RowSlices rs = row_slices(s.T, s.d);
  if (x_perm == nullptr) { /* indices only: one warp per token */
    rs.slices = 1;
    rs.vps = s.d / 8;
    const int64_t blocks = ((int64_t)s.T + 7) / 8, cap = (int64_t)num_sms() * 8;
    rs.blocks = (int)(blocks > cap ? cap : blocks);
  }
  return launch_kernel(dispatch_permute_kernel<4, false>, dim3((unsigned)rs.blocks), dim3(256), 0, stream, 1, x,
                       topk_idx, (const int32_t*)chunk, (const int32_t*)lrank, (const int32_t*)expert_offsets,
                       (int64_t)s.T, s.d, s.E, s.k, cap, L.tok_per_chunk, rs.slices, rs.vps, row_src, assign_row,
                       x_perm, status, EpTarget{},
                       fc_out ? reinterpret_cast<uint32_t*>(ws + L.fc_cnt) : (uint32_t*)nullptr, fc_out,
                       s.n_shared);
}

cudaError_t launch_dispatch_count(const moe_shape_t& s, const WsLayout& L, uint8_t* ws, const int32_t* topk_idx,
                                  int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                                  int32_t* rank_offsets, float* imbalance, bool apply_capacity, cudaStream_t stream) {
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  uint32_t* ticket = reinterpret_cast<uint32_t*>(ws + L.status + kTicketOffset);
  int32_t* chunk = reinterpret_cast<int32_t*>(ws + L.chunk);
  int32_t* lrank = reinterpret_cast<int32_t*>(ws + L.local_rank);
  if (L.n_chunks == 0)
    return launch_kernel(dispatch_empty_kernel, dim3(1), dim3(kScanThreads), 0, stream, 1, s.E, s.R, expert_counts,
                         expert_offsets, rank_counts, rank_offsets, imbalance);
  const size_t smem = (size_t)kHistWarps * s.E * sizeof(int32_t);
  const int32_t cap = apply_capacity && s.capacity > 0 ? s.capacity : 0x7FFFFFFF;
  return launch_kernel(dispatch_count_kernel, dim3((unsigned)L.n_chunks), dim3(kHistThreads), smem, stream, 1,
                       topk_idx, L.A, s.E, s.R, cap, L.tok_per_chunk * s.k, L.n_chunks, chunk, lrank, status, ticket,
                       expert_counts, expert_offsets, rank_counts, rank_offsets, imbalance, (int32_t*)nullptr);
}

cudaError_t launch_ep_scatter(const moe_shape_t& s, const WsLayout& L, uint8_t* ws, const uint16_t* x,
                              const int32_t* topk_idx, const EpTarget& ep, int32_t* send_row, cudaStream_t stream) {
  if (s.T == 0) return cudaSuccess;
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  int32_t* chunk = reinterpret_cast<int32_t*>(ws + L.chunk);
  int32_t* lrank = reinterpret_cast<int32_t*>(ws + L.local_rank);
  const RowSlices rs = row_slices(s.T, s.d);
  return launch_kernel(dispatch_permute_kernel<4, true>, dim3((unsigned)rs.blocks), dim3(256), 0, stream, 1, x,
                       topk_idx, (const int32_t*)chunk, (const int32_t*)lrank, (const int32_t*)nullptr, (int64_t)s.T,
                       s.d, s.E, s.k, (int32_t)0, L.tok_per_chunk, rs.slices, rs.vps, (int32_t*)nullptr, send_row,
                       (uint16_t*)nullptr, status, ep, (uint32_t*)nullptr, (uint16_t*)nullptr, 0);
}

}  // namespace moe
