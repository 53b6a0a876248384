/*
 * expert_ffn.cu -- the experts' SwiGLU FFN as two persistent grouped GEMMs on
 * the 5th-generation tensor cores (tcgen05.mma, TMEM accumulators, TMA loads).
 *
 * Page "Expert Parallelism" (learning-materials IX.05) §4 COMPUTE: every expert
 * multiplies its own tokens, and the differently sized per-expert GEMMs run as
 * one grouped launch; §8: looping over the experts one by one is much slower
 * than a grouped GEMM. The page "UltraEP ..." (thelatestinai.com/papers/2606.04101, the
 * makespan-aware dispatcher abstract) notes that grouped GEMM rounds each
 * expert's tokens up to 128-row M tiles: that is the tile height here, and the
 * padding rows are masked, never counted as work.
 *
 *   GEMM1 (gate/up):  h[p, :] = silu(x_perm[p] . W_gate,e^T) * (x_perm[p] . W_up,e^T)
 *   GEMM2 (down):     y_perm[p, :] = h[p] . W2_e^T
 * Groups: the E routed experts (rows [off[e], off[e+1]) of x_perm) and, when
 * n_shared = 1, a shared expert over all T rows of x.
 *
 * Schedule (device side, no host read-back of the counts): every CTA loads
 * expert_offsets and computes the m-tile prefix over the groups in shared memory.
 * The tiles are numbered group by group; inside a group the m-tiles are the inner
 * index, so consecutive tiles share one weight tile. CTAs (CTA pairs) claim tile
 * numbers from an atomic counter in the workspace header, so the tiles in flight
 * at any moment are consecutive (they share weight tiles in L2 however the CTAs
 * drift) and a CTA that finishes a tile early simply takes the next one; the last
 * CTA to finish puts the counter back to zero for the next launch.
 *
 * Two tile shapes, same roles (warp 0 claims tiles and issues TMA loads from one
 * thread, warp 1 owns TMEM and issues tcgen05.mma from one thread, warps 2-5 drain
 * the accumulator with tcgen05.ld and run the epilogue; the claimed tile numbers go
 * from warp 0 to the others through a small shared-memory queue), two TMEM
 * accumulators of 256 fp32 columns so the epilogue of tile i overlaps the main loop
 * of tile i+1:
 *   single one CTA computes a 128 x 256 (GEMM1) or 128 x BN (GEMM2) tile with
 *          cta_group::1 MMAs (4-stage ring of 48 KB);
 *   pair   a cluster of 2 CTAs on neighbouring SMs computes a 256 x 256 tile
 *          with cta_group::2 MMAs: each CTA stages its own 128 rows of A and 128
 *          of the 256 rows of B (6-stage ring of 32 KB), so each SM moves 32 KB
 *          of operands per 64-deep K step instead of 48 KB. A group's last block
 *          of at most 128 rows runs as a half-height pair tile (M = 128, 64 rows
 *          per CTA, half the MMA time), so pairs pad a group to a multiple of 128
 *          rows, like single tiles.
 * moe_set_gemm_policy chooses the shape: by default pair tiles when the experts
 * average at least 1024 rows (GEMM2 also needs d % 256 == 0), single tiles
 * otherwise.
 * GEMM1 can also gather its A rows straight from x through row_src instead of
 * reading x_perm (the GATHER instantiation: a warp of cp.async copies instead of
 * one TMA tile per stage).
 * GEMM1's B tile holds gate rows and the matching up rows, so one N=256 MMA yields
 * both halves of the SwiGLU for 128 output columns and the epilogue combines them
 * before anything leaves the SM (single: 128 gate over 128 up rows; pair: each CTA
 * 64 gate over the matching 64 up rows).
 * The hidden rows h live in the workspace, each group's rows padded to a
 * multiple of 256, so GEMM1 stores whole tiles and GEMM2 loads whole tiles with
 * either tile shape; GEMM2 masks its stores to the group's real rows.
 *
 * Every mbarrier wait is bounded (MOE_DEV_TIMEOUT on expiry); on abort each
 * role stops issuing, waits for its in-flight copies / MMAs, and the CTA frees
 * its TMEM before returning.
 */
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdio>
#include <mutex>

#include "moe_device.cuh"

namespace moe {

namespace {

constexpr int BK = 64; /* bf16 elements = 128 bytes = one swizzle row */
constexpr int kThreads = 192;
constexpr int kHPad = 256; /* h rows per group are padded to a multiple of this */
constexpr uint64_t kDrainNs = 2000000000ull;
constexpr uint32_t HALF_TILE = 128 * BK * 2; /* 16 KB: 128 rows x 64 bf16 */

struct FfnParams {
  const int32_t* expert_offsets; /* [E+1] */
  int E;
  int n_shared;
  int64_t T;
  int64_t A;
  int K;          /* reduction length: d (GEMM1) or f (GEMM2) */
  int n_tiles_n;  /* output column tiles */
  int f;
  int d;
  uint16_t* out0; /* GEMM1: h; GEMM2: y_perm */
  uint16_t* out1; /* GEMM2: y_shared */
  int64_t ld_out; /* row stride of the output in elements */
  uint32_t* status;
  uint64_t timeout_ns;
  int stall_first_stage; /* test hook: arm the first stage of each CTA's first tile but never load it */
  uint32_t* tile_ctr;    /* [0]: next tile to claim, [1]: CTAs finished (workspace header; zero between launches) */
  const int32_t* row_src;   /* GEMM1 gathering A from x: row_src of dispatch (null: A is x_perm) */
  const uint16_t* gather_x; /* x [T, d] rows to gather from */
  int k;                    /* experts per token (token of assignment a = a / k) */
  /* GEMM2 with the combine folded into its epilogue (fc_out null: y only) */
  const int32_t* fc_row_src;    /* [A] assignment held by each row of y_perm */
  const int32_t* fc_assign_row; /* [T*k] row of each assignment (-1: dropped) */
  const float* fc_gate;         /* [T, k] */
  uint16_t* fc_out;             /* [T, d] */
  uint32_t* fc_cnt;             /* [T][d / 64] rows of a token stored so far (zero at the start) */
};

struct Tile {
  int g;           /* group: expert index, or E for the shared expert */
  int m, n;        /* m-tile inside the group, n-tile */
  int valid;       /* real rows in this m-tile (<= TM) */
  int half;        /* CTA-pair tile of at most 128 rows: computed as M = 128 (64 rows per CTA) */
  int a_row;       /* first A row (TMA coordinate) */
  int b_row;       /* first B row (TMA coordinate); GEMM1: the gate rows */
  int64_t out_row; /* first output row */
};

/* Tiles are claimed at run time: each CTA (each CTA pair) takes the next tile index
 * from a counter in the workspace, so a CTA that finishes early (a half-height tile,
 * or weights already in L2) takes more tiles, and the tiles running at any moment are
 * consecutive in the order below, sharing weight tiles in L2. The claimer passes each
 * index to the CTA's other roles through a small shared-memory queue. */
constexpr int kTQ = 8; /* tile-queue slots */

/* Shared-memory schedule, built by one warp: s_off = expert_offsets,
 * s_mpref[g] = m-tiles (TM rows) of groups < g, s_hpref[g] = 256-row blocks of h
 * of groups < g. Returns false if expert_offsets is inconsistent. */
template <int TM>
__device__ __forceinline__ bool build_schedule(const FfnParams& p, int32_t* s_off, int32_t* s_mpref, int32_t* s_hpref,
                                               int lane) {
  const int E = p.E;
  const int G = E + p.n_shared;
  bool ok = true;
  for (int i = lane; i <= E; i += 32) s_off[i] = __ldg(p.expert_offsets + i);
  __syncwarp();
  int carry_m = 0, carry_h = 0;
  for (int base = 0; base < G; base += 32) {
    const int g = base + lane;
    int rows = 0;
    if (g < E) {
      const int lo = s_off[g], hi = s_off[g + 1];
      if (lo < 0 || hi < lo || hi > p.A) ok = false;
      rows = max(0, hi - lo);
    } else if (g < G) {
      rows = (int)p.T;
    }
    int im = (rows + TM - 1) / TM, ih = (rows + kHPad - 1) / kHPad;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ym = __shfl_up_sync(0xFFFFFFFFu, im, o);
      const int yh = __shfl_up_sync(0xFFFFFFFFu, ih, o);
      if (lane >= o) {
        im += ym;
        ih += yh;
      }
    }
    if (g < G) {
      s_mpref[g + 1] = carry_m + im;
      s_hpref[g + 1] = carry_h + ih;
    }
    carry_m += __shfl_sync(0xFFFFFFFFu, im, 31);
    carry_h += __shfl_sync(0xFFFFFFFFu, ih, 31);
  }
  if (lane == 0) {
    s_mpref[0] = 0;
    s_hpref[0] = 0;
    if (s_off[0] != 0) ok = false;
  }
  return __all_sync(0xFFFFFFFFu, ok);
}

/* Tile order inside a group: the m-tiles are the inner index, so the tiles running
 * at once share their weight tile and the group's A rows are re-read from L2 by every
 * weight column tile. A group whose A rows outnumber its weight rows (a shared expert
 * over a long batch) runs its m-tiles in bands of at most kBandBytes of A rows instead,
 * m-tiles inner inside a band: a band's rows stay in L2 while every column tile passes
 * over them, so the group's A rows come from DRAM once, and its (smaller) weights once
 * per band. */
constexpr int64_t kBandBytes = int64_t(24) << 20;

/* Linear tile index -> tile (groups in order; bands of m-tiles inside a group). */
template <int MODE, int TM, int BN>
__device__ __forceinline__ Tile decode_tile(int64_t L, const FfnParams& p, const int32_t* s_off,
                                            const int32_t* s_mpref, const int32_t* s_hpref) {
  const int G = p.E + p.n_shared;
  const int q = (int)(L / p.n_tiles_n); /* s_mpref[g] <= q < s_mpref[g+1] */
  int lo = 0, hi = G;                   /* the last g with s_mpref[g] <= q */
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_mpref[mid] <= q)
      lo = mid;
    else
      hi = mid;
  }
  Tile t;
  t.g = lo;
  const int mt = s_mpref[lo + 1] - s_mpref[lo];
  const int local = (int)(L - (int64_t)s_mpref[lo] * p.n_tiles_n);
  const bool shared = lo >= p.E;
  const int rows = shared ? (int)p.T : s_off[lo + 1] - s_off[lo];
  const int w_rows = p.n_tiles_n * (MODE == 0 ? 256 : BN); /* weight rows of a group */
  const int band = rows > w_rows ? (int)max((int64_t)1, kBandBytes / ((int64_t)TM * p.K * 2)) : mt;
  const int b = local / (band * p.n_tiles_n);         /* band of this tile */
  const int r = local - b * band * p.n_tiles_n;       /* index inside the band */
  const int gm = min(band, mt - b * band);             /* m-tiles in this band */
  t.n = r / gm;
  t.m = b * band + (r - t.n * gm);
  t.valid = min(TM, rows - t.m * TM);
  t.half = (TM == 256 && t.valid <= 128) ? 1 : 0;
  const int hrow = s_hpref[lo] * kHPad + t.m * TM;
  if (MODE == 0) {
    t.a_row = shared ? t.m * TM : s_off[lo] + t.m * TM;
    t.b_row = shared ? t.n * 128 : lo * 2 * p.f + t.n * 128;
    t.out_row = hrow;
  } else {
    t.a_row = hrow;
    t.b_row = shared ? t.n * BN : lo * p.d + t.n * BN;
    t.out_row = shared ? (int64_t)t.m * TM : (int64_t)s_off[lo] + t.m * TM;
  }
  return t;
}

__device__ __forceinline__ float silu_f(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

/* Per-warp epilogue staging: 32 rows x 64 bf16 (4 KB) in the 128-byte swizzled
 * layout a TMA store with a {64, 32} box expects (16-byte chunk c of row r at
 * chunk position c ^ (r % 8)). */
constexpr uint32_t kStageBytesPerWarp = 32 * 128;
constexpr uint32_t kEpiStagingBytes = 4 * kStageBytesPerWarp;

__device__ __forceinline__ void stage_row_chunk(uint32_t sbase, int lane, int chunk, uint32_t a, uint32_t b,
                                                uint32_t c, uint32_t d) {
  st_shared_v4(sbase + (uint32_t)lane * 128u + ((uint32_t)(chunk ^ (lane & 7)) << 4), a, b, c, d);
}

/* Hand the warp's staged 32 x 64 block to TMA: all lanes' shared writes are made
 * visible to the async proxy, then lane 0 issues the store. */
__device__ __forceinline__ void store_staged_block(const CUtensorMap* map, uint8_t* stage, int32_t x, int32_t y,
                                                   int lane) {
  fence_proxy_async_shared();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, stage, x, y);
    bulk_commit_group();
  }
}

/* Before a warp overwrites its staging buffer, its previous TMA store must have read it. */
__device__ __forceinline__ void staging_reusable(int lane) {
  if (lane == 0) bulk_wait_read_all();
  __syncwarp();
}

/* GEMM1 epilogue block: 32 rows (this warp's TMEM lanes) x 64 columns of
 * h = silu(gate) * up, with gate at accumulator columns [gcol, gcol + 64) and up at
 * [ucol, ucol + 64); staged in shared memory and TMA-stored at column x, row y. */
__device__ __forceinline__ void epi_swiglu_block(uint32_t taddr, int gcol, int ucol, uint8_t* stage,
                                                 const CUtensorMap* map, int32_t x, int32_t y, int lane) {
  const uint32_t sbase = smem_u32(stage);
  staging_reusable(lane);
#pragma unroll 1
  for (int hh = 0; hh < 2; ++hh) {
    const int c = hh * 32;
    uint32_t g0[16], g1[16], u0[16], u1[16];
    tmem_ld16(taddr + gcol + c, g0);
    tmem_ld16(taddr + gcol + c + 16, g1);
    tmem_ld16(taddr + ucol + c, u0);
    tmem_ld16(taddr + ucol + c + 16, u1);
    tmem_ld_wait();
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w[i] = pack_bf16x2(silu_f(__uint_as_float(g0[2 * i])) * __uint_as_float(u0[2 * i]),
                         silu_f(__uint_as_float(g0[2 * i + 1])) * __uint_as_float(u0[2 * i + 1]));
      w[8 + i] = pack_bf16x2(silu_f(__uint_as_float(g1[2 * i])) * __uint_as_float(u1[2 * i]),
                             silu_f(__uint_as_float(g1[2 * i + 1])) * __uint_as_float(u1[2 * i + 1]));
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
      stage_row_chunk(sbase, lane, hh * 4 + q, w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
  store_staged_block(map, stage, x, y, lane);
}

/* GEMM2 epilogue block: 32 rows x 64 columns of bf16 from accumulator columns
 * [col, col + 64). A warp whose 32 rows are all real (whole) stages them and
 * TMA-stores at column x, row y; a warp holding a group's ragged end stores its real
 * rows (live lanes) directly, row by row at dst (this lane's row, column x). */
__device__ __forceinline__ void epi_store_block(uint32_t taddr, int col, bool whole, bool live, uint16_t* dst,
                                                uint8_t* stage, const CUtensorMap* map, int32_t x, int32_t y,
                                                int lane) {
  uint32_t v[4][16];
#pragma unroll
  for (int q = 0; q < 4; ++q) tmem_ld16(taddr + col + q * 16, v[q]);
  tmem_ld_wait();
  if (whole) {
    const uint32_t sbase = smem_u32(stage);
    staging_reusable(lane);
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const uint32_t* r = &v[q][hf * 8];
        stage_row_chunk(sbase, lane, q * 2 + hf, pack_bf16x2(__uint_as_float(r[0]), __uint_as_float(r[1])),
                        pack_bf16x2(__uint_as_float(r[2]), __uint_as_float(r[3])),
                        pack_bf16x2(__uint_as_float(r[4]), __uint_as_float(r[5])),
                        pack_bf16x2(__uint_as_float(r[6]), __uint_as_float(r[7])));
      }
    store_staged_block(map, stage, x, y, lane);
  } else if (live) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const uint32_t* r = &v[q][hf * 8];
        st_v4(dst + q * 16 + hf * 8,
              make_uint4(pack_bf16x2(__uint_as_float(r[0]), __uint_as_float(r[1])),
                         pack_bf16x2(__uint_as_float(r[2]), __uint_as_float(r[3])),
                         pack_bf16x2(__uint_as_float(r[4]), __uint_as_float(r[5])),
                         pack_bf16x2(__uint_as_float(r[6]), __uint_as_float(r[7]))));
      }
  }
}

/* Combine of token `tok`, columns [cb * 64, cb * 64 + 64): the gate-weighted sum of
 * its k rows of y_perm in j order, plus its y_shared row, fp32, one bf16 rounding
 * (the arithmetic of the separate combine kernel). The rows were stored by any CTA
 * of this launch: read through L2. */
__device__ __forceinline__ void fused_combine_block(const FfnParams& p, int64_t tok, int cb) {
#pragma unroll 1
  for (int h = 0; h < 2; ++h) {
    const int c0 = cb * 64 + h * 32;
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
#pragma unroll 1
    for (int j = 0; j < p.k; ++j) {
      const int pr = __ldg(p.fc_assign_row + tok * p.k + j);
      if (pr < 0) continue;
      const float g = __ldg(p.fc_gate + tok * p.k + j);
      const uint4* src = reinterpret_cast<const uint4*>(p.out0 + (int64_t)pr * p.ld_out + c0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = __ldcg(src + q);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[q * 8 + 2 * i] = fmaf(g, bf16lo(w[i]), acc[q * 8 + 2 * i]);
          acc[q * 8 + 2 * i + 1] = fmaf(g, bf16hi(w[i]), acc[q * 8 + 2 * i + 1]);
        }
      }
    }
    if (p.n_shared) {
      const uint4* sh = reinterpret_cast<const uint4*>(p.out1 + tok * p.ld_out + c0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = __ldcg(sh + q);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[q * 8 + 2 * i] += bf16lo(w[i]);
          acc[q * 8 + 2 * i + 1] += bf16hi(w[i]);
        }
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(p.fc_out + tok * p.ld_out + c0);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      st_v4(dst + q, make_uint4(pack_bf16x2(acc[q * 8], acc[q * 8 + 1]), pack_bf16x2(acc[q * 8 + 2], acc[q * 8 + 3]),
                                pack_bf16x2(acc[q * 8 + 4], acc[q * 8 + 5]),
                                pack_bf16x2(acc[q * 8 + 6], acc[q * 8 + 7])));
  }
}

/* GEMM2 with the combine folded in: after this warp has stored its 32 rows of
 * columns [xcol, xcol + 64 * nblk), each row counts itself in on its token's
 * counter of every 64-column block; the row whose count completes the token (its
 * kept assignments, plus its shared row) sums that block of the token's rows.
 * Deterministic: the sum is taken in j order from memory, whichever row is last. */
__device__ __forceinline__ void fused_combine_warp(const FfnParams& p, const Tile& t, int row0, int xcol, int nblk,
                                                   int lane) {
  if (lane == 0) {
    bulk_wait_all(); /* this warp's TMA stores are complete ... */
    fence_proxy_async_global(); /* ... and ordered before what the generic proxy does next */
  }
  __syncwarp();
  const int r = row0 + lane;
  if (r >= t.valid) return;
  const bool shared = t.g >= p.E;
  const int64_t prow = t.out_row + r;
  int64_t tok;
  if (shared) {
    tok = prow;
  } else {
    const int a = __ldg(p.fc_row_src + prow);
    if (a < 0) return;
    tok = a / p.k;
  }
  uint32_t need = (uint32_t)p.n_shared;
  for (int j = 0; j < p.k; ++j) need += __ldg(p.fc_assign_row + tok * p.k + j) >= 0 ? 1u : 0u;
  __threadfence(); /* this row's stores before its count */
  const int nb = p.d / 64;
#pragma unroll 1
  for (int b = 0; b < nblk; ++b) {
    const int cb = xcol / 64 + b;
    if (atomicAdd(p.fc_cnt + tok * nb + cb, 1u) == need - 1u) {
      __threadfence(); /* every other row of the token is visible */
      fused_combine_block(p, tok, cb);
    }
  }
}

/* Epilogue of this warp's 32 accumulator rows of a single-CTA tile. `taddr`
 * addresses the warp's TMEM lane quarter at the accumulator's first column; `row0`
 * is the warp's first row inside the tile (this thread's row is row0 + lane).
 * GEMM1: the accumulator holds gate in columns [0, 128) and up in [128, 256); h =
 *        silu(gate) * up, 128 columns, stored as two blocks by every warp holding a real
 *        row (the rest of a 32-row block is h padding).
 * GEMM2: BN columns, BN / 64 blocks, masked to the group's real rows. */
template <int MODE, int BN>
__device__ __forceinline__ void epilogue_warp(const FfnParams& p, const Tile& t, uint32_t taddr, int row0, int lane,
                                              uint8_t* stage, const CUtensorMap* out0, const CUtensorMap* out1) {
  const int32_t grow = (int32_t)(t.out_row + row0); /* output row of lane 0 */
  if (MODE == 0) {
    if (row0 >= t.valid) return; /* no real row in this warp's 32: its h rows are padding, never read as results */
#pragma unroll 1
    for (int j = 0; j < 2; ++j) epi_swiglu_block(taddr, j * 64, 128 + j * 64, stage, out0, t.n * 128 + j * 64, grow, lane);
  } else {
    if (row0 >= t.valid) return; /* no real row in this warp's 32: nothing to store or count */
    const bool shared = t.g >= p.E;
    const CUtensorMap* map = shared ? out1 : out0;
    const bool whole = row0 + 32 <= t.valid; /* warp-uniform */
    const bool live = row0 + lane < t.valid;
    uint16_t* dst = (shared ? p.out1 : p.out0) + (t.out_row + row0 + lane) * p.ld_out + (int64_t)t.n * BN;
#pragma unroll 1
    for (int j = 0; j < BN / 64; ++j)
      epi_store_block(taddr, j * 64, whole, live, dst + j * 64, stage, map, t.n * BN + j * 64, grow, lane);
    if (p.fc_out) fused_combine_warp(p, t, row0, t.n * BN, BN / 64, lane);
  }
}

/* Epilogue of warp q (lane quarter q) of CTA `rank` of a CTA-pair tile.
 * Full tile (M = 256): the CTA holds rows [rank * 128, +128) of the tile, warp q
 *   rows q * 32 + [0, 32), every column of the tile.
 * Half tile (M = 128, at most 128 real rows): the CTA holds rows [rank * 64, +64);
 *   TMEM lanes 0-63 hold them for the tile's first half of columns and lanes 64-127
 *   the same rows for the second half, so warp q has rows (q % 2) * 32 + [0, 32) and
 *   column half q / 2.
 * GEMM1: each CTA staged 64 gate rows and the matching 64 up rows of the weights, so
 *   the accumulator columns run [gate 64 | up 64] per 64 columns of h: a full tile
 *   has h columns [0, 64) from gate [0, 64) / up [64, 128) and [64, 128) from gate
 *   [128, 192) / up [192, 256); a half tile's warp has its 64 h columns from gate
 *   [0, 64) / up [64, 128) of its lanes.
 * GEMM2: 256 output columns (full) or 128 per column half (half). */
template <int MODE>
__device__ __forceinline__ void epilogue_pair_warp(const FfnParams& p, const Tile& t, uint32_t taddr, int q,
                                                   uint32_t rank, int lane, uint8_t* stage, const CUtensorMap* out0,
                                                   const CUtensorMap* out1) {
  const int row0 = t.half ? (int)rank * 64 + (q & 1) * 32 : (int)rank * 128 + q * 32; /* inside the tile */
  const int col0 = t.half ? (q >> 1) * (MODE == 0 ? 64 : 128) : 0;                   /* inside the tile */
  const int32_t grow = (int32_t)(t.out_row + row0);
  if (MODE == 0) {
    if (t.half) {
      epi_swiglu_block(taddr, 0, 64, stage, out0, t.n * 128 + col0, grow, lane);
    } else {
#pragma unroll 1
      for (int j = 0; j < 2; ++j)
        epi_swiglu_block(taddr, j * 128, j * 128 + 64, stage, out0, t.n * 128 + j * 64, grow, lane);
    }
  } else {
    const bool shared = t.g >= p.E;
    const CUtensorMap* map = shared ? out1 : out0;
    const bool whole = row0 + 32 <= t.valid; /* warp-uniform */
    const bool live = row0 + lane < t.valid;
    const int xcol = t.n * 256 + col0;
    uint16_t* dst = (shared ? p.out1 : p.out0) + (t.out_row + row0 + lane) * p.ld_out + (int64_t)xcol;
    const int nblk = t.half ? 2 : 4;
#pragma unroll 1
    for (int j = 0; j < nblk; ++j)
      epi_store_block(taddr, j * 64, whole, live, dst + j * 64, stage, map, xcol + j * 64, grow, lane);
    if (p.fc_out) fused_combine_warp(p, t, row0, xcol, nblk, lane);
  }
}

/* Shared-memory control block that follows the operand ring. */
struct Ctrl {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint64_t tq_full[kTQ];  /* tile index written (claimer arrives) */
  uint64_t tq_empty[kTQ]; /* tile index read by every consumer role */
  int32_t tq[kTQ];        /* claimed tile index, -1 = no more tiles */
  uint32_t tmem_slot;
  int abort_flag;
  int ok;
  int32_t off[kMaxE + 2];
  int32_t mpref[kMaxE + 2];
  int32_t hpref[kMaxE + 2];
};

/* ======================= single-CTA tiles (128 x N) ======================== */

template <int MODE, int BN>
struct SingleCfg {
  static constexpr int STAGES = 4;
  static constexpr int B_ROWS = (MODE == 0) ? 256 : BN; /* rows of W per tile (N of the MMA) */
  static constexpr uint32_t B_BYTES = (uint32_t)B_ROWS * BK * 2;
  static constexpr uint32_t STAGE_BYTES = HALF_TILE + B_BYTES;
  static constexpr uint32_t ACC_COLS = B_ROWS;
  static constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;
  static constexpr uint32_t IDESC = umma_idesc_bf16(128, B_ROWS);
  static constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + kEpiStagingBytes + sizeof(Ctrl);
  static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation must be a power of two");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

/* Claim the next tile index (-1 once every tile is taken). One thread per CTA (per
 * CTA pair) claims; the counter sits in the workspace header. */
__device__ __forceinline__ int claim_tile(const FfnParams& p, int64_t total) {
  const uint32_t L = atomicAdd(p.tile_ctr, 1u);
  return (int64_t)L < total ? (int)L : -1;
}

/* Called once per CTA by one thread after every role has stopped claiming: the
 * last CTA of the launch to get here puts the counters back to zero, ready for the
 * next launch on this workspace (which touches them only after this one completed). */
__device__ __forceinline__ void release_tile_counter(const FfnParams& p) {
  __threadfence();
  if (atomicAdd(p.tile_ctr + 1, 1u) == gridDim.x - 1) {
    atomicExch(p.tile_ctr, 0u);
    atomicExch(p.tile_ctr + 1, 0u);
  }
}

/* A consumer role's turn on queue slot i: wait for the claimed index, read it. The
 * caller releases the slot (tq_empty) once it has the value. Returns false on
 * timeout or abort. CLUSTER: the index was written by the peer CTA of a pair. */
template <bool CLUSTER = false>
__device__ __forceinline__ bool read_tile_index(Ctrl* ctl, int i, uint64_t timeout_ns, volatile int* s_abort,
                                                int* v) {
  const int slot = i % kTQ;
  if (!mbar_wait<CLUSTER>(&ctl->tq_full[slot], (uint32_t)(i / kTQ) & 1u, timeout_ns, s_abort)) return false;
  *v = *reinterpret_cast<volatile int32_t*>(&ctl->tq[slot]);
  return true;
}

template <int MODE, int BN, bool GATHER>
__global__ void __launch_bounds__(kThreads, 1)
    ffn_gemm_single_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                           const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                           const __grid_constant__ CUtensorMap tmO0, const __grid_constant__ CUtensorMap tmO1,
                           const __grid_constant__ CUtensorMap tmA0r16, const __grid_constant__ CUtensorMap tmA0r32,
                           const __grid_constant__ CUtensorMap tmA0r64, const FfnParams p) {
  using C = SingleCfg<MODE, BN>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  /* 128-byte swizzled tiles need 1024-byte aligned shared-space addresses */
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * HALF_TILE;
  uint8_t* sEpi = sB + STAGES * C::B_BYTES;
  Ctrl* ctl = reinterpret_cast<Ctrl*>(sEpi + kEpiStagingBytes);
  volatile int* s_abort = &ctl->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  static_assert(!GATHER || MODE == 0, "only GEMM1 gathers its A rows");
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      /* gathering: lane 0's expect_tx arrival + one arrival per producer lane */
      mbar_init(&ctl->full[s], GATHER ? 33 : 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->tfull[b], 1);
      mbar_init(&ctl->tempty[b], 4);
    }
    for (int i = 0; i < kTQ; ++i) {
      mbar_init(&ctl->tq_full[i], 1);
      mbar_init(&ctl->tq_empty[i], 5); /* the MMA issuer and the 4 epilogue warps */
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
    tma_prefetch_desc(&tmO0);
    tma_prefetch_desc(&tmO1);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait(); /* expert_offsets and the A rows come from earlier kernels */
  pdl_trigger();
  if (warp == 2) {
    const bool ok = build_schedule<128>(p, ctl->off, ctl->mpref, ctl->hpref, lane);
    if (lane == 0) ctl->ok = ok ? 1 : 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = ctl->tmem_slot;
  const int G = p.E + p.n_shared;
  int64_t total = (int64_t)ctl->mpref[G] * p.n_tiles_n;
  if (!ctl->ok) {
    total = 0;
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(p.status, MOE_DEV_COUNT_MISMATCH);
  }
  const int KB = p.K / BK;

  if (warp == 0) {
    /* ---------------- producer: claims tiles, loads their operands ----------------
     * Lane 0 claims each tile and passes its index on through the tile queue. The
     * TMA form issues from lane 0 alone; the gathering form has the whole warp copy
     * the A rows (see below). */
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed_phase[STAGES];
    bool armed[STAGES];
#pragma unroll
    for (int s = 0; s < STAGES; ++s) {
      armed[s] = false;
      armed_phase[s] = 0;
    }
    bool abort = false;
    bool first = true;
    /* the claim for the next tile goes out one tile ahead, so that its round trip to
     * L2 overlaps the loads of the current tile */
    int next = lane == 0 ? claim_tile(p, total) : -1;
    /* gathering: lane l moves 16-byte chunk l % 8 of rows l / 8 + 4 i (i < 32) */
    const int chunk = lane & 7, row0 = lane >> 3;
    /* swizzle of rows row0 + 4 i: (row0 + 4 i) % 8 == row0 ^ (4 (i % 2)) since row0 < 4 */
    const uint32_t sw_even = (uint32_t)(chunk ^ row0) << 4, sw_odd = (uint32_t)(chunk ^ row0 ^ 4) << 4;
    const uint32_t row_bytes = (uint32_t)p.d * 2u; /* T * d * 2 < 2^32 is checked on the host */
    const char* xk0 = GATHER ? reinterpret_cast<const char*>(p.gather_x) + chunk * 16 : nullptr;
    for (int i = 0; !abort; ++i) {
      if (!GATHER && lane != 0) break;
      int v = -1;
      if (lane == 0) {
        const int slot = i % kTQ;
        if (!mbar_wait(&ctl->tq_empty[slot], ((uint32_t)(i / kTQ) & 1u) ^ 1u, p.timeout_ns, s_abort)) {
          abort = true;
        } else {
          v = next;
          ctl->tq[slot] = v;
          mbar_arrive(&ctl->tq_full[slot]);
          if (v >= 0) next = claim_tile(p, total);
        }
      }
      if (GATHER) {
        v = __shfl_sync(0xFFFFFFFFu, v, 0);
        abort = __shfl_sync(0xFFFFFFFFu, abort ? 1 : 0, 0) != 0;
      }
      if (abort || v < 0) break;
      const Tile t = decode_tile<MODE, 128, BN>(v, p, ctl->off, ctl->mpref, ctl->hpref);
      const bool shared = t.g >= p.E;
      if constexpr (!GATHER) {
        /* TMA tiles, lane 0 only */
        /* A routed group's last tile of at most 16, 32 or 64 real rows loads a box of
         * that many rows of A: the rows past it keep what an earlier tile left in the
         * stage, and their accumulator rows are never stored (GEMM1: h padding rows,
         * which GEMM2 computes on but never stores either) */
        const int a_rows =
            shared ? 128 : (t.valid <= 16 ? 16 : (t.valid <= 32 ? 32 : (t.valid <= 64 ? 64 : 128)));
        const CUtensorMap* mA = shared ? &tmA1
                                       : (a_rows == 16 ? &tmA0r16
                                                       : (a_rows == 32 ? &tmA0r32 : (a_rows == 64 ? &tmA0r64 : &tmA0)));
        const CUtensorMap* mB = shared ? &tmB1 : &tmB0;
        const uint32_t stage_tx = (uint32_t)a_rows * (BK * 2) + C::B_BYTES;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, p.timeout_ns, s_abort)) {
            abort = true;
            break;
          }
          mbar_arrive_expect_tx(&ctl->full[stage], stage_tx);
          if (p.stall_first_stage && first && kb == 0) {
            /* test hook: this stage's bytes never arrive, so the MMA's bounded wait runs out */
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
            continue;
          }
          armed[stage] = true;
          armed_phase[stage] = phase;
          uint8_t* a_dst = sA + stage * HALF_TILE;
          uint8_t* b_dst = sB + stage * C::B_BYTES;
          tma_load_2d(a_dst, mA, &ctl->full[stage], kb * BK, t.a_row);
          if (MODE == 0) {
            tma_load_2d(b_dst, mB, &ctl->full[stage], kb * BK, t.b_row);
            tma_load_2d(b_dst + HALF_TILE, mB, &ctl->full[stage], kb * BK, t.b_row + p.f);
          } else {
            tma_load_2d(b_dst, mB, &ctl->full[stage], kb * BK, t.b_row);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      } else {
        /* A gathered from x: lane 0 waits for free stages, arms them and TMA-loads B
         * (and A for the shared expert, whose rows are x itself). The routed rows of
         * GEMM1 come straight from x: row p of expert e is token row_src[p] / k. The
         * whole warp copies them with 16-byte cp.async into the 128-byte swizzled
         * layout of the stage; each lane's byte offsets into x stay in registers for
         * the whole tile. Every lane arrives on every stage barrier once its copies
         * have landed (the barrier counts 32 + 1). */
        uint32_t goff[32];
        if (!shared) {
          /* rows past the expert's end read token 0 (computed, never stored); a row index
           * outside [0, T * k) reads token 0 too and raises MOE_DEV_BOUNDS */
          const int r_end = ctl->off[t.g + 1];
          const int r0 = ctl->off[t.g] + t.m * 128 + row0;
          bool bad = false;
#pragma unroll
          for (int i2 = 0; i2 < 32; ++i2) {
            const int r = r0 + 4 * i2;
            uint32_t tok = r < r_end ? (uint32_t)__ldg(p.row_src + r) / (uint32_t)p.k : 0u;
            if (tok >= (uint32_t)p.T) {
              bad = true;
              tok = 0u;
            }
            goff[i2] = tok * row_bytes;
          }
          if (bad) raise_status(p.status, MOE_DEV_BOUNDS);
        }
        const uint32_t tx_bytes = shared ? C::STAGE_BYTES : C::B_BYTES;
        for (int kb = 0; kb < KB; ++kb) {
          int ok = 1, skip = 0;
          uint8_t* a_dst = sA + stage * HALF_TILE;
          uint8_t* b_dst = sB + stage * C::B_BYTES;
          if (lane == 0) {
            ok = mbar_wait(&ctl->empty[stage], phase ^ 1u, p.timeout_ns, s_abort) ? 1 : 0;
            if (ok) {
              mbar_arrive_expect_tx(&ctl->full[stage], tx_bytes);
              if (p.stall_first_stage && first && kb == 0) {
                skip = 1; /* test hook: this stage's bytes never arrive, so the MMA's bounded wait runs out */
              } else {
                armed[stage] = true;
                armed_phase[stage] = phase;
                /* the weights first: they come from DRAM, the rows of x mostly from L2 */
                const CUtensorMap* mB = shared ? &tmB1 : &tmB0;
                tma_load_2d(b_dst, mB, &ctl->full[stage], kb * BK, t.b_row);
                tma_load_2d(b_dst + HALF_TILE, mB, &ctl->full[stage], kb * BK, t.b_row + p.f);
                if (shared) tma_load_2d(a_dst, &tmA1, &ctl->full[stage], kb * BK, t.a_row);
              }
            }
          }
          ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
          skip = __shfl_sync(0xFFFFFFFFu, skip, 0);
          if (!ok) {
            abort = true;
            break;
          }
          if (!shared && !skip) {
            const uint32_t a_base = smem_u32(a_dst) + (uint32_t)row0 * 128u;
            const char* xk = xk0 + (int64_t)kb * (BK * 2);
#pragma unroll
            for (int i2 = 0; i2 < 32; ++i2)
              cp_async_16(a_base + (uint32_t)i2 * 512u + ((i2 & 1) ? sw_odd : sw_even), xk + goff[i2]);
          }
          cp_async_mbar_arrive(&ctl->full[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      first = false;
    }
    if (lane == 0) {
      if (abort) {
        raise_status(p.status, MOE_DEV_TIMEOUT);
        *s_abort = 1;
      }
      /* every armed stage's copies must land before the CTA may exit */
      for (int s = 0; s < STAGES; ++s)
        if (armed[s]) mbar_wait(&ctl->full[s], armed_phase[s], kDrainNs, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      /* ---------------- MMA issuer ---------------- */
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc = 0;
      bool abort = false;
      for (int i = 0;; ++i, ++acc) {
        int v;
        if (!read_tile_index(ctl, i, p.timeout_ns, s_abort, &v)) {
          abort = true;
          break;
        }
        mbar_arrive(&ctl->tq_empty[i % kTQ]);
        if (v < 0) break;
        const uint32_t b = acc & 1u, use = (acc >> 1) & 1u;
        if (!mbar_wait(&ctl->tempty[b], use ^ 1u, p.timeout_ns, s_abort)) {
          abort = true;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * C::ACC_COLS;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ctl->full[stage], phase, p.timeout_ns, s_abort)) {
            abort = true;
            break;
          }
          /* rows gathered by cp.async were written through the generic proxy: order them
           * before the tensor core reads the stage through the async proxy */
          if constexpr (GATHER) fence_proxy_async_shared();
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * HALF_TILE);
          const uint32_t b_addr = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            umma_bf16(d_tmem, umma_desc_sw128(a_addr + kk * 32), umma_desc_sw128(b_addr + kk * 32), C::IDESC,
                      (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&ctl->empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (abort) break;
        umma_commit(&ctl->tfull[b]);
      }
      if (abort) {
        raise_status(p.status, MOE_DEV_TIMEOUT);
        *s_abort = 1;
      }
      /* all issued MMAs must finish before TMEM is released */
      umma_commit(&ctl->drain);
      mbar_wait(&ctl->drain, 0, kDrainNs, nullptr);
    }
  } else {
    /* ---------------- epilogue (warps 2..5, 128 threads) ---------------- */
    const int q = warp & 3; /* TMEM lane quarter this warp may access */
    uint32_t acc = 0;
    for (int i = 0;; ++i, ++acc) {
      int v = -1;
      const bool got = read_tile_index(ctl, i, p.timeout_ns, s_abort, &v);
      __syncwarp();
      if (!got) {
        if (lane == 0) {
          raise_status(p.status, MOE_DEV_TIMEOUT);
          *s_abort = 1;
        }
        break;
      }
      if (lane == 0) mbar_arrive(&ctl->tq_empty[i % kTQ]);
      if (v < 0) break;
      const Tile t = decode_tile<MODE, 128, BN>(v, p, ctl->off, ctl->mpref, ctl->hpref);
      const uint32_t b = acc & 1u, use = (acc >> 1) & 1u;
      if (!mbar_wait(&ctl->tfull[b], use, p.timeout_ns, s_abort)) {
        if (lane == 0) {
          raise_status(p.status, MOE_DEV_TIMEOUT);
          *s_abort = 1;
        }
        break;
      }
      tc_fence_after();
      epilogue_warp<MODE, BN>(p, t, tmem_base + ((uint32_t)(q * 32) << 16) + b * C::ACC_COLS, q * 32, lane,
                              sEpi + q * kStageBytesPerWarp, &tmO0, &tmO1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->tempty[b]);
    }
    if (lane == 0) bulk_wait_all(); /* this warp's TMA stores are complete */
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
  if (threadIdx.x == 0) release_tile_counter(p);
}

/* ================= CTA-pair tiles (256 x 256, cta_group::2) ================= */

struct PairCfg {
  static constexpr int STAGES = 6;
  static constexpr uint32_t STAGE_BYTES = 2 * HALF_TILE;       /* per CTA: 128 rows of A + 128 rows of B */
  static constexpr uint32_t STAGE_TX = 2 * STAGE_BYTES;        /* bytes landing per stage in both CTAs */
  static constexpr uint32_t STAGE_TX_HALF = 2 * (HALF_TILE / 2 + HALF_TILE); /* 64 rows of A per CTA */
  static constexpr uint32_t ACC_COLS = 256;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t IDESC = umma_idesc_bf16(256, 256);
  static constexpr uint32_t IDESC_HALF = umma_idesc_bf16(128, 256);
  static constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + kEpiStagingBytes + sizeof(Ctrl);
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

/* A cluster of two CTAs (ranks 0 and 1) works on one tile of up to 256 rows x 256
 * columns. Full tile: rank r stages A rows [r*128, r*128+128) of the tile, holds
 * accumulator rows [r*128, +128) in its own TMEM, and the MMAs are M = 256. Half
 * tile (a group's last block of at most 128 rows): rank r stages A rows
 * [r*64, r*64+64) and the MMAs are M = 128, at half the cost. Either way rank r
 * stages 128 of the 256 B rows: GEMM2 rows [r*128, +128); GEMM1 the 64 gate rows
 * [n*128 + r*64, +64) of the tile's 128 h columns and the matching 64 up rows.
 * Rank 0 claims the tiles and writes each index into both CTAs' queues, arms the
 * stage barrier for the bytes of both CTAs and issues the MMAs; its commits arrive
 * on the barriers of both CTAs; rank 1's consumers release queue slots and
 * accumulators on rank 0's barriers. */
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    ffn_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                         const __grid_constant__ CUtensorMap tmA0h, const __grid_constant__ CUtensorMap tmA1h,
                         const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                         const __grid_constant__ CUtensorMap tmO0, const __grid_constant__ CUtensorMap tmO1,
                         const FfnParams p) {
  using C = PairCfg;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * HALF_TILE;
  uint8_t* sEpi = sB + STAGES * HALF_TILE;
  Ctrl* ctl = reinterpret_cast<Ctrl*>(sEpi + kEpiStagingBytes);
  volatile int* s_abort = &ctl->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->tfull[b], 1);
      mbar_init(&ctl->tempty[b], 8); /* 4 epilogue warps in each CTA */
    }
    for (int i = 0; i < kTQ; ++i) {
      mbar_init(&ctl->tq_full[i], 1);
      /* rank 0's barrier counts every consumer of a queue slot: its MMA issuer and 4
       * epilogue warps, rank 1's producer and 4 epilogue warps */
      mbar_init(&ctl->tq_empty[i], 10);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmA0h);
    tma_prefetch_desc(&tmA1h);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
    tma_prefetch_desc(&tmO0);
    tma_prefetch_desc(&tmO1);
  }
  if (warp == 1) {
    tmem_alloc_pair(&ctl->tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  pdl_wait(); /* expert_offsets and the A rows come from earlier kernels */
  pdl_trigger();
  if (warp == 2) {
    const bool ok = build_schedule<256>(p, ctl->off, ctl->mpref, ctl->hpref, lane);
    if (lane == 0) ctl->ok = ok ? 1 : 0;
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync(); /* both CTAs' barriers are initialised before any remote arrive */
  tc_fence_after();

  const uint32_t tmem_base = ctl->tmem_slot;
  const int G = p.E + p.n_shared;
  int64_t total = (int64_t)ctl->mpref[G] * p.n_tiles_n;
  if (!ctl->ok) {
    total = 0;
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(p.status, MOE_DEV_COUNT_MISMATCH);
  }
  const int KB = p.K / BK;
  /* a consumer releases a queue slot on rank 0's barrier */
  auto release_slot = [&](int i) {
    if (leader)
      mbar_arrive(&ctl->tq_empty[i % kTQ]);
    else
      mbar_arrive_cluster(mapa_shared(smem_u32(&ctl->tq_empty[i % kTQ]), 0));
  };

  if (warp == 0) {
    if (lane == 0) {
      /* ---------------- tile claimer (rank 0) and TMA producers (both CTAs) ---------------- */
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed_phase[STAGES];
      bool armed[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) {
        armed[s] = false;
        armed_phase[s] = 0;
      }
      bool abort = false;
      bool first = true;
      int next = leader ? claim_tile(p, total) : -1; /* claimed one tile ahead (see the single kernel) */
      for (int i = 0;; ++i) {
        const int slot = i % kTQ;
        int v = -1;
        if (leader) {
          if (!mbar_wait<true>(&ctl->tq_empty[slot], ((uint32_t)(i / kTQ) & 1u) ^ 1u, p.timeout_ns, s_abort)) {
            abort = true;
            break;
          }
          v = next;
          ctl->tq[slot] = v;
          st_shared_cluster_u32(mapa_shared(smem_u32(&ctl->tq[slot]), 1), (uint32_t)v);
          mbar_arrive(&ctl->tq_full[slot]);
          mbar_arrive_cluster(mapa_shared(smem_u32(&ctl->tq_full[slot]), 1)); /* release: orders the store */
          if (v >= 0) next = claim_tile(p, total);
        } else {
          if (!read_tile_index<true>(ctl, i, p.timeout_ns, s_abort, &v)) {
            abort = true;
            break;
          }
          release_slot(i);
        }
        if (v < 0) break;
        const Tile t = decode_tile<MODE, 256, 256>(v, p, ctl->off, ctl->mpref, ctl->hpref);
        const bool shared = t.g >= p.E;
        const CUtensorMap* mA = t.half ? (shared ? &tmA1h : &tmA0h) : (shared ? &tmA1 : &tmA0);
        const CUtensorMap* mB = shared ? &tmB1 : &tmB0;
        const int a_row = t.a_row + (int)rank * (t.half ? 64 : 128);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, p.timeout_ns, s_abort)) {
            abort = true;
            break;
          }
          const bool stall = p.stall_first_stage && first && kb == 0;
          if (leader) {
            mbar_arrive_expect_tx(&ctl->full[stage], t.half ? C::STAGE_TX_HALF : C::STAGE_TX);
            armed[stage] = !stall;
            armed_phase[stage] = phase;
          }
          if (stall) {
            /* test hook: this stage's bytes never arrive, so the MMA's bounded wait runs out */
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
            continue;
          }
          const uint32_t full_leader = mapa_shared(smem_u32(&ctl->full[stage]), 0);
          tma_load_2d_pair(sA + stage * HALF_TILE, mA, full_leader, kb * BK, a_row);
          if (MODE == 0) {
            /* 64 gate rows, then the matching 64 up rows */
            const int g_row = t.b_row + (int)rank * 64;
            tma_load_2d_pair(sB + stage * HALF_TILE, mB, full_leader, kb * BK, g_row);
            tma_load_2d_pair(sB + stage * HALF_TILE + HALF_TILE / 2, mB, full_leader, kb * BK, g_row + p.f);
          } else {
            tma_load_2d_pair(sB + stage * HALF_TILE, mB, full_leader, kb * BK, t.b_row + (int)rank * 128);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (abort) break;
        first = false;
      }
      if (!abort) {
        /* wait until the MMAs have released every stage this CTA filled, so no
         * commit is still on its way to this CTA's barriers when it exits */
        for (int i = 0; i < STAGES; ++i) {
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, p.timeout_ns, s_abort)) {
            abort = true;
            break;
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (abort) {
        raise_status(p.status, MOE_DEV_TIMEOUT);
        *s_abort = 1;
      }
      /* the leader's stage barriers count both CTAs' copies: wait for them to land */
      for (int s = 0; s < STAGES; ++s)
        if (armed[s]) mbar_wait(&ctl->full[s], armed_phase[s], kDrainNs, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      /* ---------------- MMA issuer (rank 0) ---------------- */
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc = 0;
      bool abort = false;
      for (int i = 0;; ++i, ++acc) {
        int v;
        if (!read_tile_index<true>(ctl, i, p.timeout_ns, s_abort, &v)) {
          abort = true;
          break;
        }
        release_slot(i);
        if (v < 0) break;
        const Tile t = decode_tile<MODE, 256, 256>(v, p, ctl->off, ctl->mpref, ctl->hpref);
        const uint32_t idesc = t.half ? C::IDESC_HALF : C::IDESC;
        const uint32_t b = acc & 1u, use = (acc >> 1) & 1u;
        if (!mbar_wait(&ctl->tempty[b], use ^ 1u, p.timeout_ns, s_abort)) {
          abort = true;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * C::ACC_COLS;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ctl->full[stage], phase, p.timeout_ns, s_abort)) {
            abort = true;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * HALF_TILE);
          const uint32_t b_addr = smem_u32(sB + stage * HALF_TILE);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            umma_bf16_pair(d_tmem, umma_desc_sw128(a_addr + kk * 32), umma_desc_sw128(b_addr + kk * 32), idesc,
                           (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair_mc(&ctl->empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (abort) break;
        umma_commit_pair_mc(&ctl->tfull[b], 0x3);
      }
      if (!abort) {
        /* both CTAs' epilogues have released both accumulators (so no remote
         * arrive is still on its way to this CTA) */
        for (int i = 0; i < 2; ++i, ++acc) {
          if (!mbar_wait(&ctl->tempty[acc & 1u], ((acc >> 1) & 1u) ^ 1u, p.timeout_ns, s_abort)) {
            abort = true;
            break;
          }
        }
      }
      if (abort) {
        raise_status(p.status, MOE_DEV_TIMEOUT);
        *s_abort = 1;
      }
      umma_commit_pair(&ctl->drain);
      mbar_wait(&ctl->drain, 0, kDrainNs, nullptr);
    }
  } else {
    /* ---------------- epilogue (warps 2..5 of both CTAs) ---------------- */
    const int q = warp & 3;
    uint32_t acc = 0;
    for (int i = 0;; ++i, ++acc) {
      int v = -1;
      const bool got = read_tile_index<true>(ctl, i, p.timeout_ns, s_abort, &v);
      __syncwarp();
      if (!got) {
        if (lane == 0) {
          raise_status(p.status, MOE_DEV_TIMEOUT);
          *s_abort = 1;
        }
        break;
      }
      if (lane == 0) release_slot(i);
      if (v < 0) break;
      const Tile t = decode_tile<MODE, 256, 256>(v, p, ctl->off, ctl->mpref, ctl->hpref);
      const uint32_t b = acc & 1u, use = (acc >> 1) & 1u;
      if (!mbar_wait(&ctl->tfull[b], use, p.timeout_ns, s_abort)) {
        if (lane == 0) {
          raise_status(p.status, MOE_DEV_TIMEOUT);
          *s_abort = 1;
        }
        break;
      }
      tc_fence_after();
      epilogue_pair_warp<MODE>(p, t, tmem_base + ((uint32_t)(q * 32) << 16) + b * C::ACC_COLS, q, rank, lane,
                               sEpi + q * kStageBytesPerWarp, &tmO0, &tmO1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&ctl->tempty[b]), 0));
    }
    if (lane == 0) bulk_wait_all(); /* this warp's TMA stores are complete */
  }

  __syncthreads();
  cluster_sync(); /* neither CTA releases TMEM or exits while its peer still works */
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
  if (threadIdx.x == 0) release_tile_counter(p);
}

/* ---- host side ------------------------------------------------------------ */

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

/* 2D bf16 tensor [rows, cols] row-major; box = box_rows x 64 columns, 128 B swizzle. */
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {BK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

/* The opt-in to more than 48 KB of dynamic shared memory is a property of the
 * kernel on one device: set it once per device (and kernel instantiation) before
 * the first launch there. A failed attempt is retried on the next launch. */
constexpr int kMaxDevices = 64;

template <typename Kernel>
cudaError_t smem_opt_in(std::atomic<int> (&done)[kMaxDevices], Kernel kernel, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done[dev].store(1, std::memory_order_release);
  return e;
}

template <int MODE, int BN, bool GATHER = false>
cudaError_t launch_single(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b0, const CUtensorMap& b1,
                          const CUtensorMap& o0, const CUtensorMap& o1, const CUtensorMap& a0r16,
                          const CUtensorMap& a0r32, const CUtensorMap& a0r64, const FfnParams& p,
                          cudaStream_t stream) {
  using C = SingleCfg<MODE, BN>;
  static std::atomic<int> attr_done[kMaxDevices];
  const cudaError_t attr_err = smem_opt_in(attr_done, ffn_gemm_single_kernel<MODE, BN, GATHER>, C::SMEM_BYTES);
  if (attr_err != cudaSuccess) return attr_err;
  return launch_kernel(ffn_gemm_single_kernel<MODE, BN, GATHER>, dim3((unsigned)num_sms()), dim3(kThreads),
                       C::SMEM_BYTES, stream, 1, a0, a1, b0, b1, o0, o1, a0r16, a0r32, a0r64, p);
}

/* Number of CTA pairs that can be resident at once (per device, cached). */
template <int MODE>
int pair_clusters() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * (unsigned)num_sms(), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = PairCfg::SMEM_BYTES;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaOccupancyMaxActiveClusters(&n, ffn_gemm_pair_kernel<MODE>, &cfg) != cudaSuccess) n = 0;
  if (n > num_sms() / 2) n = num_sms() / 2;
  if (n > 0) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

template <int MODE>
cudaError_t launch_pair(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& a0h, const CUtensorMap& a1h,
                        const CUtensorMap& b0, const CUtensorMap& b1, const CUtensorMap& o0, const CUtensorMap& o1,
                        const FfnParams& p, cudaStream_t stream, bool* launched) {
  *launched = false;
  static std::atomic<int> attr_done[kMaxDevices];
  const cudaError_t attr_err = smem_opt_in(attr_done, ffn_gemm_pair_kernel<MODE>, PairCfg::SMEM_BYTES);
  if (attr_err != cudaSuccess) return attr_err;
  const int clusters = pair_clusters<MODE>();
  if (debug_log()) std::fprintf(stderr, "[moe] pair GEMM%d: %d resident clusters of 2 CTAs\n", MODE + 1, clusters);
  if (clusters <= 0) return cudaSuccess; /* caller falls back to single-CTA tiles */
  const cudaError_t e = launch_kernel(ffn_gemm_pair_kernel<MODE>, dim3(2 * (unsigned)clusters), dim3(kThreads),
                                     PairCfg::SMEM_BYTES, stream, 2, a0, a1, a0h, a1h, b0, b1, o0, o1, p);
  if (e == cudaSuccess) *launched = true;
  return e;
}

FfnParams base_params(const moe_shape_t& s, const WsLayout& L, uint8_t* ws, const int32_t* expert_offsets,
                      size_t ctr_offset) {
  FfnParams p;
  p.expert_offsets = expert_offsets;
  p.E = s.E;
  p.n_shared = s.n_shared;
  p.T = s.T;
  p.A = L.A;
  p.f = s.f;
  p.d = s.d;
  p.status = reinterpret_cast<uint32_t*>(ws + L.status);
  p.timeout_ns = wait_timeout_ns();
  p.stall_first_stage = test_stall() ? 1 : 0;
  p.tile_ctr = reinterpret_cast<uint32_t*>(ws + L.status + ctr_offset);
  p.row_src = nullptr;
  p.gather_x = nullptr;
  p.k = s.k;
  p.fc_row_src = nullptr;
  p.fc_assign_row = nullptr;
  p.fc_gate = nullptr;
  p.fc_out = nullptr;
  p.fc_cnt = nullptr;
  return p;
}

}  // namespace

cudaError_t launch_gate_up(const moe_shape_t& s, const WsLayout& L, uint8_t* ws, const uint16_t* x_perm,
                           const int32_t* row_src, const int32_t* expert_offsets, const uint16_t* w13,
                           const uint16_t* x, const uint16_t* w13s, cudaStream_t stream) {
  if (s.T == 0) return cudaSuccess;
  const bool sh = s.n_shared != 0;
  const bool gather = x_perm == nullptr; /* A rows gathered from x through row_src */
  /* CTA-pair tiles when the experts average at least 1024 rows (each SM then stages a
   * third fewer operand bytes per K step, which is what holds this GEMM back at full
   * clock); single-CTA tiles otherwise, where short groups end in half-height pair
   * tiles that cost nearly as much as full ones. Never pairs when gathering rows. */
  const int pol = gather ? kGemmSingle : gemm_policy();
  const bool pair = pol == kGemmPair || (pol == kGemmAuto && L.A >= (int64_t)1024 * s.E);
  /* A = x_perm [A, d] (routed; rows of x gathered by the producer warp instead when x_perm is
   * null) / x [T, d] (shared); B = w13 [E*2f, d] / w13s [2f, d] */
  if (gather && (uint64_t)s.T * (uint64_t)s.d * 2u > 0xFFFFFFFFull) return cudaErrorInvalidValue;
  const uint16_t* a_routed = gather ? x : x_perm;
  const uint64_t a_rows = gather ? (uint64_t)s.T : (uint64_t)L.A;
  const uint16_t* a_sh = sh || gather ? x : x_perm;
  const uint64_t a_sh_rows = sh || gather ? (uint64_t)s.T : (uint64_t)L.A;
  const uint16_t* b_sh = sh ? w13s : w13;
  const uint64_t b_rows = (uint64_t)s.E * 2 * s.f, b_sh_rows = sh ? (uint64_t)2 * s.f : b_rows;
  CUtensorMap o0; /* h [h_rows, f], stored as 32 x 64 blocks */
  if (!make_map(&o0, ws + L.h, (uint64_t)L.h_rows, s.f, 32)) return cudaErrorInvalidValue;
  FfnParams p = base_params(s, L, ws, expert_offsets, kGemm1CtrOffset);
  p.K = s.d;
  p.n_tiles_n = s.f / 128;
  p.out0 = reinterpret_cast<uint16_t*>(ws + L.h);
  p.out1 = nullptr;
  p.ld_out = s.f;
  p.row_src = gather ? row_src : nullptr;
  p.gather_x = gather ? x : nullptr;
  CUtensorMap a0, a1, b0, b1;
  if (!make_map(&a0, a_routed, a_rows, s.d, 128) || !make_map(&a1, a_sh, a_sh_rows, s.d, 128))
    return cudaErrorInvalidValue;
  if (pair) {
    /* each CTA of a pair stages 64 gate and 64 up rows (64-row B boxes) and, in a
     * half-height tile, 64 rows of A (64-row A boxes) */
    CUtensorMap a0h, a1h;
    if (!make_map(&a0h, a_routed, a_rows, s.d, 64) || !make_map(&a1h, a_sh, a_sh_rows, s.d, 64) ||
        !make_map(&b0, w13, b_rows, s.d, 64) || !make_map(&b1, b_sh, b_sh_rows, s.d, 64))
      return cudaErrorInvalidValue;
    bool launched = false;
    const cudaError_t e = launch_pair<0>(a0, a1, a0h, a1h, b0, b1, o0, o0, p, stream, &launched);
    if (e != cudaSuccess || launched) return e;
  }
  if (!make_map(&b0, w13, b_rows, s.d, 128) || !make_map(&b1, b_sh, b_sh_rows, s.d, 128))
    return cudaErrorInvalidValue;
  if (gather) return launch_single<0, 256, true>(a0, a1, b0, b1, o0, o0, a0, a0, a0, p, stream);
  CUtensorMap a0r16, a0r32, a0r64; /* short A boxes for a group's last tile of <= 16 / 32 / 64 rows */
  if (!make_map(&a0r16, a_routed, a_rows, s.d, 16) || !make_map(&a0r32, a_routed, a_rows, s.d, 32) ||
      !make_map(&a0r64, a_routed, a_rows, s.d, 64))
    return cudaErrorInvalidValue;
  return launch_single<0, 256>(a0, a1, b0, b1, o0, o0, a0r16, a0r32, a0r64, p, stream);
}

cudaError_t launch_down(const moe_shape_t& s, const WsLayout& L, uint8_t* ws, const int32_t* expert_offsets,
                        const uint16_t* w2, const uint16_t* w2s, uint16_t* y_perm, uint16_t* y_shared,
                        cudaStream_t stream, const FusedCombine* fc) {
  if (s.T == 0) return cudaSuccess;
  const bool sh = s.n_shared != 0;
  const bool bn256 = (s.d % 256) == 0;
  /* CTA-pair tiles (256 output columns per tile) when every expert averages >= 1024
   * rows, or on request */
  const int pol = bn256 ? gemm_policy() : kGemmSingle;
  const bool pair = pol == kGemmPair || (pol == kGemmAuto && L.A >= (int64_t)1024 * s.E);
  const uint32_t bn = bn256 ? 256 : 128;
  const uint16_t* b_sh = sh ? w2s : w2;
  const uint64_t b_rows = (uint64_t)s.E * s.d, b_sh_rows = sh ? (uint64_t)s.d : b_rows;
  /* A = h [h_rows, f] (workspace); B = w2 [E*d, f] / w2s [d, f] */
  CUtensorMap a0, b0, b1;
  if (!make_map(&a0, ws + L.h, (uint64_t)L.h_rows, s.f, 128)) return cudaErrorInvalidValue;
  CUtensorMap o0, o1; /* y_perm [A, d] and y_shared [T, d], stored as 32 x 64 blocks */
  if (!make_map(&o0, y_perm, (uint64_t)L.A, s.d, 32)) return cudaErrorInvalidValue;
  if (!make_map(&o1, sh ? y_shared : y_perm, sh ? (uint64_t)s.T : (uint64_t)L.A, s.d, 32)) return cudaErrorInvalidValue;
  FfnParams p = base_params(s, L, ws, expert_offsets, kGemm2CtrOffset);
  p.K = s.f;
  p.n_tiles_n = s.d / (int)bn;
  p.out0 = y_perm;
  p.out1 = sh ? y_shared : nullptr;
  p.ld_out = s.d;
  if (fc) {
    p.fc_row_src = fc->row_src;
    p.fc_assign_row = fc->assign_row;
    p.fc_gate = fc->topk_gate;
    p.fc_out = fc->out;
    p.fc_cnt = reinterpret_cast<uint32_t*>(ws + L.fc_cnt);
  }
  if (pair) {
    CUtensorMap a0h;
    if (!make_map(&a0h, ws + L.h, (uint64_t)L.h_rows, s.f, 64) || !make_map(&b0, w2, b_rows, s.f, 128) ||
        !make_map(&b1, b_sh, b_sh_rows, s.f, 128))
      return cudaErrorInvalidValue;
    bool launched = false;
    const cudaError_t e = launch_pair<1>(a0, a0, a0h, a0h, b0, b1, o0, o1, p, stream, &launched);
    if (e != cudaSuccess || launched) return e;
  }
  if (!make_map(&b0, w2, b_rows, s.f, bn) || !make_map(&b1, b_sh, b_sh_rows, s.f, bn)) return cudaErrorInvalidValue;
  CUtensorMap a0r16, a0r32, a0r64; /* short A boxes (rows of h) for a group's last tile of <= 16 / 32 / 64 rows */
  if (!make_map(&a0r16, ws + L.h, (uint64_t)L.h_rows, s.f, 16) ||
      !make_map(&a0r32, ws + L.h, (uint64_t)L.h_rows, s.f, 32) ||
      !make_map(&a0r64, ws + L.h, (uint64_t)L.h_rows, s.f, 64))
    return cudaErrorInvalidValue;
  return bn256 ? launch_single<1, 256>(a0, a0, b0, b1, o0, o1, a0r16, a0r32, a0r64, p, stream)
               : launch_single<1, 128>(a0, a0, b0, b1, o0, o1, a0r16, a0r32, a0r64, p, stream);
}

}  // namespace moe
