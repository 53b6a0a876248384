/*
 * expert_ffn.cu -- the experts' SwiGLU FFN as two persistent grouped GEMMs on
 * the 5th-generation tensor cores (tcgen05.mma, TMEM accumulators, TMA loads).
 *
 * Page "Expert Parallelism" (learning-materials IX.05) §4 COMPUTE: "Grouped
 * GEMM: each expert processes its tokens ... many different-shaped GEMMs in one
 * launch"; §8: "A naive per-expert loop is far slower than a proper grouped
 * GEMM". The page "UltraEP ..." (thelatestinai.com/papers/2606.04101, the
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
 * expert_offsets, computes the m-tile prefix over the groups in shared memory,
 * and walks the linear tile index L = blockIdx.x, blockIdx.x + gridDim.x, ...
 * Inside a group the 128-row m-tiles are the inner index, so consecutive tiles
 * (running on neighbouring SMs at the same time) share one weight tile in L2.
 *
 * CTA = 6 warps: warp 0 issues TMA loads (one thread), warp 1 allocates TMEM
 * and issues tcgen05.mma (one thread), warps 2-5 drain the accumulator
 * (tcgen05.ld) and run the epilogue. 4-stage shared-memory ring (A 128x64 +
 * B 256x64 bf16 per stage, 128-byte swizzle), two TMEM accumulators of 128 x
 * 256 fp32 so the epilogue of tile i overlaps the main loop of tile i+1.
 * GEMM1's B tile stacks 128 gate rows over the matching 128 up rows, so one
 * N=256 MMA yields both halves of the SwiGLU for 128 output columns and the
 * epilogue combines them before anything leaves the SM.
 * The hidden rows h live in the workspace, padded to 128 rows per expert, so
 * GEMM1 stores whole tiles and GEMM2 loads whole tiles; GEMM2 masks its stores
 * to the expert's real rows.
 *
 * Every mbarrier wait is bounded (MOE_DEV_TIMEOUT on expiry); on abort each
 * role stops issuing, waits for its in-flight copies / MMAs, and the CTA frees
 * its TMEM before returning.
 */
#include <cudaTypedefs.h>

#include <mutex>

#include "moe_device.cuh"

namespace moe {

namespace {

constexpr int BM = 128;
constexpr int BK = 64; /* bf16 elements = 128 bytes = one swizzle row */
constexpr int STAGES = 4;
constexpr int kThreads = 192;
constexpr uint32_t A_BYTES = BM * BK * 2;
constexpr uint64_t kDrainNs = 2000000000ull;

template <int MODE, int BN>
struct Cfg {
  static constexpr int B_ROWS = (MODE == 0) ? 256 : BN; /* rows of W per tile (N of the MMA) */
  static constexpr int N_OUT = (MODE == 0) ? 128 : BN;  /* output columns per tile */
  static constexpr uint32_t B_BYTES = (uint32_t)B_ROWS * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t ACC_COLS = B_ROWS;
  static constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;
  static constexpr uint32_t IDESC = umma_idesc_bf16(BM, B_ROWS);
  static constexpr size_t SMEM_BYTES = 1024 /* alignment slack */ + (size_t)STAGES * STAGE_BYTES + 4096;
  static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation must be a power of two");
};

struct FfnParams {
  const int32_t* expert_offsets; /* [E+1] */
  int E;
  int n_shared;
  int64_t T;
  int64_t A;
  int K;           /* reduction length: d (GEMM1) or f (GEMM2) */
  int n_tiles_n;   /* output column tiles */
  int f;
  int d;
  uint16_t* out0;  /* GEMM1: h; GEMM2: y_perm */
  uint16_t* out1;  /* GEMM2: y_shared */
  int64_t ld_out;  /* row stride of the output in elements */
  uint32_t* status;
  uint64_t timeout_ns;
};

struct Tile {
  int g;           /* group: expert index, or E for the shared expert */
  int m, n;        /* m-tile inside the group, n-tile */
  int valid;       /* real rows in this m-tile (<= 128) */
  int a_row;       /* first A row (TMA coordinate) */
  int b_row;       /* first B row (TMA coordinate); GEMM1: the gate rows */
  int64_t out_row; /* first output row */
};

/* Shared-memory schedule: s_mpref[g] = m-tiles of groups < g (prefix, G+1 entries);
 * s_off = expert_offsets. */
__device__ __forceinline__ bool build_schedule(const FfnParams& p, int32_t* s_off, int32_t* s_mpref, int lane) {
  const int E = p.E;
  const int G = E + p.n_shared;
  bool ok = true;
  for (int i = lane; i <= E; i += 32) s_off[i] = __ldg(p.expert_offsets + i);
  __syncwarp();
  int carry = 0;
  for (int base = 0; base < G; base += 32) {
    const int g = base + lane;
    int mt = 0;
    if (g < E) {
      const int lo = s_off[g], hi = s_off[g + 1];
      if (lo < 0 || hi < lo || hi > p.A) ok = false;
      mt = (max(0, hi - lo) + BM - 1) / BM;
    } else if (g < G) {
      mt = (int)((p.T + BM - 1) / BM);
    }
    int incl = mt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    if (g < G) s_mpref[g + 1] = carry + incl;
    carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
  }
  if (lane == 0) {
    s_mpref[0] = 0;
    if (s_off[0] != 0) ok = false;
  }
  ok = __all_sync(0xFFFFFFFFu, ok);
  return ok;
}

template <int MODE, int BN>
__device__ __forceinline__ Tile decode_tile(int64_t L, const FfnParams& p, const int32_t* s_off,
                                            const int32_t* s_mpref) {
  const int G = p.E + p.n_shared;
  const int q = (int)(L / p.n_tiles_n); /* s_mpref[g] <= q < s_mpref[g+1] */
  int lo = 0, hi = G;                   /* find the last g with s_mpref[g] <= q */
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
  t.n = local / mt;
  t.m = local - t.n * mt;
  const bool shared = lo >= p.E;
  const int rows = shared ? (int)p.T : s_off[lo + 1] - s_off[lo];
  t.valid = min(BM, rows - t.m * BM);
  const int hrow = (s_mpref[lo] + t.m) * BM;
  if (MODE == 0) {
    t.a_row = shared ? t.m * BM : s_off[lo] + t.m * BM;
    t.b_row = shared ? t.n * 128 : lo * 2 * p.f + t.n * 128;
    t.out_row = hrow;
  } else {
    t.a_row = hrow;
    t.b_row = shared ? t.n * BN : lo * p.d + t.n * BN;
    t.out_row = shared ? (int64_t)t.m * BM : (int64_t)s_off[lo] + t.m * BM;
  }
  return t;
}

__device__ __forceinline__ float silu_f(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

template <int MODE, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_ffn_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                            const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                            const FfnParams p) {
  using C = Cfg<MODE, BN>;
  extern __shared__ uint8_t smem_raw[];
  /* 128-byte swizzled tiles need 1024-byte aligned shared-space addresses */
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * C::B_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_ok = reinterpret_cast<int*>(tmem_slot + 2);
  int32_t* s_off = reinterpret_cast<int32_t*>(tmem_slot + 4);
  int32_t* s_mpref = s_off + (kMaxE + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 2) {
    const bool ok = build_schedule(p, s_off, s_mpref, lane);
    if (lane == 0) *s_ok = ok ? 1 : 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = *tmem_slot;
  const int G = p.E + p.n_shared;
  int64_t total = (int64_t)s_mpref[G] * p.n_tiles_n;
  if (!*s_ok) {
    total = 0;
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(p.status, MOE_DEV_COUNT_MISMATCH);
  }
  const int KB = p.K / BK;

  if (warp == 0) {
    if (lane == 0) {
      /* ---------------- TMA producer ---------------- */
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
      for (int64_t L = blockIdx.x; L < total && !abort; L += gridDim.x) {
        const Tile t = decode_tile<MODE, BN>(L, p, s_off, s_mpref);
        const bool shared = t.g >= p.E;
        const CUtensorMap* mA = shared ? &tmA1 : &tmA0;
        const CUtensorMap* mB = shared ? &tmB1 : &tmB0;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.timeout_ns, s_abort)) {
            abort = true;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          armed[stage] = true;
          armed_phase[stage] = phase;
          uint8_t* a_dst = sA + stage * A_BYTES;
          uint8_t* b_dst = sB + stage * C::B_BYTES;
          tma_load_2d(a_dst, mA, &full[stage], kb * BK, t.a_row);
          if (MODE == 0) {
            tma_load_2d(b_dst, mB, &full[stage], kb * BK, t.b_row);
            tma_load_2d(b_dst + 128 * BK * 2, mB, &full[stage], kb * BK, t.b_row + p.f);
          } else {
            tma_load_2d(b_dst, mB, &full[stage], kb * BK, t.b_row);
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
      /* every armed stage's copies must land before the CTA may exit */
      for (int s = 0; s < STAGES; ++s)
        if (armed[s]) mbar_wait(&full[s], armed_phase[s], kDrainNs, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      /* ---------------- MMA issuer ---------------- */
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc = 0;
      bool abort = false;
      for (int64_t L = blockIdx.x; L < total && !abort; L += gridDim.x, ++acc) {
        const uint32_t b = acc & 1u, use = (acc >> 1) & 1u;
        if (!mbar_wait(&tempty[b], use ^ 1u, p.timeout_ns, s_abort)) {
          abort = true;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * C::ACC_COLS;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.timeout_ns, s_abort)) {
            abort = true;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            umma_bf16(d_tmem, umma_desc_sw128(a_addr + kk * 32), umma_desc_sw128(b_addr + kk * 32), C::IDESC,
                      (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (abort) break;
        umma_commit(&tfull[b]);
      }
      if (abort) {
        raise_status(p.status, MOE_DEV_TIMEOUT);
        *s_abort = 1;
      }
      /* all issued MMAs must finish before TMEM is released */
      umma_commit(drain);
      mbar_wait(drain, 0, kDrainNs, nullptr);
    }
  } else {
    /* ---------------- epilogue (warps 2..5, 128 threads) ---------------- */
    const int q = warp & 3; /* TMEM lane quarter this warp may access */
    const int row = q * 32 + lane;
    uint32_t acc = 0;
    for (int64_t L = blockIdx.x; L < total; L += gridDim.x, ++acc) {
      const Tile t = decode_tile<MODE, BN>(L, p, s_off, s_mpref);
      const uint32_t b = acc & 1u, use = (acc >> 1) & 1u;
      if (!mbar_wait(&tfull[b], use, p.timeout_ns, s_abort)) {
        if (lane == 0) {
          raise_status(p.status, MOE_DEV_TIMEOUT);
          *s_abort = 1;
        }
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + b * C::ACC_COLS;
      if (MODE == 0) {
        uint16_t* dst = p.out0 + (t.out_row + row) * p.ld_out + (int64_t)t.n * 128;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 16) {
          uint32_t gr[16], ur[16];
          tmem_ld16(taddr + c0, gr);
          tmem_ld16(taddr + 128 + c0, ur);
          tmem_ld_wait();
          uint32_t hw[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float h0 = silu_f(__uint_as_float(gr[2 * i])) * __uint_as_float(ur[2 * i]);
            const float h1 = silu_f(__uint_as_float(gr[2 * i + 1])) * __uint_as_float(ur[2 * i + 1]);
            hw[i] = pack_bf16x2(h0, h1);
          }
          st_v4(dst + c0, make_uint4(hw[0], hw[1], hw[2], hw[3]));
          st_v4(dst + c0 + 8, make_uint4(hw[4], hw[5], hw[6], hw[7]));
        }
      } else {
        const bool shared = t.g >= p.E;
        uint16_t* base = shared ? p.out1 : p.out0;
        uint16_t* dst = base + (t.out_row + row) * p.ld_out + (int64_t)t.n * BN;
        const bool live = row < t.valid;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          uint32_t vr[16];
          tmem_ld16(taddr + c0, vr);
          tmem_ld_wait();
          if (live) {
            uint32_t hw[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) hw[i] = pack_bf16x2(__uint_as_float(vr[2 * i]), __uint_as_float(vr[2 * i + 1]));
            st_v4(dst + c0, make_uint4(hw[0], hw[1], hw[2], hw[3]));
            st_v4(dst + c0 + 8, make_uint4(hw[4], hw[5], hw[6], hw[7]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[b]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
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

template <int MODE, int BN>
cudaError_t launch_gemm(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b0, const CUtensorMap& b1,
                        const FfnParams& p, cudaStream_t stream) {
  using C = Cfg<MODE, BN>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(grouped_ffn_gemm_kernel<MODE, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)C::SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return attr_err;
  grouped_ffn_gemm_kernel<MODE, BN><<<num_sms(), kThreads, C::SMEM_BYTES, stream>>>(a0, a1, b0, b1, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate_up(const moe_shape_t& s, const WsLayout& L, uint8_t* ws, const uint16_t* x_perm,
                           const int32_t* expert_offsets, const uint16_t* w13, const uint16_t* x,
                           const uint16_t* w13s, cudaStream_t stream) {
  if (s.T == 0) return cudaSuccess;
  const bool sh = s.n_shared != 0;
  CUtensorMap a0, a1, b0, b1;
  /* A = x_perm [A, d] (routed) / x [T, d] (shared); B = w13 [E*2f, d] / w13s [2f, d] */
  if (!make_map(&a0, x_perm, (uint64_t)L.A, s.d, BM)) return cudaErrorInvalidValue;
  if (!make_map(&a1, sh ? x : x_perm, sh ? (uint64_t)s.T : (uint64_t)L.A, s.d, BM)) return cudaErrorInvalidValue;
  if (!make_map(&b0, w13, (uint64_t)s.E * 2 * s.f, s.d, 128)) return cudaErrorInvalidValue;
  if (!make_map(&b1, sh ? w13s : w13, sh ? (uint64_t)2 * s.f : (uint64_t)s.E * 2 * s.f, s.d, 128))
    return cudaErrorInvalidValue;
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
  p.K = s.d;
  p.n_tiles_n = s.f / 128;
  p.out0 = reinterpret_cast<uint16_t*>(ws + L.h);
  p.out1 = nullptr;
  p.ld_out = s.f;
  return launch_gemm<0, 256>(a0, a1, b0, b1, p, stream);
}

cudaError_t launch_down(const moe_shape_t& s, const WsLayout& L, uint8_t* ws, const int32_t* expert_offsets,
                        const uint16_t* w2, const uint16_t* w2s, uint16_t* y_perm, uint16_t* y_shared,
                        cudaStream_t stream) {
  if (s.T == 0) return cudaSuccess;
  const bool sh = s.n_shared != 0;
  const bool bn256 = (s.d % 256) == 0;
  const uint32_t bn = bn256 ? 256 : 128;
  CUtensorMap a0, b0, b1;
  /* A = h [h_rows, f] (workspace); B = w2 [E*d, f] / w2s [d, f] */
  if (!make_map(&a0, ws + L.h, (uint64_t)L.h_rows, s.f, BM)) return cudaErrorInvalidValue;
  if (!make_map(&b0, w2, (uint64_t)s.E * s.d, s.f, bn)) return cudaErrorInvalidValue;
  if (!make_map(&b1, sh ? w2s : w2, sh ? (uint64_t)s.d : (uint64_t)s.E * s.d, s.f, bn)) return cudaErrorInvalidValue;
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
  p.K = s.f;
  p.n_tiles_n = s.d / (int)bn;
  p.out0 = y_perm;
  p.out1 = sh ? y_shared : nullptr;
  p.ld_out = s.d;
  return bn256 ? launch_gemm<1, 256>(a0, a0, b0, b1, p, stream) : launch_gemm<1, 128>(a0, a0, b0, b1, p, stream);
}

}  // namespace moe
