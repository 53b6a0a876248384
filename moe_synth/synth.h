/*
 * moe_synth/synth.h -- seeded, counter-based synthetic inputs for the MoE layer.
 *
 * This module is shared by the CUDA path's tests/bench and by the CPU oracle's
 * tests. It holds no arithmetic of the MoE method itself: it only turns
 * (seed, tensor id, element index) into a value. Every element is a pure
 * function of its index, so any subset (one expert's weights, one token's
 * logits) can be regenerated on either side without generating the rest.
 *
 * Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014) used in counter mode:
 *     bits(key, i) = mix64(key + (i + 1) * GAMMA)
 * with mix64 the SplitMix64 output finaliser and GAMMA = 0x9E3779B97F4A7C15.
 *
 * Value distribution: an Irwin-Hall sum of four independent 16-bit uniforms,
 * centred: s = u0+u1+u2+u3 - 2*65535, an integer in [-131070, 131070] with
 * variance 4*(65536^2 - 1)/12. It is close to a normal (CLT with 4 terms, tails
 * truncated at about 3.46 sigma). The element value is
 *     float(s) * c            (one IEEE fp32 multiply, c = scale / sigma_s)
 * optionally followed by one IEEE fp32 add of a per-column bias. float(s) is
 * exact (|s| < 2^24), so the CPU and the GPU produce bit-identical values:
 * no transcendental function is involved. bf16 values are the fp32 value
 * rounded to nearest-even.
 *
 * This header compiles as C (gcc) and as CUDA (nvcc, host + device).
 */
#ifndef MOE_SYNTH_H
#define MOE_SYNTH_H

#include <stdint.h>

#if defined(__CUDACC__)
#define SYNTH_FN static __host__ __device__ __forceinline__
#else
#define SYNTH_FN static inline
#endif

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ull
/* standard deviation of the centred Irwin-Hall(4) integer: sqrt(4*(65536^2-1)/12) */
#define SYNTH_IH4_SIGMA 37837.2265747413

/* tensor ids: one independent stream per input tensor */
enum {
  SYNTH_X = 1,      /* token activations x [T, d] */
  SYNTH_LOGITS = 2, /* router logits [T, E] */
  SYNTH_W13 = 3,    /* routed gate/up weights [E, 2f, d] */
  SYNTH_W2 = 4,     /* routed down weights [E, d, f] */
  SYNTH_W13S = 5,   /* shared-expert gate/up weights [2f, d] */
  SYNTH_W2S = 6,    /* shared-expert down weights [d, f] */
  SYNTH_PERM = 7    /* keys of the expert popularity permutation */
};

SYNTH_FN uint64_t synth_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* per-(seed, tensor) stream key */
SYNTH_FN uint64_t synth_key(uint64_t seed, uint32_t tensor_id) {
  return synth_mix64(synth_mix64(seed + SYNTH_GAMMA) ^ ((uint64_t)tensor_id * 0xD1B54A32D192ED03ull));
}

/* 64 random bits for element i of the stream */
SYNTH_FN uint64_t synth_bits(uint64_t key, uint64_t i) {
  return synth_mix64(key + (i + 1ull) * SYNTH_GAMMA);
}

/* centred Irwin-Hall(4) integer in [-131070, 131070] */
SYNTH_FN int32_t synth_ih4(uint64_t b) {
  return (int32_t)(b & 0xFFFFu) + (int32_t)((b >> 16) & 0xFFFFu) +
         (int32_t)((b >> 32) & 0xFFFFu) + (int32_t)(b >> 48) - 131070;
}

/* fp32 -> bf16 bits, round to nearest even (finite inputs) */
SYNTH_FN uint16_t synth_f32_to_bf16(float v) {
  union { float f; uint32_t u; } c;
  c.f = v;
  uint32_t u = c.u;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

#endif /* MOE_SYNTH_H */
