/*
 * synth.h - seeded, counter-based input generator.
 *
 * This module produces every synthetic input of the decode step: model
 * weights, norm gains, fp8 expert codes and their block scales, the
 * pre-filled KV context, prompt / decode tokens and speculative proposals.
 * It holds none of the decoder's arithmetic.  The same header is compiled
 * by gcc (CPU oracle, host-side test helpers) and by nvcc (device fill
 * kernels), so both sides see bit-identical bytes for the same
 * (seed, stream, index) triple.
 *
 * Generator core: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014).  Output i of a stream with
 * key K is mix64(K + (i + 1) * gamma), which makes it random-access.
 *
 * Normal deviates: Irwin-Hall sum of the four 16-bit lanes of one 64-bit
 * output, centred (an integer in [-131070, 131070], exact in fp32) and
 * multiplied once in fp32 by a scale = sigma / std(sum).  Rounding to bf16 is
 * round-to-nearest-even on the fp32 bit pattern.  Every floating-point step
 * is a single IEEE operation (no contraction), so host and device agree.
 */
#ifndef MK_SYNTH_H
#define MK_SYNTH_H

#include <stdint.h>
#include <string.h>

#if defined(__CUDACC__)
#define SYN_FN __host__ __device__ static inline
#else
#define SYN_FN static inline
#endif

#define SYN_GAMMA 0x9E3779B97F4A7C15ULL

/* Tensor kinds: the stream id of a tensor is (kind, layer, expert). */
enum syn_kind {
  SYN_EMBED = 1,
  SYN_ATTN_NORM = 2,
  SYN_WQKV = 3,       /* dense attention: rows q(Hq*d) | k(Hkv*d) | v(Hkv*d), cols H */
  SYN_WO = 4,         /* [H, Hq*d] */
  SYN_FFN_NORM = 5,
  SYN_WGATE = 6,      /* [I, H] */
  SYN_WUP = 7,        /* [I, H] */
  SYN_WDOWN = 8,      /* [H, I] */
  SYN_ROUTER = 9,     /* [E, H] */
  SYN_SH_GATE = 10,   /* shared expert j: expert index = j */
  SYN_SH_UP = 11,
  SYN_SH_DOWN = 12,
  SYN_EX_GATE = 13,   /* routed expert e */
  SYN_EX_UP = 14,
  SYN_EX_DOWN = 15,
  SYN_FINAL_NORM = 16,
  SYN_LM_HEAD = 17,   /* [V, H] */
  SYN_MLA_WQ = 18,    /* [Hq*(dn+dr), H], per head rows: nope(dn) | rope(dr) */
  SYN_MLA_WDKV = 19,  /* [R+dr, H], rows: latent c (R) | shared rope key (dr) */
  SYN_MLA_WUK = 20,   /* [Hq*dn, R] */
  SYN_MLA_WUV = 21,   /* [Hq*dv, R] */
  SYN_FP8_SCALE = 22, /* block scales of an fp8 matrix; expert/kind packed below */
  SYN_KV_K = 23,      /* synthetic pre-filled context: keys */
  SYN_KV_V = 24,      /* values */
  SYN_KV_LAT = 25,    /* latent cache rows [c | k_rope] */
  SYN_TOKENS = 26,
  SYN_PROPOSALS = 27
};

SYN_FN uint64_t syn_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

SYN_FN uint64_t syn_stream(uint32_t kind, uint32_t layer, uint32_t expert) {
  return ((uint64_t)kind << 48) ^ ((uint64_t)(layer & 0xFFFFFF) << 24) ^ (uint64_t)(expert & 0xFFFFFF);
}

/* Key of one stream under one seed. */
SYN_FN uint64_t syn_key(uint64_t seed, uint64_t stream) {
  return syn_mix64(seed * SYN_GAMMA + syn_mix64(stream + SYN_GAMMA));
}

/* Output i of the stream. */
SYN_FN uint64_t syn_u64(uint64_t key, uint64_t i) {
  return syn_mix64(key + (i + 1ULL) * SYN_GAMMA);
}

/* Centred Irwin-Hall(4) integer of one output. */
SYN_FN int32_t syn_ih4(uint64_t u) {
  uint32_t s = (uint32_t)(u & 0xFFFFu) + (uint32_t)((u >> 16) & 0xFFFFu) +
               (uint32_t)((u >> 32) & 0xFFFFu) + (uint32_t)(u >> 48);
  return (int32_t)s - 131070;
}

/* std of the centred sum: sqrt(4 * (65536^2 - 1) / 12). */
SYN_FN double syn_ih4_std(void) { return 37837.22690186340; }

/* fp32 multiplier turning the integer into N(0, sigma^2). Host-side only. */
static inline float syn_normal_scale(double sigma) {
  return (float)(sigma / 37837.22690186340);
}

SYN_FN float syn_fmul(float a, float b) {
#if defined(__CUDA_ARCH__)
  return __fmul_rn(a, b);
#else
  return a * b;
#endif
}

SYN_FN float syn_fadd(float a, float b) {
#if defined(__CUDA_ARCH__)
  return __fadd_rn(a, b);
#else
  return a + b;
#endif
}

SYN_FN uint32_t syn_f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
SYN_FN float syn_u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* fp32 -> bf16 bits, round to nearest even (finite inputs only). */
SYN_FN uint16_t syn_bf16_rne(float f) {
  uint32_t b = syn_f2u(f);
  b += 0x7FFFu + ((b >> 16) & 1u);
  return (uint16_t)(b >> 16);
}

/* Normal weight as bf16 bits. */
SYN_FN uint16_t syn_bf16_normal(uint64_t key, uint64_t i, float scale) {
  return syn_bf16_rne(syn_fmul((float)syn_ih4(syn_u64(key, i)), scale));
}

/* Norm gain 1 + normal(sigma) as bf16 bits (exactly 1.0 when scale == 0). */
SYN_FN uint16_t syn_bf16_gain(uint64_t key, uint64_t i, float scale) {
  return syn_bf16_rne(syn_fadd(1.0f, syn_fmul((float)syn_ih4(syn_u64(key, i)), scale)));
}

/*
 * fp32 -> OCP FP8 E4M3 code, round to nearest even, saturating at 448.
 * Used only to generate expert weight codes.
 */
SYN_FN uint8_t syn_e4m3_rne(float f) {
  uint32_t bits = syn_f2u(f);
  uint8_t sign = (uint8_t)((bits >> 31) << 7);
  uint32_t a = bits & 0x7FFFFFFFu;
  if (a >= 0x43E80000u) return (uint8_t)(sign | 0x7E); /* >= 464: saturate to 448 */
  int e = (int)(a >> 23) - 127;                            /* unbiased exponent */
  if (e < -6) {                                            /* subnormal range: unit 2^-9 */
    /* value * 2^9, exact scaling; round half to even on the integer part */
    float v = syn_fmul(syn_u2f(a), 512.0f);
    uint32_t q = (uint32_t)v;
    float frac = v - (float)q;
    if (frac > 0.5f || (frac == 0.5f && (q & 1u))) q += 1u;
    return (uint8_t)(sign | q); /* q == 8 is the smallest normal, code 0x08 */
  }
  /* normal: keep 3 mantissa bits, RNE on the 20 dropped bits */
  uint32_t m = a & 0x7FFFFFu;
  uint32_t keep = m >> 20, rest = m & 0xFFFFFu;
  if (rest > 0x80000u || (rest == 0x80000u && (keep & 1u))) keep += 1u;
  uint32_t code = ((uint32_t)(e + 7) << 3) + keep; /* carry into the exponent is intended */
  if (code > 0x7Eu) code = 0x7Eu;
  return (uint8_t)(sign | code);
}

/* Expert weight code: e4m3(N(0,1) * 16). `scale` = syn_normal_scale(16.0). */
SYN_FN uint8_t syn_e4m3_normal(uint64_t key, uint64_t i, float scale) {
  return syn_e4m3_rne(syn_fmul((float)syn_ih4(syn_u64(key, i)), scale));
}

/* Block scale: base * (1 + j/8), j in 0..7 -> one fp32 rounding. */
SYN_FN float syn_block_scale(uint64_t key, uint64_t blk, float base) {
  uint32_t j = (uint32_t)(syn_u64(key, blk) >> 61);
  return syn_fmul(base, 1.0f + 0.125f * (float)j);
}

/* Uniform token in [0, V). */
SYN_FN int32_t syn_token(uint64_t key, uint64_t i, uint32_t V) {
  return (int32_t)(((syn_u64(key, i) >> 32) * (uint64_t)V) >> 32);
}

#endif /* MK_SYNTH_H */
