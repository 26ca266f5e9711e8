/*
 * skvgen/core.h -- seeded, counter-based synthetic input generator.
 *
 * Shared verbatim by the host generator (host.c, used to build the oracle's
 * inputs) and the device generator (device.cu, used to fill GPU buffers), so
 * that both produce bit-identical tensors.  It holds no attention arithmetic:
 * only random numbers and the workload recipe (sink / heavy-token structure,
 * Gaussian-mixture keys and their centroids).
 *
 * Random numbers: SplitMix64 (S. Vigna, "Further scramblings of Marsaglia's
 * xorshift generators", 2015 / the public splitmix64.c), used as a counter-based
 * hash: value(key, i) = splitmix64 output number i of a generator seeded with
 * `key`.  A "normal" value is Irwin-Hall(12) - 6 built from twelve 21-bit
 * uniforms taken from four such outputs: mean 0, variance 1, range [-6, 6],
 * exact in fp32, rounded to bf16 by round-to-nearest-even in integer code.
 *
 * All floating-point recipe steps run in IEEE fp64 with explicit
 * round-to-nearest operations (no contraction), so host and device agree to
 * the bit.  fp64 -> bf16 rounding is done in integer code.
 */
#ifndef SKVGEN_CORE_H
#define SKVGEN_CORE_H

#include <stdint.h>

#if defined(__CUDACC__)
#define SKVG_HD __host__ __device__ __forceinline__
#else
#define SKVG_HD static inline
#endif

#if defined(__CUDA_ARCH__)
#define SKVG_DADD(a, b) __dadd_rn((a), (b))
#define SKVG_DMUL(a, b) __dmul_rn((a), (b))
#define SKVG_DDIV(a, b) __ddiv_rn((a), (b))
#define SKVG_DSQRT(a) __dsqrt_rn((a))
#else
#include <math.h>
#define SKVG_DADD(a, b) ((a) + (b))
#define SKVG_DMUL(a, b) ((a) * (b))
#define SKVG_DDIV(a, b) ((a) / (b))
#define SKVG_DSQRT(a) sqrt((a))
#endif

/* Stream ids: which tensor a counter belongs to. */
enum {
  SKVG_S_Q = 1,
  SKVG_S_K = 2,
  SKVG_S_V = 3,
  SKVG_S_CENTER = 4,
  SKVG_S_ASSIGN = 5,
  SKVG_S_PERM = 6,
  SKVG_S_HEAVY = 7,
  SKVG_S_ROUTE = 8,
  SKVG_S_KCHUNK = 9, /* keys/values of a query chunk's own tokens */
  SKVG_S_VCHUNK = 10
};

#define SKVG_GOLDEN 0x9E3779B97F4A7C15ull

/* SplitMix64 output function applied to state z (state already advanced). */
SKVG_HD uint64_t skvg_fmix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* Output number i (0-based) of SplitMix64 seeded with `key`. */
SKVG_HD uint64_t skvg_hash(uint64_t key, uint64_t i) {
  return skvg_fmix(key + (i + 1ull) * SKVG_GOLDEN);
}

/* Per-tensor key: seed, stream id and layer index mixed into one 64-bit key. */
SKVG_HD uint64_t skvg_key(uint64_t seed, uint32_t stream, uint32_t layer) {
  return skvg_hash(seed ^ ((uint64_t)stream << 48) ^ ((uint64_t)layer << 32), 0);
}

/* Irwin-Hall(12) - 6 as an exact fp32 value. */
SKVG_HD float skvg_normal(uint64_t key, uint64_t idx) {
  const uint64_t m21 = (1ull << 21) - 1ull;
  int32_t s = 0;
  for (int j = 0; j < 4; ++j) {
    uint64_t h = skvg_hash(key, idx * 4ull + (uint64_t)j);
    s += (int32_t)(h & m21) + (int32_t)((h >> 21) & m21) + (int32_t)((h >> 42) & m21);
  }
  s -= 6 * (1 << 21);
  return (float)s * (1.0f / 2097152.0f); /* |s| < 2^24: exact */
}

SKVG_HD uint32_t skvg_f32_bits(float f) {
  union { float f; uint32_t u; } c;
  c.f = f;
  return c.u;
}
SKVG_HD uint64_t skvg_f64_bits(double f) {
  union { double f; uint64_t u; } c;
  c.f = f;
  return c.u;
}
SKVG_HD float skvg_bits_f32(uint32_t u) {
  union { float f; uint32_t u; } c;
  c.u = u;
  return c.f;
}

/* fp32 -> bf16, round to nearest even (NaN -> canonical quiet NaN). */
SKVG_HD uint16_t skvg_f32_to_bf16(float f) {
  uint32_t u = skvg_f32_bits(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)0x7FC0u;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

SKVG_HD double skvg_bf16_to_f64(uint16_t h) { return (double)skvg_bits_f32((uint32_t)h << 16); }

/* fp64 -> bf16, one correctly rounded step (nearest even), integer code. */
SKVG_HD uint16_t skvg_f64_to_bf16(double x) {
  uint64_t b = skvg_f64_bits(x);
  uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
  uint64_t a = b & 0x7FFFFFFFFFFFFFFFull;
  if (a > 0x7FF0000000000000ull) return (uint16_t)0x7FC0u; /* NaN */
  if (a == 0x7FF0000000000000ull) return (uint16_t)(sign | 0x7F80u);
  if (a == 0) return sign;
  int e = (int)(a >> 52) - 1023;
  uint64_t m = a & ((1ull << 52) - 1ull);
  if (e >= -126) {
    if (e > 127) return (uint16_t)(sign | 0x7F80u);
    uint32_t keep = (uint32_t)(m >> 45);
    uint64_t rem = m & ((1ull << 45) - 1ull);
    uint64_t half = 1ull << 44;
    uint32_t r = ((uint32_t)(e + 127) << 7) | keep;
    if (rem > half || (rem == half && (keep & 1u))) r += 1u; /* carry may reach inf */
    return (uint16_t)(sign | r);
  }
  /* bf16 subnormal: units of 2^-133; |x| * 2^133 is exact in fp64 here. */
  {
    double s = SKVG_DMUL(x < 0 ? -x : x, 10889035741470030830827987437816582766592.0); /* 2^133 */
    uint64_t q = (uint64_t)s; /* floor */
    double fr = SKVG_DADD(s, -(double)q);
    if (fr > 0.5 || (fr == 0.5 && (q & 1ull))) q += 1ull;
    return (uint16_t)(sign | (uint16_t)q); /* q == 128 becomes the smallest normal */
  }
}

/* bf16 "normal" sample. */
SKVG_HD uint16_t skvg_normal_bf16(uint64_t key, uint64_t idx) {
  return skvg_f32_to_bf16(skvg_normal(key, idx));
}

/* Heavy-token test: each token t in [1, L) of a KV group is "heavy" with
 * probability 42949673 / 2^32 (= 1.0000000 %), independently. */
SKVG_HD int skvg_is_heavy(uint64_t key_heavy, uint64_t group, uint64_t L, uint64_t t) {
  if (t == 0) return 0;
  uint64_t h = skvg_hash(key_heavy, group * L + t);
  return (uint32_t)(h >> 32) < 42949673u;
}

/* Structured key element: base bf16 value k plus coef * qhat_j (fp64), rounded
 * once to bf16.  coef is 6 for token 0 (attention sink), 4 for heavy tokens. */
SKVG_HD uint16_t skvg_shift_bf16(uint16_t k, double coef, double qhat_j) {
  return skvg_f64_to_bf16(SKVG_DADD(skvg_bf16_to_f64(k), SKVG_DMUL(coef, qhat_j)));
}

/* Mixture component of slot i (uniform over 1024 components: top 10 bits). */
SKVG_HD uint32_t skvg_component(uint64_t key_assign, uint64_t group, uint64_t L, uint64_t i,
                                uint32_t n_comp_log2) {
  return (uint32_t)(skvg_hash(key_assign, group * L + i) >> (64 - n_comp_log2));
}

/* Mixture key element: center (bf16) + 0.3 * noise, fp64, rounded once. */
SKVG_HD uint16_t skvg_mixture_key(uint16_t center, float noise) {
  return skvg_f64_to_bf16(SKVG_DADD(skvg_bf16_to_f64(center), SKVG_DMUL(0.3, (double)noise)));
}

/* Route bit of layer l: 1 = full attention (+ART), 0 = sink + recent window. */
SKVG_HD int skvg_route_bit(uint64_t key_route, uint64_t layer) {
  return (int)(skvg_hash(key_route, layer) >> 63);
}

#endif /* SKVGEN_CORE_H */
