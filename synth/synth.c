/*
 * Seeded synthetic inputs for the batch-1 decoder workloads.
 *
 * This file holds only the input generator: counter-based random numbers,
 * the Gaussian transform and the rounding of each draw to the 16-bit
 * storage type.  It computes nothing of the decoder itself, and both the
 * oracle tests and the GPU path read the bytes it writes.
 *
 *   - SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014; constants as in Vigna's public-domain
 *     splitmix64.c): output n of the stream keyed by k is mix(k + (n+1)*gamma).
 *     Every draw is addressed by (seed, tensor index, element index), so the
 *     bytes do not depend on the thread count.
 *   - Box-Muller (Box & Muller 1958), cosine branch, in double.
 *   - Round to nearest, ties to even, into IEEE binary16 or bfloat16, written
 *     from the format definitions (sign, biased exponent, fraction).
 *   - Token ids: Lemire's multiply-shift range reduction of the top 32 bits.
 *   - FNV-1a 64-bit hash of a byte range (Fowler/Noll/Vo), for checksums.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t sm64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Output n (0-based) of the SplitMix64 stream whose state starts at key. */
static inline uint64_t sm64_at(uint64_t key, uint64_t n) {
  return sm64_mix(key + (n + 1) * GOLDEN_GAMMA);
}

/* Key of one tensor: the seed and the tensor index are each scrambled so
 * that neighbouring seeds or indices give unrelated streams. */
static inline uint64_t tensor_key(uint64_t seed, uint64_t tensor) {
  return sm64_mix(seed * GOLDEN_GAMMA + 0x632BE59BD9B4E019ULL) ^
         sm64_mix((tensor + 1) * 0xD1B54A32D192ED03ULL);
}

/* Uniform in (0,1) from the top 53 bits; never 0, so log() is finite. */
static inline double u53(uint64_t z) {
  return ((double)(z >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

/* Round a double to an IEEE-754 binary16 bit pattern (round half to even). */
static uint16_t f64_to_f16_rne(double x) {
  uint16_t sign = signbit(x) ? 0x8000u : 0u;
  double a = fabs(x);
  if (isnan(x)) return 0x7E00u;
  if (isinf(a) || a >= 65520.0) return sign | 0x7C00u; /* 65520 = halfway past max */
  if (a < 6.103515625e-05) {                         /* below 2^-14: subnormal */
    double m = nearbyint(a * 16777216.0);            /* units of 2^-24 */
    return sign | (uint16_t)m;                        /* m == 1024 -> min normal */
  }
  int e2;
  double f = frexp(a, &e2); /* a = f * 2^e2, f in [0.5, 1) */
  int e = e2 - 1;           /* a = 1.xxx * 2^e */
  double m = nearbyint(ldexp(f, 11)); /* 11 significant bits, in [1024, 2048] */
  if (m >= 2048.0) { m = 1024.0; e += 1; }
  if (e + 15 >= 31) return sign | 0x7C00u;
  return sign | (uint16_t)((e + 15) << 10) | (uint16_t)((int)m - 1024);
}

/* Round a double to a bfloat16 bit pattern (1 sign, 8 exponent, 7 fraction). */
static uint16_t f64_to_bf16_rne(double x) {
  uint16_t sign = signbit(x) ? 0x8000u : 0u;
  double a = fabs(x);
  if (isnan(x)) return 0x7FC0u;
  if (isinf(a)) return sign | 0x7F80u;
  if (a < 1.1754943508222875e-38) {                   /* below 2^-126 */
    double m = nearbyint(ldexp(a, 133));              /* units of 2^-133 */
    return sign | (uint16_t)m;
  }
  int e2;
  double f = frexp(a, &e2);
  int e = e2 - 1;
  double m = nearbyint(ldexp(f, 8)); /* 8 significant bits, in [128, 256] */
  if (m >= 256.0) { m = 128.0; e += 1; }
  if (e + 127 >= 255) return sign | 0x7F80u;
  return sign | (uint16_t)((e + 127) << 7) | (uint16_t)((int)m - 128);
}

uint16_t synth_round_f16(double x) { return f64_to_f16_rne(x); }
uint16_t synth_round_bf16(double x) { return f64_to_bf16_rne(x); }

/*
 * Fill out[0..n) with  mean + std * N(0,1)  rounded to the storage type
 * (dtype 0 = binary16, 1 = bfloat16).  std == 0 writes the constant mean.
 * Element i of the tensor uses stream outputs 2*i and 2*i+1.
 */
void synth_fill_normal(uint16_t *out, int64_t n, uint64_t seed, uint64_t tensor,
                       double mean, double std, int dtype) {
  const uint64_t key = tensor_key(seed, tensor);
  const double two_pi = 6.283185307179586476925286766559;
#pragma omp parallel for schedule(static, 65536)
  for (int64_t i = 0; i < n; ++i) {
    double v = mean;
    if (std != 0.0) {
      double u1 = u53(sm64_at(key, 2 * (uint64_t)i));
      double u2 = u53(sm64_at(key, 2 * (uint64_t)i + 1));
      v = mean + std * (sqrt(-2.0 * log(u1)) * cos(two_pi * u2));
    }
    out[i] = dtype == 0 ? f64_to_f16_rne(v) : f64_to_bf16_rne(v);
  }
}

/* Uniform token ids in [0, vocab) for a prompt or a forced-token sequence. */
void synth_fill_tokens(int32_t *out, int64_t n, uint64_t seed, uint64_t stream,
                       int32_t vocab) {
  const uint64_t key = tensor_key(seed, stream);
  for (int64_t i = 0; i < n; ++i) {
    uint64_t hi = sm64_at(key, (uint64_t)i) >> 32;
    out[i] = (int32_t)((hi * (uint64_t)vocab) >> 32);
  }
}

/* FNV-1a, 64-bit, over n bytes, continuing from h (start with the offset
 * basis 0xcbf29ce484222325). */
uint64_t synth_fnv1a64(const void *data, int64_t n, uint64_t h) {
  const unsigned char *p = (const unsigned char *)data;
  for (int64_t i = 0; i < n; ++i) {
    h ^= p[i];
    h *= 0x100000001B3ULL;
  }
  return h;
}
