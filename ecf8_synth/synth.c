/*
 * Seeded synthetic FP8 E4M3 weight tensors: the inputs that both the CPU
 * oracle and the GPU decoder are checked and timed on.
 *
 * This file holds no part of the codec: it only draws numbers and casts them
 * to E4M3 bytes.  Every value is a pure function of (seed, element index), so
 * any slice of any tensor can be regenerated on its own and in parallel.
 *
 * Distributions ("To Compress or Not? ... Exponent Concentration", p1 §2.1 of
 * the ECF8 walkthrough): trained weights follow a symmetric alpha-stable law
 * S_alpha(beta=0, gamma, delta) with alpha in [1.5, 2.0]; alpha = 2 is the
 * Gaussian.  The samplers below are textbook methods, named where used.
 *
 * Counter-based generator: SplitMix64 (Steele, Lea, Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014) applied to
 * seed + (counter + 1) * golden_gamma.  Element i draws counters 2i and 2i+1.
 */
#include <math.h>
#include <string.h>
#include <stdint.h>
#include <stddef.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t splitmix64_at(uint64_t seed, uint64_t counter) {
  uint64_t z = seed + (counter + 1) * GOLDEN_GAMMA;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Uniform double strictly inside (0, 1): the top 53 bits plus one half ulp. */
static inline double uniform_open(uint64_t seed, uint64_t counter) {
  return ((double)(splitmix64_at(seed, counter) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

uint64_t synth_splitmix64(uint64_t seed, uint64_t counter) { return splitmix64_at(seed, counter); }
double synth_uniform(uint64_t seed, uint64_t counter) { return uniform_open(seed, counter); }

/* Standard normal by Box-Muller (1958): sqrt(-2 ln u1) cos(2 pi u2). */
static inline double normal_at(uint64_t seed, uint64_t i) {
  double u1 = uniform_open(seed, 2 * i), u2 = uniform_open(seed, 2 * i + 1);
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

/* Symmetric alpha-stable, gamma = 1, by Chambers, Mallows and Stuck (1976):
 * V ~ U(-pi/2, pi/2), W ~ Exp(1),
 * X = sin(aV) / cos(V)^(1/a) * (cos(V - aV) / W)^((1 - a) / a).
 * For a = 2 this is 2 sin(V) sqrt(W), a N(0, 2) variate. */
static inline double sas_at(uint64_t seed, uint64_t i, double a) {
  double v = 3.141592653589793 * (uniform_open(seed, 2 * i) - 0.5);
  double w = -log(uniform_open(seed, 2 * i + 1));
  if (a == 1.0) return tan(v);
  return sin(a * v) / pow(cos(v), 1.0 / a) * pow(cos(v - a * v) / w, (1.0 - a) / a);
}

/* Round-to-nearest-even cast of a double to OCP FP8 E4M3FN (bias 7, no
 * infinities, largest finite 448), saturating to +-448.  Written from the
 * format definition: normals are (1 + m/8) 2^(E-7) for E in 1..15 (E = 15,
 * m = 7 is NaN), subnormals m/8 2^-6. */
uint8_t synth_e4m3(double x) {
  uint8_t sign = 0;
  if (isnan(x)) return 0x7F;
  if (signbit(x)) { sign = 0x80; x = -x; }
  if (x >= 448.0) return sign | 0x7E;
  if (x < 0.015625) {                      /* below 2^-6: subnormal grid step 2^-9 */
    double m = nearbyint(x * 512.0);       /* ties to even under the default mode */
    return sign | (uint8_t)m;              /* m == 8 is the smallest normal, 0x08 */
  }
  int e;
  double f = frexp(x, &e);                 /* x = f 2^e, f in [0.5, 1) */
  double m = nearbyint((2.0 * f - 1.0) * 8.0);
  int ex = e - 1 + 7;                      /* biased exponent of 2f in [1, 2) */
  if (m == 8.0) { m = 0.0; ex += 1; }
  if (ex > 15 || (ex == 15 && m > 6.0)) return sign | 0x7E;
  return sign | (uint8_t)(ex << 3) | (uint8_t)m;
}

/* out[i] = E4M3(sigma * N_i), i in [begin, begin + count). */
void synth_gaussian(uint64_t seed, uint64_t begin, uint64_t count, double sigma, uint8_t* out) {
  long long c = (long long)count;
#pragma omp parallel for schedule(static)
  for (long long k = 0; k < c; ++k) out[k] = synth_e4m3(sigma * normal_at(seed, begin + (uint64_t)k));
}

/* BF16 bit pattern of a double: cast to float32 (round to nearest even),
 * then keep the top 16 bits, rounding the dropped 16 to nearest even; NaN
 * stays a quiet NaN.  BF16 is the upper half of an IEEE binary32. */
uint16_t synth_bf16(double x) {
  float f = (float)x;
  uint32_t u;
  memcpy(&u, &f, 4);
  if (isnan(f)) return (uint16_t)((u >> 16) | 0x40);
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

/* out[i] = BF16(sigma * N_i), i in [begin, begin + count). */
void synth_gaussian_bf16(uint64_t seed, uint64_t begin, uint64_t count, double sigma, uint16_t* out) {
  long long c = (long long)count;
#pragma omp parallel for schedule(static)
  for (long long k = 0; k < c; ++k) out[k] = synth_bf16(sigma * normal_at(seed, begin + (uint64_t)k));
}

/* max |X_i| over i in [0, n) of the alpha-stable sample. */
double synth_sas_max_abs(uint64_t seed, uint64_t n, double a) {
  double m = 0.0;
  long long c = (long long)n;
#pragma omp parallel for schedule(static) reduction(max : m)
  for (long long k = 0; k < c; ++k) {
    double v = fabs(sas_at(seed, (uint64_t)k, a));
    if (v > m) m = v;
  }
  return m;
}

/* out[i] = E4M3(scale * X_i), i in [begin, begin + count). */
void synth_sas(uint64_t seed, uint64_t begin, uint64_t count, double a, double scale, uint8_t* out) {
  long long c = (long long)count;
#pragma omp parallel for schedule(static)
  for (long long k = 0; k < c; ++k) out[k] = synth_e4m3(scale * sas_at(seed, begin + (uint64_t)k, a));
}

/* Raw draws, for tests of the samplers themselves. */
void synth_normal_raw(uint64_t seed, uint64_t begin, uint64_t count, double* out) {
  for (uint64_t k = 0; k < count; ++k) out[k] = normal_at(seed, begin + k);
}
void synth_sas_raw(uint64_t seed, uint64_t begin, uint64_t count, double a, double* out) {
  for (uint64_t k = 0; k < count; ++k) out[k] = sas_at(seed, begin + k, a);
}

int synth_max_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
