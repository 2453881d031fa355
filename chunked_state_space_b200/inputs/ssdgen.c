/*
 * Seeded synthetic input generator for the chunked SSD scan.
 *
 * This file holds NO arithmetic of the scan itself: it only draws the input
 * tensors (x, dt, A, B, C, D, initial state) with the distributions of the
 * workloads.  Both the fp64 oracle (through the tests) and the CUDA path
 * consume the buffers it fills; neither side re-implements it.
 *
 * Generator: counter-based splitmix64.  Element i of a stream with key k is
 *     z = mix64(k + (i + 1) * 0x9E3779B97F4A7C15)
 * where mix64 is the splitmix64 output function published by Steele, Lea and
 * Flood ("Fast splittable pseudorandom number generators", OOPSLA 2014).
 * Because every element depends only on (key, index), any slice of a tensor
 * can be regenerated independently and the result does not depend on the
 * number of threads.
 *
 * Uniforms use the top 53 bits: u = (z >> 11) * 2^-53, in [0, 1).
 * Normals use the Box-Muller transform on the pair (2j, 2j+1):
 *     r = sqrt(-2 ln(1 - u_{2j})), element 2j = r cos(2 pi u_{2j+1}),
 *                                  element 2j+1 = r sin(2 pi u_{2j+1}).
 * All of this runs in double and is rounded once to fp32 (round to nearest);
 * bf16 output rounds that fp32 value to nearest-even.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline double u01(uint64_t key, uint64_t i) {
  uint64_t z = mix64(key + (i + 1ULL) * GOLDEN_GAMMA);
  return (double)(z >> 11) * (1.0 / 9007199254740992.0);
}

static inline double std_normal(uint64_t key, uint64_t i) {
  const double two_pi = 6.283185307179586476925286766559;
  uint64_t j = i >> 1;
  double u1 = u01(key, 2 * j);
  double u2 = u01(key, 2 * j + 1);
  double r = sqrt(-2.0 * log1p(-u1));
  return (i & 1) ? r * sin(two_pi * u2) : r * cos(two_pi * u2);
}

/* Derive a stream key from (seed, workload id, layer, tensor id). */
uint64_t ssdgen_key(uint64_t seed, uint64_t workload, uint64_t layer, uint64_t tensor) {
  uint64_t k = mix64(seed + GOLDEN_GAMMA);
  k = mix64(k ^ (workload * 0xD1B54A32D192ED03ULL + 1));
  k = mix64(k ^ (layer * 0xAEF17502108EF2D9ULL + 2));
  k = mix64(k ^ (tensor * 0xDB4F0B9175AE2165ULL + 3));
  return k;
}

enum {
  SSDGEN_NORMAL = 0,        /* mean p0, standard deviation p1 */
  SSDGEN_UNIFORM = 1,       /* U[p0, p1) */
  SSDGEN_SOFTPLUS_NORMAL = 2, /* softplus(N(p0, p1^2)): log(1 + exp(z)) */
  SSDGEN_NEG_EXP_UNIFORM = 3, /* -exp(U[p0, p1)) */
  SSDGEN_CONSTANT = 4       /* p0 */
};

static inline double draw(int dist, uint64_t key, uint64_t i, double p0, double p1) {
  switch (dist) {
    case SSDGEN_NORMAL: return p0 + p1 * std_normal(key, i);
    case SSDGEN_UNIFORM: return p0 + (p1 - p0) * u01(key, i);
    case SSDGEN_SOFTPLUS_NORMAL: {
      double z = p0 + p1 * std_normal(key, i);
      /* stable softplus: max(z,0) + log1p(exp(-|z|)) */
      return (z > 0 ? z : 0.0) + log1p(exp(-fabs(z)));
    }
    case SSDGEN_NEG_EXP_UNIFORM: return -exp(p0 + (p1 - p0) * u01(key, i));
    default: return p0;
  }
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/*
 * Fill n elements starting at element index `first` of the stream `key`.
 * out_dtype: 0 = fp32, 1 = bf16 (raw 16-bit pattern).
 */
void ssdgen_fill(void* out, int out_dtype, int64_t first, int64_t n, uint64_t key, int dist,
                 double p0, double p1) {
  if (out_dtype == 0) {
    float* o = (float*)out;
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < n; ++k) o[k] = (float)draw(dist, key, (uint64_t)(first + k), p0, p1);
  } else {
    uint16_t* o = (uint16_t*)out;
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < n; ++k)
      o[k] = f32_to_bf16_rne((float)draw(dist, key, (uint64_t)(first + k), p0, p1));
  }
}

/* Gather variant: element indices given explicitly (for sampled slices). */
void ssdgen_fill_indexed(void* out, int out_dtype, const int64_t* idx, int64_t n, uint64_t key,
                         int dist, double p0, double p1) {
  if (out_dtype == 0) {
    float* o = (float*)out;
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < n; ++k) o[k] = (float)draw(dist, key, (uint64_t)idx[k], p0, p1);
  } else {
    uint16_t* o = (uint16_t*)out;
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < n; ++k)
      o[k] = f32_to_bf16_rne((float)draw(dist, key, (uint64_t)idx[k], p0, p1));
  }
}

/* Raw generator outputs, for the generator's own tests. */
void ssdgen_raw_u64(uint64_t* out, uint64_t key, int64_t first, int64_t n) {
  for (int64_t k = 0; k < n; ++k) out[k] = mix64(key + ((uint64_t)(first + k) + 1ULL) * GOLDEN_GAMMA);
}
