/*
 * Seeded synthetic inputs for the sparse-prefill workloads.
 *
 * This module holds no part of the attention method: it only draws the bf16
 * Q/K/V tensors that both the CUDA path and the CPU oracle consume, so that the
 * two sides see bit-identical inputs without sharing any of the method's code.
 *
 * Generator: counter-based.  Element n of stream (seed, stream) is derived from
 * one 64-bit draw  z = splitmix64(key(seed, stream, n))  where splitmix64 is the
 * mixing function published by Steele, Lea and Flood ("Fast splittable
 * pseudorandom number generators", OOPSLA 2014).  The two 32-bit halves of z
 * give two uniforms, turned into one standard normal by the Box-Muller
 * transform (Box and Muller, 1958), computed in double precision and rounded
 * to fp32, then (optionally) shifted by a per-row bias vector and rounded to
 * bf16 with round-to-nearest-even.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t mix64(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

static inline uint64_t key_of(uint64_t seed, uint64_t stream, uint64_t n) {
  /* n < 2^40 elements per stream, stream < 2^16, seed folded through one mix */
  return mix64(seed * 0x2545F4914F6CDD1Dull + 1u) ^ (stream << 40) ^ n;
}

static inline double normal_at(uint64_t seed, uint64_t stream, uint64_t n) {
  uint64_t z = mix64(key_of(seed, stream, n));
  uint32_t hi = (uint32_t)(z >> 32), lo = (uint32_t)z;
  double u1 = ((double)(hi >> 8) + 1.0) * (1.0 / 16777216.0); /* (0, 1] */
  double u2 = (double)(lo >> 8) * (1.0 / 16777216.0);         /* [0, 1) */
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16); /* inf / nan kept */
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* Standard normals as doubles: out[i] = N(0,1) draw n = first + i of the stream. */
void wl_normals_f64(double* out, int64_t count, uint64_t seed, uint64_t stream, int64_t first) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i) out[i] = normal_at(seed, stream, (uint64_t)(first + i));
}

/*
 * Fill a [rows, d] bf16 matrix (row-major, contiguous) with N(0,1) draws of one
 * stream, element (r, c) using counter r*d + c.  Rows r with bias_rows[r] != 0
 * get bias_scale * bias[c] added in fp32 before rounding to bf16.
 */
void wl_fill_bf16(uint16_t* out, int64_t rows, int32_t d, uint64_t seed, uint64_t stream,
                  const float* bias, const uint8_t* bias_rows, float bias_scale) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    int add = bias && bias_rows && bias_rows[r];
    for (int32_t c = 0; c < d; ++c) {
      float v = (float)normal_at(seed, stream, (uint64_t)(r * d + c));
      if (add) v = v + bias_scale * bias[c];
      out[r * d + c] = f32_to_bf16_rne(v);
    }
  }
}

/*
 * Position-structured variant: row r is (noise_scale * N(0,1) + shared_scale * shared[c]
 * [+ bias_scale * bias[c] on flagged rows]) rotated by the rotary position embedding of
 * position r (Su et al., "RoFormer", 2021, in the half-split layout): dimensions m and
 * m + d/2 form a pair rotated by the angle r * base^(-2m/d).  Dot products of two such rows then
 * depend on their positions only through the offset between them, as in the rotary models the
 * benchmark layers stand for.  Angles and rotations in double precision, rounded to fp32, then
 * to bf16 (round to nearest even).
 */
void wl_fill_rope_bf16(uint16_t* out, int64_t rows, int32_t d, uint64_t seed, uint64_t stream,
                       float noise_scale, const float* shared, float shared_scale, double base,
                       const float* bias, const uint8_t* bias_rows, float bias_scale) {
  const int32_t half = d / 2;
  double freq[256];
  if (d > 512) return;
  for (int32_t m = 0; m < half; ++m) freq[m] = pow(base, -2.0 * (double)m / (double)d);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    int add = bias && bias_rows && bias_rows[r];
    float v[512];
    for (int32_t c = 0; c < d; ++c) {
      float x = noise_scale * (float)normal_at(seed, stream, (uint64_t)(r * d + c));
      if (shared) x = x + shared_scale * shared[c];
      if (add) x = x + bias_scale * bias[c];
      v[c] = x;
    }
    for (int32_t m = 0; m < half; ++m) {
      const double ang = (double)r * freq[m];
      const double cs = cos(ang), sn = sin(ang);
      const double a = v[m], b = v[m + half];
      out[r * d + m] = f32_to_bf16_rne((float)(a * cs - b * sn));
      out[r * d + m + half] = f32_to_bf16_rne((float)(a * sn + b * cs));
    }
  }
}
