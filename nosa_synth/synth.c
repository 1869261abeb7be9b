/*
 * Seeded synthetic inputs for the NOSA sparse-decode step.
 *
 * This module is shared by the tests, the benchmark and the fp64 oracle. It
 * holds only random-number generation and the input recipe (shifts, sinks,
 * rounding to bf16); none of the method's arithmetic (pooling, selection,
 * residency, attention) lives here.
 *
 * Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014) used as a counter-based hash. A stream is
 * named by (seed, tensor, a, b, c); element i of the stream is a pure function
 * of that key and i, so any slice can be regenerated on its own and in parallel.
 * Gaussians: Box-Muller (1958) on two uniforms in (0, 1), cosine branch for
 * even i and sine branch for odd i of the same pair.
 * bf16: round-to-nearest-even of the fp32 value (double -> float first).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t sm64(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint32_t tensor, uint32_t a, uint32_t b,
                                  uint32_t c) {
  uint64_t h = sm64(seed ^ 0x6E6F7361ull); /* "nosa" */
  h = sm64(h ^ (uint64_t)tensor);
  h = sm64(h ^ ((uint64_t)a << 1));
  h = sm64(h ^ ((uint64_t)b << 2));
  h = sm64(h ^ ((uint64_t)c << 3));
  return h;
}

static inline uint64_t elem_hash(uint64_t key, uint64_t i, uint64_t lane) {
  return sm64(key ^ sm64(i * 4u + lane));
}

/* uniform in the open interval (0, 1) from the top 53 bits */
static inline double to_u01(uint64_t h) { return ((double)(h >> 11) + 0.5) * 0x1p-53; }

static inline double gauss_at(uint64_t key, uint64_t i) {
  const uint64_t pair = i >> 1;
  const double u1 = to_u01(elem_hash(key, pair, 0));
  const double u2 = to_u01(elem_hash(key, pair, 1));
  const double r = sqrt(-2.0 * log(u1));
  const double th = 6.283185307179586476925286766559 * u2;
  return (i & 1u) ? r * sin(th) : r * cos(th);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0u; /* NaN */
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* ---------------------------------------------------------------- exports */

void synth_hash_u64(uint64_t seed, uint32_t tensor, uint32_t a, uint32_t b, uint32_t c,
                    uint64_t i0, uint64_t n, uint64_t* out) {
  const uint64_t key = stream_key(seed, tensor, a, b, c);
  for (uint64_t i = 0; i < n; ++i) out[i] = elem_hash(key, i0 + i, 2);
}

void synth_uniform_f64(uint64_t seed, uint32_t tensor, uint32_t a, uint32_t b, uint32_t c,
                       uint64_t i0, uint64_t n, double* out) {
  const uint64_t key = stream_key(seed, tensor, a, b, c);
  for (uint64_t i = 0; i < n; ++i) out[i] = to_u01(elem_hash(key, i0 + i, 3));
}

void synth_gauss_f64(uint64_t seed, uint32_t tensor, uint32_t a, uint32_t b, uint32_t c,
                     uint64_t i0, uint64_t n, double* out) {
  const uint64_t key = stream_key(seed, tensor, a, b, c);
  for (uint64_t i = 0; i < n; ++i) out[i] = gauss_at(key, i0 + i);
}

void synth_round_bf16(const double* in, uint64_t n, uint16_t* out) {
  for (uint64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne((float)in[i]);
}

void synth_round_f32(const double* in, uint64_t n, float* out) {
  for (uint64_t i = 0; i < n; ++i) out[i] = (float)in[i];
}

/*
 * Gaussian rows rounded to bf16, for the large key/value tensors.
 * Element (r, i) of the stream (seed, tensor, a, b, c) is gauss(idx) with
 * idx = (row0 + r) * d + i; the stored value is
 *     bf16( float( scale * gauss + offset[row_off[r]][i] ) )
 * where row_off[r] < 0 (or row_off == NULL) means no offset.
 * out rows are written with stride out_stride (elements).
 */
void synth_gauss_rows_bf16(uint64_t seed, uint32_t tensor, uint32_t a, uint32_t b, uint32_t c,
                           int64_t row0, int64_t rows, int32_t d, double scale,
                           const double* offsets, const int8_t* row_off, uint16_t* out,
                           int64_t out_stride) {
  const uint64_t key = stream_key(seed, tensor, a, b, c);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const int o = row_off ? row_off[r] : -1;
    const double* off = (o >= 0) ? offsets + (int64_t)o * d : 0;
    uint16_t* dst = out + r * out_stride;
    const uint64_t base = (uint64_t)(row0 + r) * (uint64_t)d;
    for (int32_t i = 0; i < d; ++i) {
      double v = scale * gauss_at(key, base + (uint64_t)i);
      if (off) v += off[i];
      dst[i] = f32_to_bf16_rne((float)v);
    }
  }
}
