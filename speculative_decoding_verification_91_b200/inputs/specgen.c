/*
 * Seeded, counter-based input generator for the synthetic verify-step
 * workloads.  It produces weights, context keys/values, token ids and the
 * uniform draws that decide drafts.  It holds none of the verify step's own
 * arithmetic: it only turns (seed, stream, counter) into numbers.
 *
 * Definitions (each element is a pure function of its counter, so any slice
 * of a tensor can be regenerated on its own and threads cannot change it):
 *
 *   mix(z)        SplitMix64 output function (Steele, Lea, Flood,
 *                 "Fast splittable pseudorandom number generators", 2014):
 *                 z ^= z>>30; z *= 0xbf58476d1ce4e5b9;
 *                 z ^= z>>27; z *= 0x94d049bb133111eb; z ^= z>>31.
 *   key(s, t)     mix(s ^ mix(t + G)), G = 0x9e3779b97f4a7c15 (the
 *                 SplitMix64 increment), s = seed, t = stream id.
 *   draw(K, c)    mix(K + (c + 1) * G): the c-th SplitMix64 output of a
 *                 generator whose state starts at K.
 *   unit(x)       (x >> 11) * 2^-53, a double in [0, 1).
 *
 *   normal pair t (Box and Muller, 1958):
 *       u1 = 1 - unit(draw(K, 2t))   in (0, 1]
 *       u2 = unit(draw(K, 2t + 1))
 *       r  = sqrt(-2 ln u1),  a = 2 pi u2
 *       element 2t = r cos a,  element 2t+1 = r sin a
 *   bf16 output: (float)(z * scale), then round-to-nearest-even to the upper
 *   16 bits of the IEEE binary32 pattern.
 *
 * Stream ids are 64-bit FNV-1a hashes of a tensor name (computed by the
 * Python wrapper), so every named tensor has its own independent sequence.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SG_GAMMA 0x9e3779b97f4a7c15ULL

static inline uint64_t sg_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}

static inline uint64_t sg_key(uint64_t seed, uint64_t stream) {
  return sg_mix(seed ^ sg_mix(stream + SG_GAMMA));
}

static inline uint64_t sg_draw(uint64_t key, uint64_t ctr) {
  return sg_mix(key + (ctr + 1ULL) * SG_GAMMA);
}

static inline double sg_unit(uint64_t x) {
  return (double)(x >> 11) * (1.0 / 9007199254740992.0);
}

static inline uint16_t sg_f32_to_bf16_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return 0x7fc0; /* NaN */
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* Raw 64-bit draws: out[i] = draw(key, offset + i). */
void sg_raw_u64(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, uint64_t* out) {
  const uint64_t key = sg_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = sg_draw(key, offset + (uint64_t)i);
}

/* Uniform doubles in [0, 1): out[i] = unit(draw(key, offset + i)). */
void sg_uniform(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double* out) {
  const uint64_t key = sg_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = sg_unit(sg_draw(key, offset + (uint64_t)i));
}

/* Integers in [lo, hi): lo + floor(unit * (hi - lo)). */
void sg_randint(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, int64_t lo, int64_t hi,
                int64_t* out) {
  const uint64_t key = sg_key(seed, stream);
  const double span = (double)(hi - lo);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    int64_t v = (int64_t)floor(sg_unit(sg_draw(key, offset + (uint64_t)i)) * span);
    if (v >= hi - lo) v = hi - lo - 1;
    out[i] = lo + v;
  }
}

static inline double sg_normal_at(uint64_t key, uint64_t idx) {
  const uint64_t t = idx >> 1;
  const double u1 = 1.0 - sg_unit(sg_draw(key, 2 * t));
  const double u2 = sg_unit(sg_draw(key, 2 * t + 1));
  const double r = sqrt(-2.0 * log(u1));
  const double a = 6.283185307179586 * u2;
  return (idx & 1) ? r * sin(a) : r * cos(a);
}

/* Normal(0, scale^2) values as float32: out[i] = (float)(z(offset+i) * scale). */
void sg_normal_f32(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double scale,
                   float* out) {
  const uint64_t key = sg_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (float)(sg_normal_at(key, offset + (uint64_t)i) * scale);
}

/* Same values rounded to bfloat16 (bit patterns). */
void sg_normal_bf16(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double scale,
                    uint16_t* out) {
  const uint64_t key = sg_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = sg_f32_to_bf16_bits((float)(sg_normal_at(key, offset + (uint64_t)i) * scale));
}

/*
 * Strided variant for tensors whose generated region is a sub-block: row r
 * (r in [0, rows)) of `cols` elements is generated from counter
 * offset + r * row_stride and written to out + r * cols.
 */
void sg_normal_bf16_rows(uint64_t seed, uint64_t stream, uint64_t offset, int64_t rows,
                         int64_t cols, uint64_t row_stride, double scale, uint16_t* out) {
  const uint64_t key = sg_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const uint64_t base = offset + (uint64_t)r * row_stride;
    uint16_t* o = out + r * cols;
    for (int64_t c = 0; c < cols; ++c)
      o[c] = sg_f32_to_bf16_bits((float)(sg_normal_at(key, base + (uint64_t)c) * scale));
  }
}

int sg_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
