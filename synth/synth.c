/*
 * Seeded synthetic input generator for the LServe-style sparse-attention
 * workloads.  It is shared by the CUDA path's tests/benchmarks and by the
 * CPU oracle's tests, and it deliberately contains none of the attention
 * method's arithmetic: it only draws numbers and lays them out.
 *
 * Generator definition (counter based, so any slice can be regenerated
 * without the rest):
 *   mix64(z)      : the SplitMix64 output function (Steele, Lea & Flood,
 *                   "Fast splittable pseudorandom number generators",
 *                   OOPSLA 2014):  z ^= z>>30; z *= 0xBF58476D1CE4E5B9;
 *                   z ^= z>>27; z *= 0x94D049BB133111EB; z ^= z>>31.
 *   draw(key, i)  : mix64(key + (i + 1) * 0x9E3779B97F4A7C15)
 *   uniform(x)    : ((x >> 11) + 0.5) * 2^-53, in the open interval (0, 1)
 *   normal(key,i) : Box-Muller on the pair j = floor(i/2):
 *                   r = sqrt(-2 ln u1), a = 2 pi u2 with u1 = uniform(draw(key, 2j)),
 *                   u2 = uniform(draw(key, 2j+1)); even i -> r cos a, odd i -> r sin a
 *   bf16(x)       : x rounded to float (round-to-nearest-even), then to
 *                   bfloat16 (round-to-nearest-even on the upper 16 bits).
 *
 * Element (b, h, t, c) of a per-sequence K or V stream uses
 *   key_bh = mix64(key ^ ((b * H + h + 1) * 0xD1B54A32D192ED03)),
 *   i      = t * D + c,
 *   value  = bf16(normal(key_bh, i) * scale[h][c] + shift[h][c])
 * where scale/shift default to 1/0 and the shift is applied only on the pages
 * a caller marks (used for the planted high-similarity pages).
 *
 * Built with:  gcc -O2 -fopenmp -shared -fPIC synth.c -o libsynth.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL
#define SEQMIX 0xD1B54A32D192ED03ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t draw(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GOLDEN); }

static inline double uniform01(uint64_t x) { return ((double)(x >> 11) + 0.5) * 0x1.0p-53; }

static inline void normal_pair(uint64_t key, uint64_t j, double* z0, double* z1) {
  const double two_pi = 6.283185307179586476925286766559;
  double u1 = uniform01(draw(key, 2 * j));
  double u2 = uniform01(draw(key, 2 * j + 1));
  double r = sqrt(-2.0 * log(u1));
  double a = two_pi * u2;
  *z0 = r * cos(a);
  *z1 = r * sin(a);
}

static inline double normal_at(uint64_t key, uint64_t i) {
  double z0, z1;
  normal_pair(key, i >> 1, &z0, &z1);
  return (i & 1) ? z1 : z0;
}

/* n consecutive normals starting at counter i0, two per Box-Muller pair */
static inline void normal_run(uint64_t key, uint64_t i0, int64_t n, double* z) {
  int64_t k = 0;
  if ((i0 & 1) && n > 0) z[k++] = normal_at(key, i0);
  for (; k + 1 < n; k += 2) normal_pair(key, (i0 + k) >> 1, &z[k], &z[k + 1]);
  if (k < n) z[k] = normal_at(key, i0 + k);
}

static inline uint16_t to_bf16(double x) {
  float f = (float)x;
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16); /* inf/nan: truncate */
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

uint64_t synth_mix64(uint64_t z) { return mix64(z); }
uint64_t synth_draw(uint64_t key, uint64_t i) { return draw(key, i); }
double synth_normal(uint64_t key, uint64_t i) { return normal_at(key, i); }

/* head dims above this are rejected by the Python wrapper */
int64_t synth_max_row(void) { return 512; }
uint16_t synth_to_bf16(double x) { return to_bf16(x); }

uint64_t synth_seq_key(uint64_t key, int64_t b, int64_t H, int64_t h) {
  return mix64(key ^ ((uint64_t)(b * H + h + 1) * SEQMIX));
}

/* out[r * out_stride + c] = bf16(normal(key, counter0 + r*cols + c) * scale[c] + shift[c]) */
void synth_fill_normal_bf16(uint64_t key, uint64_t counter0, int64_t rows, int64_t cols,
                            const double* scale, const double* shift, uint16_t* out,
                            int64_t out_stride) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    double z[512];
    for (int64_t c0 = 0; c0 < cols; c0 += 512) {
    int64_t w = cols - c0 < 512 ? cols - c0 : 512;
    normal_run(key, counter0 + (uint64_t)(r * cols + c0), w, z);
    for (int64_t c = c0; c < c0 + w; ++c) {
      double x = z[c - c0];
      if (scale) x *= scale[c];
      if (shift) x += shift[c];
      out[r * out_stride + c] = to_bf16(x);
    }
    }
  }
}

/*
 * One sequence b of a paged K or V pool, all heads:
 *   pool layout  [num_pool_pages][H][page][D]  (bf16 bits)
 *   block_row    [npages] pool id of each page ordinal of the sequence
 *   scale/shift  [H][D] (nullable); shift_pages[npages] (nullable: shift all)
 *   pad          bit pattern written to rows t >= n of the last page
 */
void synth_fill_pool_seq(uint64_t key, int64_t b, int64_t H, int64_t D, int64_t page, int64_t n,
                         const int32_t* block_row, const double* scale, const double* shift,
                         const uint8_t* shift_pages, uint16_t pad, uint16_t* pool) {
  int64_t npages = (n + page - 1) / page;
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t m = 0; m < npages; ++m) {
    for (int64_t h = 0; h < H; ++h) {
      uint64_t kbh = synth_seq_key(key, b, H, h);
      uint16_t* dst = pool + (((int64_t)block_row[m] * H + h) * page) * D;
      int do_shift = shift && (!shift_pages || shift_pages[m]);
      double z[512];
      for (int64_t r = 0; r < page; ++r) {
        int64_t t = m * page + r;
        if (t < n) normal_run(kbh, (uint64_t)(t * D), D, z);
        for (int64_t c = 0; c < D; ++c) {
          if (t >= n) {
            dst[r * D + c] = pad;
            continue;
          }
          double x = z[c];
          if (scale) x *= scale[h * D + c];
          if (do_shift) x += shift[h * D + c];
          dst[r * D + c] = to_bf16(x);
        }
      }
    }
  }
}

/* The same values as synth_fill_pool_seq for one head, laid out densely [n][D]. */
void synth_fill_seq_dense(uint64_t key, int64_t b, int64_t H, int64_t h, int64_t D, int64_t page,
                          int64_t n, const double* scale, const double* shift,
                          const uint8_t* shift_pages, uint16_t* out) {
  uint64_t kbh = synth_seq_key(key, b, H, h);
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < n; ++t) {
    int64_t m = t / page;
    int do_shift = shift && (!shift_pages || shift_pages[m]);
    double z[512];
    normal_run(kbh, (uint64_t)(t * D), D, z);
    for (int64_t c = 0; c < D; ++c) {
      double x = z[c];
      if (scale) x *= scale[h * D + c];
      if (do_shift) x += shift[h * D + c];
      out[t * D + c] = to_bf16(x);
    }
  }
}
