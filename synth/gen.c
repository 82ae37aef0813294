/*
 * Seeded, counter-based synthetic inputs shared by the CUDA path's tests/bench
 * and by the CPU oracle.  This file holds NO attention or cache arithmetic: it
 * only turns (seed, tensor id, sequence, head, position, channel) coordinates
 * into numbers, so any element of any history position can be regenerated on
 * its own (a 131072-token history never has to exist in memory).
 *
 * Hash: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014), applied once per coordinate.
 * Normals: Box-Muller transform of two 53-bit uniforms, in double, then
 * rounded to float32 (and, on request, to bfloat16 with round-to-nearest-even,
 * the rounding torch's .to(torch.bfloat16) applies).
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <pthread.h>

static inline uint64_t sm64(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

static inline uint64_t row_key(uint64_t seed, uint32_t tid, uint64_t seq,
                               uint64_t head, uint64_t pos) {
  uint64_t h = sm64(seed ^ ((uint64_t)tid << 56));
  h = sm64(h ^ seq);
  h = sm64(h ^ (head + 0x1000));
  h = sm64(h ^ (pos + 0x100000000ull));
  return h;
}

static inline double normal_from(uint64_t h) {
  const double two_pi = 6.283185307179586476925286766559;
  uint64_t h2 = sm64(h);
  double u1 = ((double)((h >> 11) + 1)) * 0x1.0p-53; /* (0, 1] */
  double u2 = ((double)(h2 >> 11)) * 0x1.0p-53;      /* [0, 1) */
  return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

double synth_normal(uint64_t seed, uint32_t tid, uint64_t seq, uint64_t head,
                    uint64_t pos, uint64_t dim) {
  return normal_from(sm64(row_key(seed, tid, seq, head, pos) ^ (dim * 0xD1B54A32D192ED03ull)));
}

/* Uniform integer in [lo, hi] for draw number `index` of stream `tid`. */
int64_t synth_uniform_int(uint64_t seed, uint32_t tid, uint64_t index, int64_t lo, int64_t hi) {
  uint64_t h = sm64(row_key(seed, tid, 0, 0, index));
  uint64_t span = (uint64_t)(hi - lo) + 1ull;
  return lo + (int64_t)(h % span);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  union { float f; uint32_t u; } c;
  c.f = f;
  uint32_t u = c.u;
  uint32_t rounding = ((u >> 16) & 1u) + 0x7FFFu;
  return (uint16_t)((u + rounding) >> 16);
}

typedef struct {
  uint64_t seed; uint32_t tid; uint64_t seq; int H; int64_t pos0; int64_t npos; int d;
  const double* chan_scale; /* [H][d] multiplier or NULL */
  float* out_f32;           /* [npos][H][d] or NULL */
  uint16_t* out_bf16;       /* [npos][H][d] or NULL */
  int64_t r0, r1;           /* rows (npos*H) handled by this worker */
} fill_job;

static void* fill_worker(void* arg) {
  fill_job* j = (fill_job*)arg;
  for (int64_t r = j->r0; r < j->r1; ++r) {
    int64_t ip = r / j->H;
    int h = (int)(r % j->H);
    uint64_t key = row_key(j->seed, j->tid, j->seq, (uint64_t)h, (uint64_t)(j->pos0 + ip));
    for (int c = 0; c < j->d; ++c) {
      double z = normal_from(sm64(key ^ ((uint64_t)c * 0xD1B54A32D192ED03ull)));
      if (j->chan_scale) z *= j->chan_scale[(size_t)h * j->d + c];
      float f = (float)z;
      size_t o = (size_t)r * j->d + c;
      if (j->out_f32) j->out_f32[o] = f;
      if (j->out_bf16) j->out_bf16[o] = f32_to_bf16_rne(f);
    }
  }
  return NULL;
}

/*
 * Fill rows for positions [pos0, pos0+npos) of one sequence, all H heads,
 * token-major [npos][H][d].  Element (p, h, c) equals
 * float32(synth_normal(seed, tid, seq, h, p, c) * scale[h][c]).
 */
void synth_fill_rows(uint64_t seed, uint32_t tid, uint64_t seq, int H, int64_t pos0,
                     int64_t npos, int d, const double* chan_scale, float* out_f32,
                     uint16_t* out_bf16, int nthreads) {
  int64_t rows = npos * H;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 64) nthreads = 64;
  if (rows < 4096) nthreads = 1;
  pthread_t th[64];
  fill_job jobs[64];
  for (int i = 0; i < nthreads; ++i) {
    fill_job j = {seed, tid, seq, H, pos0, npos, d, chan_scale, out_f32, out_bf16,
                  rows * i / nthreads, rows * (i + 1) / nthreads};
    jobs[i] = j;
  }
  for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, fill_worker, &jobs[i]);
  fill_worker(&jobs[0]);
  for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
}

/* Round float32 values to bfloat16 bits (round to nearest even). */
void synth_f32_to_bf16(const float* in, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}
