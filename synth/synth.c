/*
 * synth.c - seeded, counter-based generator for the synthetic attention
 * workloads (Q, K, V tensors with planted directions).
 *
 * This module holds no attention arithmetic. It only turns (seed, stream,
 * index) into numbers, so that the CPU oracle and the CUDA path read the very
 * same input bytes.
 *
 * Random source: the SplitMix64 generator (Steele, Lea, Flood, "Fast
 * splittable pseudorandom number generators", OOPSLA 2014), used in counter
 * mode: draw i of a stream is the finaliser applied to key + (i+1)*gamma,
 * which is exactly the (i+1)-th output of a SplitMix64 sequence whose state
 * starts at `key`. The finaliser constants are the ones SplitMix64 publishes
 * (Stafford's "variant 13" mixer).
 *
 * Normals: Box-Muller (Box and Muller, 1958), one normal per 64-bit draw:
 * the high and low 32-bit halves give the two uniforms in (0,1); the cosine
 * branch is kept.
 *
 * Tensor fill: element (b, h, pos, x) of a [B, H, L, d] tensor is
 *     N(0,1)[flat index] + amp_u[b, hk, pos] * u[b, hk, x]
 *                        + amp_w * w[b, hk, (pos + offset) / seg_len, x]
 * with hk = h / g, computed in double, rounded to fp32 (round to nearest
 * even), and, when a bf16 copy is requested, rounded again from fp32 to bf16
 * (round to nearest even); the fp32 copy then holds the widened bf16 value so
 * both copies describe the same number.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL
#define SYNTH_STREAM_MUL 0xD1B54A32D192ED03ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return mix64(mix64(seed) ^ (stream * SYNTH_STREAM_MUL));
}

static inline uint64_t draw(uint64_t key, uint64_t idx) {
  return mix64(key + (idx + 1ULL) * SYNTH_GAMMA);
}

static inline double normal_from(uint64_t r) {
  const double two_m32 = 2.3283064365386963e-10; /* 2^-32 */
  double u1 = ((double)(r >> 32) + 0.5) * two_m32;
  double u2 = ((double)(r & 0xffffffffULL) + 0.5) * two_m32;
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

static inline float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* ---- raw streams -------------------------------------------------------- */

uint64_t synth_mix64(uint64_t x) { return mix64(x); }

void synth_u64(uint64_t seed, uint64_t stream, uint64_t start, int64_t n,
               uint64_t *out) {
  uint64_t key = stream_key(seed, stream);
  for (int64_t i = 0; i < n; ++i) out[i] = draw(key, start + (uint64_t)i);
}

void synth_normal(uint64_t seed, uint64_t stream, uint64_t start, int64_t n,
                  double *out) {
  uint64_t key = stream_key(seed, stream);
  for (int64_t i = 0; i < n; ++i)
    out[i] = normal_from(draw(key, start + (uint64_t)i));
}

/* ---- tensor fill -------------------------------------------------------- */

typedef struct {
  int64_t B, H, L, d;   /* output shape [B, H, L, d] */
  int64_t Hkv;          /* structure heads: row (b, h) uses hk = h / (H / Hkv) */
  uint64_t seed, stream;
  const float *amp_u;   /* [B, Hkv, L] amplitude on u, or NULL for none */
  const double *u;      /* [B, Hkv, d] directions, or NULL */
  int64_t seg_len;      /* 0: no segment directions */
  double amp_w;         /* amplitude on the segment direction */
  const double *w;      /* [B, Hkv, nseg, d] */
  int64_t seg_pos_offset; /* row pos lies in segment (pos + offset) / seg_len */
  int64_t nseg;         /* segments per head in w */
  float *out_f32;       /* nullable */
  uint16_t *out_bf16;   /* nullable; when set, values are rounded to bf16 */
  int nthreads;         /* <= 0: all online cores */
} synth_fill_args;

typedef struct {
  const synth_fill_args *a;
  int64_t row0, row1;   /* flat rows [row0, row1) of B*H*L */
} fill_job;

static void *fill_worker(void *p) {
  const fill_job *job = (const fill_job *)p;
  const synth_fill_args *a = job->a;
  const int64_t g = a->H / a->Hkv;
  const int64_t nseg = a->nseg;
  uint64_t key = stream_key(a->seed, a->stream);
  for (int64_t row = job->row0; row < job->row1; ++row) {
    int64_t pos = row % a->L;
    int64_t bh = row / a->L;
    int64_t h = bh % a->H, b = bh / a->H;
    int64_t hk = h / g;
    double au = 0.0;
    const double *u = NULL, *w = NULL;
    if (a->amp_u && a->u) {
      au = a->amp_u[(b * a->Hkv + hk) * a->L + pos];
      u = a->u + (b * a->Hkv + hk) * a->d;
    }
    if (a->seg_len > 0 && a->w && a->amp_w != 0.0) {
      int64_t seg = (pos + a->seg_pos_offset) / a->seg_len;
      if (seg >= 0 && seg < nseg) w = a->w + ((b * a->Hkv + hk) * nseg + seg) * a->d;
    }
    for (int64_t x = 0; x < a->d; ++x) {
      uint64_t idx = (uint64_t)(row * a->d + x);
      double val = normal_from(draw(key, idx));
      if (u && au != 0.0) val += au * u[x];
      if (w) val += a->amp_w * w[x];
      float f = (float)val;
      int64_t o = row * a->d + x;
      if (a->out_bf16) {
        uint16_t hb = f32_to_bf16_rne(f);
        a->out_bf16[o] = hb;
        f = bf16_to_f32(hb);
      }
      if (a->out_f32) a->out_f32[o] = f;
    }
  }
  return NULL;
}

int synth_fill(const synth_fill_args *a) {
  if (!a || a->B <= 0 || a->H <= 0 || a->L <= 0 || a->d <= 0 || a->Hkv <= 0 ||
      a->H % a->Hkv != 0 || (!a->out_f32 && !a->out_bf16))
    return -1;
  int nt = a->nthreads;
  if (nt <= 0) {
    long c = sysconf(_SC_NPROCESSORS_ONLN);
    nt = c > 0 ? (int)c : 1;
  }
  int64_t rows = a->B * a->H * a->L;
  if (nt > rows) nt = (int)rows;
  if (nt > 256) nt = 256;
  pthread_t th[256];
  fill_job jobs[256];
  int threaded[256];
  int64_t per = (rows + nt - 1) / nt;
  for (int t = 0; t < nt; ++t) {
    threaded[t] = 0;
    jobs[t].a = a;
    jobs[t].row0 = (int64_t)t * per;
    jobs[t].row1 = jobs[t].row0 + per < rows ? jobs[t].row0 + per : rows;
    if (jobs[t].row0 >= jobs[t].row1) continue;
    if (pthread_create(&th[t], NULL, fill_worker, &jobs[t]) == 0)
      threaded[t] = 1;
    else
      fill_worker(&jobs[t]);
  }
  for (int t = 0; t < nt; ++t)
    if (threaded[t]) pthread_join(th[t], NULL);
  return 0;
}
