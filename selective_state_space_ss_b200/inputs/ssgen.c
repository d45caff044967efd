/*
 * ssgen.c -- seeded, counter-based synthetic input generator.
 *
 * Shared by the tests, the benchmark and the oracle comparisons: the same host
 * buffers feed the fp64 oracle and the host->device copy.  It holds none of
 * the selective-scan arithmetic, only random numbers:
 *
 *  - SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
 *    generators", OOPSLA 2014): output i of a generator seeded with k is the
 *    finaliser applied to k + (i+1)*gamma, so any element can be drawn on its
 *    own, in any order, by any thread.
 *  - a stream key per (seed, stream) is output `stream` of SplitMix64 seeded
 *    with `seed`.
 *  - uniforms in the open interval (0,1) from the top 53 bits.
 *  - normals by the Box-Muller transform (Box and Muller, 1958), one normal
 *    per pair of uniforms (cosine branch), pair j = draws 2j and 2j+1.
 *  - bfloat16 by round-to-nearest-even of the binary32 value.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define SM64_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t sm64_finalise(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t sm64_at(uint64_t key, uint64_t i) {
  return sm64_finalise(key + (i + 1) * SM64_GAMMA);
}

static inline double to_unit_open(uint64_t r) {
  return ((double)(r >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t bits;
  memcpy(&bits, &f, sizeof bits);
  bits += 0x7FFFu + ((bits >> 16) & 1u);
  return (uint16_t)(bits >> 16);
}

uint64_t ssgen_stream_key(uint64_t seed, uint64_t stream) {
  return sm64_at(seed, stream);
}

double ssgen_uniform_at(uint64_t key, uint64_t i) {
  return to_unit_open(sm64_at(key, i));
}

double ssgen_normal_at(uint64_t key, uint64_t i) {
  const double u1 = to_unit_open(sm64_at(key, 2 * i));
  const double u2 = to_unit_open(sm64_at(key, 2 * i + 1));
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

typedef struct {
  uint64_t key, offset;
  int64_t begin, end;
  double mean, scale;
  int kind;      /* 0 normal, 1 uniform */
  int out_type;  /* 0 f32, 1 bf16, 2 f64 */
  void* out;
} fill_t;

static void* fill_range(void* arg) {
  const fill_t* F = (const fill_t*)arg;
  for (int64_t j = F->begin; j < F->end; ++j) {
    const uint64_t i = F->offset + (uint64_t)j;
    const double r = F->kind == 0 ? ssgen_normal_at(F->key, i) : ssgen_uniform_at(F->key, i);
    const double v = F->mean + F->scale * r;
    if (F->out_type == 0) {
      ((float*)F->out)[j] = (float)v;
    } else if (F->out_type == 1) {
      ((uint16_t*)F->out)[j] = f32_to_bf16_rne((float)v);
    } else {
      ((double*)F->out)[j] = v;
    }
  }
  return NULL;
}

/* Fill out[0..count) with mean + scale * draw(offset + j).  kind: 0 normal,
 * 1 uniform(0,1).  out_type: 0 f32, 1 bf16 bits, 2 f64.  Returns 0 or -1. */
int ssgen_fill(uint64_t seed, uint64_t stream, uint64_t offset, int64_t count,
               double mean, double scale, int kind, int out_type, void* out,
               int nthreads) {
  if (!out || count < 0 || kind < 0 || kind > 1 || out_type < 0 || out_type > 2) return -1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (count < 65536) nthreads = 1;
  const uint64_t key = ssgen_stream_key(seed, stream);
  fill_t jobs[256];
  pthread_t tids[256];
  const int64_t per = (count + nthreads - 1) / nthreads;
  int started = 0;
  for (int t = 0; t < nthreads; ++t) {
    fill_t* F = &jobs[t];
    F->key = key; F->offset = offset; F->mean = mean; F->scale = scale;
    F->kind = kind; F->out_type = out_type; F->out = out;
    F->begin = (int64_t)t * per;
    F->end = F->begin + per < count ? F->begin + per : count;
    if (F->begin >= F->end) { F->end = F->begin; continue; }
    if (t == 0) continue;
    if (pthread_create(&tids[started], NULL, fill_range, F) == 0) {
      ++started;
    } else {
      fill_range(F);
    }
  }
  fill_range(&jobs[0]);
  for (int t = 0; t < started; ++t) pthread_join(tids[t], NULL);
  return 0;
}
