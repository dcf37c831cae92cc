/*
 * Seeded synthetic inputs for the MoE dispatch path: router logits -> top-K
 * expert ids and gate weights, hidden rows, replica gradients.
 *
 * This module produces INPUTS only.  It holds none of the arithmetic of the
 * method under test (histogram, plan, layout, align-sort, dispatch, combine,
 * gradient reduction); both the CPU oracle and the CUDA path consume what it
 * writes.  The router step (top-K by descending logit, ties to the lower
 * expert id, softmax over the K chosen logits) is the model's gate, which sits
 * upstream of the expert-parallel layer.
 *
 * Random numbers: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
 * numbers: as easy as 1, 2, 3", SC'11), key = (seed low word, stream),
 * counter = (block index low, block index high, seed high word, 0).  A standard-normal-like variate
 * is the classical sum of twelve uniforms minus six, with each uniform taken
 * as the top 20 bits of one Philox output word.  The sum is an integer below
 * 2^24, so it converts to fp32 exactly, and the scale by 2^-20 and the
 * subtraction of 6 are exact too: the value depends on integer arithmetic
 * only, and the CUDA twin of this generator (gen_dev.cu) reproduces it bit
 * for bit.  Mean 0, variance 1, support [-6, 6).
 *
 * Multithreaded with pthreads; every element depends only on (seed, stream,
 * index), so the thread split does not change the output.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

static inline void philox4x32_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
  for (int r = 0; r < 10; ++r) {
    uint64_t p0 = (uint64_t)PHILOX_M0 * c[0];
    uint64_t p1 = (uint64_t)PHILOX_M1 * c[2];
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c[1] ^ k0;
    uint32_t n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
    k0 += PHILOX_W0;
    k1 += PHILOX_W1;
  }
}

/* Philox block b of (seed, stream): four 32-bit words.
 * key = (seed low word, stream); counter = (b low, b high, seed high, 0). */
static inline void philox_block(uint64_t seed, uint32_t stream, uint64_t b, uint32_t out[4]) {
  out[0] = (uint32_t)b;
  out[1] = (uint32_t)(b >> 32);
  out[2] = (uint32_t)(seed >> 32);
  out[3] = 0;
  philox4x32_10(out, (uint32_t)seed, stream);
}

/* Element i uses Philox blocks 3i, 3i+1, 3i+2 (twelve words). */
float gen_normal12_at(uint64_t seed, uint32_t stream, uint64_t i) {
  uint32_t sum = 0;
  for (int b = 0; b < 3; ++b) {
    uint32_t w[4];
    philox_block(seed, stream, 3 * i + (uint64_t)b, w);
    sum += (w[0] >> 12) + (w[1] >> 12) + (w[2] >> 12) + (w[3] >> 12);
  }
  float s = (float)sum;         /* exact: sum < 2^24 */
  float scaled = s * 0x1p-20f;  /* exact: power-of-two scale */
  return scaled - 6.0f;         /* exact: |result| < 8 on a 2^-20 grid */
}

/* fp32 -> bf16 bits, round to nearest even (finite inputs only). */
static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ */
/* thread pool helper                                                 */

typedef struct {
  int kind; /* 0: f32, 1: bf16 */
  uint64_t seed;
  uint32_t stream;
  uint64_t offset;
  int64_t begin, end;
  void* out;
} fill_job;

static void* fill_worker(void* arg) {
  fill_job* j = (fill_job*)arg;
  for (int64_t i = j->begin; i < j->end; ++i) {
    float z = gen_normal12_at(j->seed, j->stream, j->offset + (uint64_t)i);
    if (j->kind == 0)
      ((float*)j->out)[i] = z;
    else
      ((uint16_t*)j->out)[i] = f32_to_bf16_rne(z);
  }
  return NULL;
}

static void fill_parallel(int kind, uint64_t seed, uint32_t stream, uint64_t offset, int64_t n, void* out,
                          int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (n < 65536) nthreads = 1;
  pthread_t th[256];
  fill_job jobs[256];
  int64_t per = (n + nthreads - 1) / nthreads;
  int launched = 0;
  for (int t = 0; t < nthreads; ++t) {
    int64_t b = (int64_t)t * per, e = b + per;
    if (e > n) e = n;
    if (b >= e) break;
    jobs[t] = (fill_job){kind, seed, stream, offset, b, e, out};
    if (nthreads == 1) {
      fill_worker(&jobs[t]);
    } else {
      pthread_create(&th[t], NULL, fill_worker, &jobs[t]);
      ++launched;
    }
  }
  for (int t = 0; t < launched; ++t) pthread_join(th[t], NULL);
}

/* out[i] = normal12(seed, stream, offset + i), i in [0, n) */
void gen_fill_normal_f32(uint64_t seed, uint32_t stream, uint64_t offset, int64_t n, float* out, int nthreads) {
  fill_parallel(0, seed, stream, offset, n, out, nthreads);
}

/* out[i] = bf16_rne(normal12(seed, stream, offset + i)) */
void gen_fill_normal_bf16(uint64_t seed, uint32_t stream, uint64_t offset, int64_t n, uint16_t* out,
                          int nthreads) {
  fill_parallel(1, seed, stream, offset, n, out, nthreads);
}

/* ------------------------------------------------------------------ */
/* router: logits -> top-K ids (descending logit, ties to lower id) and */
/* gate weights = softmax over the K chosen logits                     */

typedef struct {
  uint64_t seed;
  uint32_t stream;
  int64_t t0, t1; /* token range */
  int E, K;
  const float* bias;   /* [E] */
  int force_expert0;   /* single-expert case: logit[t,0] := max(row) + 1 */
  int uniform_ids;     /* uniform case: ids (t*K+k) mod E */
  int32_t* topk;       /* [T, K] */
  float* w;            /* [T, K] */
} route_job;

static void* route_worker(void* arg) {
  route_job* j = (route_job*)arg;
  int E = j->E, K = j->K;
  float* row = (float*)malloc(sizeof(float) * (size_t)E);
  int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)K);
  float* chosen = (float*)malloc(sizeof(float) * (size_t)K);
  unsigned char* taken = (unsigned char*)malloc((size_t)E);
  for (int64_t t = j->t0; t < j->t1; ++t) {
    for (int e = 0; e < E; ++e)
      row[e] = gen_normal12_at(j->seed, j->stream, (uint64_t)t * (uint64_t)E + (uint64_t)e) + j->bias[e];
    if (j->force_expert0) {
      float mx = row[0];
      for (int e = 1; e < E; ++e)
        if (row[e] > mx) mx = row[e];
      row[0] = mx + 1.0f;
    }
    if (j->uniform_ids) {
      for (int k = 0; k < K; ++k) {
        ids[k] = (int32_t)(((int64_t)t * K + k) % E);
        chosen[k] = row[ids[k]];
      }
    } else {
      memset(taken, 0, (size_t)E);
      for (int k = 0; k < K; ++k) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
          if (taken[e]) continue;
          if (best < 0 || row[e] > row[best]) best = e; /* strict '>' keeps the lower id on ties */
        }
        taken[best] = 1;
        ids[k] = best;
        chosen[k] = row[best];
      }
    }
    double mx = chosen[0];
    for (int k = 1; k < K; ++k)
      if (chosen[k] > mx) mx = chosen[k];
    double z = 0.0;
    for (int k = 0; k < K; ++k) z += exp((double)chosen[k] - mx);
    for (int k = 0; k < K; ++k) {
      j->topk[t * K + k] = ids[k];
      j->w[t * K + k] = (float)(exp((double)chosen[k] - mx) / z);
    }
  }
  free(row);
  free(ids);
  free(chosen);
  free(taken);
  return NULL;
}

/*
 * topk[T,K], w[T,K] for tokens [0, T).  bias[E] is added to every row of
 * normal12 logits drawn from (seed, stream) at index t*E + e.
 */
void gen_routing(uint64_t seed, uint32_t stream, int64_t T, int E, int K, const float* bias, int force_expert0,
                 int uniform_ids, int32_t* topk, float* w, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (T < 1024) nthreads = 1;
  pthread_t th[256];
  route_job jobs[256];
  int64_t per = (T + nthreads - 1) / nthreads;
  int launched = 0;
  for (int i = 0; i < nthreads; ++i) {
    int64_t b = (int64_t)i * per, e = b + per;
    if (e > T) e = T;
    if (b >= e) break;
    jobs[i] = (route_job){seed, stream, b, e, E, K, bias, force_expert0, uniform_ids, topk, w};
    if (nthreads == 1) {
      route_worker(&jobs[i]);
    } else {
      pthread_create(&th[i], NULL, route_worker, &jobs[i]);
      ++launched;
    }
  }
  for (int i = 0; i < launched; ++i) pthread_join(th[i], NULL);
}
