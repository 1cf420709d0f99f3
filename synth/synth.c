/*
 * Seeded synthetic workload generator for hierarchical block-sparse attention.
 *
 * This module only draws inputs. It holds none of the method's arithmetic
 * (no pooling, no scoring, no selection, no attention). Both the CPU oracle
 * and the CUDA path receive the tensors it writes, so the two sides always
 * see bit-identical inputs.
 *
 * Random numbers: a counter-based generator. Every value is a pure function
 * of (seed, stream, counter), so tensors can be filled in parallel and in any
 * order. The bit mixer is the SplitMix64 finaliser (Steele, Lea and Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014, with the
 * mixing constants published by Vigna). Uniforms take the top 53 bits;
 * normals use the Box-Muller transform (Box and Muller, 1958) on the pair of
 * uniforms (2p, 2p+1), the even counter taking the cosine branch.
 *
 * Workload recipe (the structure of the long-context retrieval workloads that
 * the PISA and PHBA pages evaluate on; datasets are not available here):
 *   Q, K, V ~ N(0, 1) iid.
 *   Each key block j of each (batch, kv head) gets an offset vector
 *   o_j ~ N(0, sigma_off^2 I_d) added to all of its keys.
 *   Planted needles: for query block i = 1 .. nqb-1 in ascending order,
 *   min(n_needle, i) distinct earlier key blocks j < i are drawn; every key
 *   of block j is overwritten with 2 * mean(query rows of block i, over the
 *   kv group's heads) + N(0, 0.1^2); owner[j] = i records the last writer.
 *   Decode workloads (one query row at position N-1) plant n_needle blocks
 *   in [0, i_q) aligned to that single query row.
 *
 * Storage: fp32, or bf16 rounded to nearest-even from the fp32 draw.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define STREAM_Q 0u
#define STREAM_K 1u
#define STREAM_V 2u
#define STREAM_OFF 3u
#define STREAM_NOISE 4u
#define STREAM_POS 5u

enum { SYN_F32 = 0, SYN_BF16 = 1 };
enum { NEEDLE_UNIFORM = 0, NEEDLE_LOGUNIFORM = 1, NEEDLE_DECODE = 2 };

static inline uint64_t splitmix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* 64 random bits for (seed, stream, counter); counters up to 2^56. */
static inline uint64_t draw_bits(uint64_t seed, uint32_t stream, uint64_t ctr) {
  uint64_t key = splitmix64(seed ^ splitmix64(0xA5A5A5A500000000ull + stream));
  return splitmix64(key ^ (ctr * 0xD1342543DE82EF95ull));
}

/* Uniform in the open interval (0, 1). */
static inline double draw_uniform(uint64_t seed, uint32_t stream, uint64_t ctr) {
  return ((double)(draw_bits(seed, stream, ctr) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

/* Standard normal number `ctr` of a stream (Box-Muller on uniform pair). */
static inline double draw_normal(uint64_t seed, uint32_t stream, uint64_t ctr) {
  uint64_t p = ctr >> 1;
  double u1 = draw_uniform(seed, stream, 2 * p);
  double u2 = draw_uniform(seed, stream, 2 * p + 1);
  double r = sqrt(-2.0 * log(u1));
  double a = 6.283185307179586476925286766559 * u2;
  return (ctr & 1) ? r * sin(a) : r * cos(a);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16); /* inf/nan */
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static inline float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static inline void store(void* base, int dtype, uint64_t i, double v) {
  if (dtype == SYN_F32)
    ((float*)base)[i] = (float)v;
  else
    ((uint16_t*)base)[i] = f32_to_bf16_rne((float)v);
}

static inline double load(const void* base, int dtype, uint64_t i) {
  if (dtype == SYN_F32) return (double)((const float*)base)[i];
  return (double)bf16_to_f32(((const uint16_t*)base)[i]);
}

/* Fill `n` consecutive normals of one stream, scaled, into dst[0..n). */
int syn_fill_normal(uint64_t seed, uint32_t stream, void* dst, int dtype, uint64_t n, double scale) {
  if (!dst) return 1;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < (int64_t)n; i++) store(dst, dtype, (uint64_t)i, scale * draw_normal(seed, stream, (uint64_t)i));
  return 0;
}

/* Uniform doubles in (0,1): used by tests that need seeded scalars. */
int syn_fill_uniform(uint64_t seed, uint32_t stream, double* dst, uint64_t n) {
  if (!dst) return 1;
  for (uint64_t i = 0; i < n; i++) dst[i] = draw_uniform(seed, stream, i);
  return 0;
}

/* Draw a needle source block for query block i, attempt a (0-based). */
static int64_t needle_block(uint64_t seed, int mode, uint64_t unit, int64_t i, int a) {
  double u = draw_uniform(seed, STREAM_POS, (unit * 1048576ull + (uint64_t)i) * 4096ull + (uint64_t)a);
  if (mode == NEEDLE_LOGUNIFORM) {
    /* distance delta = i - j, log-uniform on [1, i] */
    double delta = floor(exp(u * log((double)i)) + 0.5);
    if (delta < 1.0) delta = 1.0;
    if (delta > (double)i) delta = (double)i;
    return i - (int64_t)delta;
  }
  int64_t j = (int64_t)floor(u * (double)i);
  if (j >= i) j = i - 1;
  return j;
}

/*
 * Fill one workload.
 *   Q: [B][Hq][Nq][d], K, V: [B][Hkv][N][d] in `dtype`.
 *   owner: [B][Hkv][nb] int32 (nullable); -1 where no needle was planted.
 * Query row t sits at position q_offset + t. Prefill has Nq = N, q_offset = 0.
 * Decode has Nq = 1, q_offset = N - 1 and needle mode NEEDLE_DECODE.
 * Returns 0 on success.
 */
int syn_workload(uint64_t seed, int B, int Hq, int Hkv, int N, int Nq, int q_offset, int d, int bs,
                 int dtype, double sigma_off, int n_needle, int needle_mode, double needle_noise,
                 void* Q, void* K, void* V, int32_t* owner) {
  if (!Q || !K || !V || B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || N <= 0 || Nq <= 0 || d <= 0 || bs <= 0)
    return 1;
  if (q_offset < 0 || q_offset + Nq > N) return 1;
  const int G = Hq / Hkv;
  const int64_t nb = (N + bs - 1) / bs;
  const uint64_t nq_el = (uint64_t)B * Hq * Nq * d;
  const uint64_t nk_el = (uint64_t)B * Hkv * N * d;

#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < (int64_t)nq_el; i++) store(Q, dtype, (uint64_t)i, draw_normal(seed, STREAM_Q, (uint64_t)i));
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < (int64_t)nk_el; i++) {
    uint64_t e = (uint64_t)i % (uint64_t)d;
    uint64_t row = (uint64_t)i / (uint64_t)d; /* (b*Hkv + h)*N + t */
    uint64_t unit = row / (uint64_t)N, t = row % (uint64_t)N;
    uint64_t oc = (unit * (uint64_t)nb + t / (uint64_t)bs) * (uint64_t)d + e;
    double k = draw_normal(seed, STREAM_K, (uint64_t)i) + sigma_off * draw_normal(seed, STREAM_OFF, oc);
    store(K, dtype, (uint64_t)i, k);
    store(V, dtype, (uint64_t)i, draw_normal(seed, STREAM_V, (uint64_t)i));
  }
  if (owner)
    for (int64_t i = 0; i < (int64_t)B * Hkv * nb; i++) owner[i] = -1;
  if (n_needle <= 0) return 0;

  const int64_t i_first = q_offset / bs, i_last = (q_offset + Nq - 1) / bs;
#pragma omp parallel for schedule(dynamic)
  for (int64_t unit = 0; unit < (int64_t)B * Hkv; unit++) {
    const int64_t bi = unit / Hkv, hk = unit % Hkv;
    double* mean = (double*)malloc(sizeof(double) * (size_t)d);
    int64_t* chosen = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_needle > 0 ? n_needle : 1));
    for (int64_t i = (i_first > 1 ? i_first : 1); i <= i_last; i++) {
      /* query rows of block i, relative row range [r0, r1) */
      int64_t p0 = i * bs, p1 = (i + 1) * bs;
      if (p0 < q_offset) p0 = q_offset;
      if (p1 > q_offset + Nq) p1 = q_offset + Nq;
      const int64_t r0 = p0 - q_offset, r1 = p1 - q_offset;
      for (int e = 0; e < d; e++) mean[e] = 0.0;
      for (int g = 0; g < G; g++) {
        const int64_t hq = hk * G + g;
        for (int64_t r = r0; r < r1; r++) {
          const uint64_t base = (((uint64_t)bi * Hq + hq) * Nq + r) * d;
          for (int e = 0; e < d; e++) mean[e] += load(Q, dtype, base + e);
        }
      }
      const double inv = 1.0 / (double)(G * (r1 - r0));
      for (int e = 0; e < d; e++) mean[e] *= inv;

      const int64_t limit = i; /* blocks strictly before i */
      int want = n_needle < limit ? n_needle : (int)limit;
      int got = 0;
      for (int a = 0; got < want && a < 4096; a++) {
        int64_t j = needle_block(seed, needle_mode == NEEDLE_LOGUNIFORM ? NEEDLE_LOGUNIFORM : NEEDLE_UNIFORM,
                                 (uint64_t)unit, i, a);
        int dup = 0;
        for (int c = 0; c < got; c++) dup |= (chosen[c] == j);
        if (!dup) chosen[got++] = j;
      }
      for (int c = 0; c < got; c++) {
        const int64_t j = chosen[c];
        const int64_t t0 = j * bs, t1 = (j + 1) * bs < N ? (j + 1) * bs : N;
        for (int64_t t = t0; t < t1; t++) {
          const uint64_t base = (((uint64_t)bi * Hkv + hk) * N + t) * d;
          for (int e = 0; e < d; e++)
            store(K, dtype, base + e, 2.0 * mean[e] + needle_noise * draw_normal(seed, STREAM_NOISE, base + e));
        }
        if (owner) owner[unit * nb + j] = (int32_t)i;
      }
    }
    free(mean);
    free(chosen);
  }
  return 0;
}
