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

/* Normals 2p and 2p + 1 of a stream: the cosine and the sine branch of one
 * Box-Muller pair (the same values draw_normal gives for either counter). */
static inline void draw_normal_pair(uint64_t seed, uint32_t stream, uint64_t p, double* even, double* odd) {
  double u1 = draw_uniform(seed, stream, 2 * p);
  double u2 = draw_uniform(seed, stream, 2 * p + 1);
  double r = sqrt(-2.0 * log(u1));
  double a = 6.283185307179586476925286766559 * u2;
  *even = r * cos(a);
  *odd = r * sin(a);
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

/* Fill `n` consecutive normals of one stream, scaled, into dst[0..n); one
 * Box-Muller pair per two elements. */
int syn_fill_normal(uint64_t seed, uint32_t stream, void* dst, int dtype, uint64_t n, double scale) {
  if (!dst) return 1;
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < (int64_t)(n / 2); p++) {
    double a, b;
    draw_normal_pair(seed, stream, (uint64_t)p, &a, &b);
    store(dst, dtype, 2 * (uint64_t)p, scale * a);
    store(dst, dtype, 2 * (uint64_t)p + 1, scale * b);
  }
  if (n & 1) store(dst, dtype, n - 1, scale * draw_normal(seed, stream, n - 1));
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
  if (!Q || !K || !V || B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || N <= 0 || Nq <= 0 || d <= 0 || d > 1024 ||
      bs <= 0)
    return 1;
  if (q_offset < 0 || q_offset + Nq > N) return 1;
  const int G = Hq / Hkv;
  const int64_t nb = (N + bs - 1) / bs;
  const uint64_t nq_el = (uint64_t)B * Hq * Nq * d;
  const uint64_t nk_el = (uint64_t)B * Hkv * N * d;

  /* element i of Q is normal i of STREAM_Q; element i = row * d + e of K is
   * normal i of STREAM_K plus sigma_off times normal (unit * nb + block) * d + e
   * of STREAM_OFF (one offset vector per key block); V is STREAM_V. Pairs of
   * normals come from one Box-Muller draw; a block's offsets are drawn once. */
  syn_fill_normal(seed, STREAM_Q, Q, dtype, nq_el, 1.0);
  const int64_t nblk = (int64_t)B * Hkv * nb;
  if (d % 2 == 0) {
#pragma omp parallel for schedule(static)
    for (int64_t ub = 0; ub < nblk; ub++) {
      const uint64_t unit = (uint64_t)(ub / nb), blk = (uint64_t)(ub % nb);
      double off[1024];
      for (int e = 0; e < d && e < 1024; e += 2)
        draw_normal_pair(seed, STREAM_OFF, ((uint64_t)ub * (uint64_t)d + (uint64_t)e) / 2, &off[e], &off[e + 1]);
      const uint64_t t0 = blk * (uint64_t)bs, t1 = (blk + 1) * (uint64_t)bs < (uint64_t)N ? (blk + 1) * (uint64_t)bs
                                                                                          : (uint64_t)N;
      for (uint64_t t = t0; t < t1; t++) {
        const uint64_t base = (unit * (uint64_t)N + t) * (uint64_t)d;
        for (int e = 0; e < d; e += 2) {
          double k0, k1, v0, v1;
          draw_normal_pair(seed, STREAM_K, (base + (uint64_t)e) / 2, &k0, &k1);
          draw_normal_pair(seed, STREAM_V, (base + (uint64_t)e) / 2, &v0, &v1);
          store(K, dtype, base + e, k0 + sigma_off * off[e]);
          store(K, dtype, base + e + 1, k1 + sigma_off * off[e + 1]);
          store(V, dtype, base + e, v0);
          store(V, dtype, base + e + 1, v1);
        }
      }
    }
  } else {
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
  }
  if (owner)
    for (int64_t i = 0; i < (int64_t)B * Hkv * nb; i++) owner[i] = -1;
  if (n_needle <= 0) return 0;

  /* Needles: for query blocks i ascending, min(n_needle, i) distinct earlier
   * blocks j get keys 2 * mean(query rows of block i over the group's heads)
   * + needle_noise * normal(element index) of STREAM_NOISE. A later i that
   * picks the same j overwrites it, and the noise depends only on the element,
   * so the keys of block j are those of its last writer: the owners are found
   * first, then every owned block is written once. */
  const int64_t i_first = q_offset / bs, i_last = (q_offset + Nq - 1) / bs;
#pragma omp parallel for schedule(dynamic)
  for (int64_t unit = 0; unit < (int64_t)B * Hkv; unit++) {
    const int64_t bi = unit / Hkv, hk = unit % Hkv;
    double* mean = (double*)malloc(sizeof(double) * (size_t)d);
    int64_t* chosen = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_needle > 0 ? n_needle : 1));
    int32_t* own = (int32_t*)malloc(sizeof(int32_t) * (size_t)nb);
    for (int64_t j = 0; j < nb; j++) own[j] = -1;
    for (int64_t i = (i_first > 1 ? i_first : 1); i <= i_last; i++) {
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
      for (int c = 0; c < got; c++) own[chosen[c]] = (int32_t)i;
    }
    for (int64_t j = 0; j < nb; j++) {
      const int64_t i = own[j];
      if (i < 0) continue;
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
      const int64_t t0 = j * bs, t1 = (j + 1) * bs < N ? (j + 1) * bs : N;
      for (int64_t t = t0; t < t1; t++) {
        const uint64_t base = (((uint64_t)bi * Hkv + hk) * N + t) * d;
        int e = 0;
        if (base % 2 == 0)
          for (; e + 1 < d; e += 2) {
            double n0, n1;
            draw_normal_pair(seed, STREAM_NOISE, (base + (uint64_t)e) / 2, &n0, &n1);
            store(K, dtype, base + e, 2.0 * mean[e] + needle_noise * n0);
            store(K, dtype, base + e + 1, 2.0 * mean[e + 1] + needle_noise * n1);
          }
        for (; e < d; e++)
          store(K, dtype, base + e, 2.0 * mean[e] + needle_noise * draw_normal(seed, STREAM_NOISE, base + e));
      }
      if (owner) owner[unit * nb + j] = (int32_t)i;
    }
    free(mean);
    free(chosen);
    free(own);
  }
  return 0;
}
