/*
 * plain_rht_quant.c -- the plain CPU baseline of the rotate + quantise step.
 *
 * TEST INFRASTRUCTURE ONLY (like the rest of oracle/): timed beside the GPU as the honest
 * CPU speed line, never called by the library. Shares no code with the CUDA path.
 *
 * Per row, in the style of the Hadamard-Int4-Accuracy wiki's probe (Method: fwht_norm,
 * q_dequant_vec): apply the random signs, run the in-place radix-2 fast Walsh-Hadamard
 * transform (log2 K passes of a+b / a-b over pairs at distance h = 1, 2, 4, ...), scale by
 * 1/sqrt(K), then per group of G coordinates: absmax, binary16 scale s = fp16(absmax / qmax),
 * q = clamp(round_half_away(y / s), -qmax, qmax) (s == 0 gives 0), packed two's complement
 * (int4: byte j = q[2j] | q[2j+1] << 4; int2: byte j holds q[4j+i] in bits 2i..2i+1).
 * Everything is fp32 scalar C with O(K log K) work per row; rows run in parallel (OpenMP).
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC plain_rht_quant.c -o _lib/libplain_rht_quant.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* IEEE binary32 -> binary16, round to nearest even (written from the format definitions). */
static uint16_t f32_to_f16(float f) {
  uint32_t x;
  memcpy(&x, &f, 4);
  const uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
  const uint32_t ax = x & 0x7fffffffu;
  if (ax > 0x7f800000u) return sign | 0x7e00u;   /* NaN */
  if (ax == 0x7f800000u) return sign | 0x7c00u;  /* inf */
  if (ax == 0) return sign;
  int e = (int)(ax >> 23) - 127;
  uint32_t m = ax & 0x7fffffu;
  if (e == -127) e = -126;                       /* binary32 subnormal: no hidden bit */
  else m |= 0x800000u;
  int shift, he;
  if (e >= -14) { shift = 13; he = e + 15; }     /* binary16 normal: keep 11 bits */
  else { shift = 13 + (-14 - e); he = 0; }       /* binary16 subnormal: unit 2^-24 */
  if (shift > 31) return sign;
  uint32_t q = m >> shift;
  const uint32_t rem = m & ((1u << shift) - 1u), half = 1u << (shift - 1);
  if (rem > half || (rem == half && (q & 1u))) q++;
  const uint32_t bits = he == 0 ? q : (((uint32_t)he << 10) + (q - 0x400u));
  if (bits >= 0x7c00u) return sign | 0x7c00u;
  return (uint16_t)(sign | bits);
}

static float f16_to_f32(uint16_t h) {
  const uint32_t e = (h >> 10) & 0x1fu, m = h & 0x3ffu;
  float v;
  if (e == 0) v = ldexpf((float)m, -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexpf((float)(m | 0x400u), (int)e - 25);
  return (h & 0x8000u) ? -v : v;
}

/* Rotate + quantise M rows of A (fp32, row pitch lda). signs: K entries +-1 or NULL.
 * codes: [M, K*bits/8]; scales: [M, K/G] binary16 bits. Returns 0, or -1 on bad arguments. */
int plain_rht_quant(const float* A, int64_t M, int64_t lda, int K, const int8_t* signs, int bits, int G,
                    uint8_t* codes, uint16_t* scales, int threads) {
  if (K < 2 || (K & (K - 1)) != 0 || (bits != 4 && bits != 2) || G <= 0 || K % G != 0 || G % (8 / bits) != 0)
    return -1;
  const float qmax = bits == 4 ? 7.0f : 1.0f;
  const float norm = (float)(1.0 / sqrt((double)K));
  const int per = 8 / bits;
  const int64_t cbytes = (int64_t)K / per;
#ifdef _OPENMP
  if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel
#endif
  {
    float* x = (float*)malloc(sizeof(float) * (size_t)K);
    int* q = (int*)malloc(sizeof(int) * (size_t)G);
#ifdef _OPENMP
#pragma omp for schedule(static)
#endif
    for (int64_t r = 0; r < M; ++r) {
      const float* a = A + r * lda;
      for (int k = 0; k < K; ++k) x[k] = signs ? (float)signs[k] * a[k] : a[k];
      for (int h = 1; h < K; h <<= 1)
        for (int i = 0; i < K; i += 2 * h)
          for (int j = i; j < i + h; ++j) {
            const float u = x[j], v = x[j + h];
            x[j] = u + v;
            x[j + h] = u - v;
          }
      for (int k = 0; k < K; ++k) x[k] *= norm;
      uint8_t* crow = codes + r * cbytes;
      for (int g0 = 0; g0 < K; g0 += G) {
        float m = 0.0f;
        for (int j = 0; j < G; ++j) m = fmaxf(m, fabsf(x[g0 + j]));
        const uint16_t sh = f32_to_f16(m / qmax);
        const float s = f16_to_f32(sh);
        scales[r * (K / G) + g0 / G] = sh;
        for (int j = 0; j < G; ++j) {
          int c = 0;
          if (s != 0.0f) {
            float v = roundf(x[g0 + j] / s);
            if (v > qmax) v = qmax;
            if (v < -qmax) v = -qmax;
            c = (int)v;
          }
          q[j] = c;
        }
        for (int j = 0; j < G; j += per) {
          unsigned b = 0;
          for (int i = 0; i < per; ++i) b |= ((unsigned)q[j + i] & ((1u << bits) - 1u)) << (bits * i);
          crow[(g0 + j) / per] = (uint8_t)b;
        }
      }
    }
    free(q);
    free(x);
  }
  return 0;
}

int plain_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
