/* Bulk random draws for the synthetic workloads (trits and residual sites).
 *
 * Counter-based SplitMix64 (Steele, Lea & Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014): the i-th output of the
 * stream with seed s is mix(s + (i + 1) * 0x9E3779B97F4A7C15), where mix is
 * the published 64-bit finaliser.  Because every output depends only on
 * (seed, counter), the result does not depend on the number of threads.
 *
 * Nothing here packs, decodes or multiplies anything: it only draws the
 * dense component arrays that both the oracle and the CUDA library consume.
 */
#include <stdint.h>

static inline uint64_t sm64_draw(uint64_t seed, uint64_t i) {
  uint64_t z = seed + (i + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* T[i] in {-1, 0, +1}: each 64-bit draw gives four 16-bit uniforms u;
 * t = -1 if u < thr_neg, 0 if u < thr_pos, else +1. */
void wal_synth_trits(int8_t* T, int64_t n, uint64_t seed, uint32_t thr_neg, uint32_t thr_pos) {
  int64_t nb = (n + 3) / 4;
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < nb; ++b) {
    uint64_t r = sm64_draw(seed, (uint64_t)b);
    for (int q = 0; q < 4; ++q) {
      int64_t i = 4 * b + q;
      if (i >= n) break;
      uint32_t u = (uint32_t)((r >> (16 * q)) & 0xFFFFu);
      T[i] = (int8_t)(u < thr_neg ? -1 : (u < thr_pos ? 0 : 1));
    }
  }
}

/* k distinct uniform positions in [0, 128) per group by Floyd's subset
 * sampling, stored ascending, with fair +-1 signs.  Draw counters for group g
 * are 16 g + i (positions) and 16 g + 15 (sign bits). */
void wal_synth_sites(uint8_t* pos, int8_t* sign, int64_t n_groups, int k, uint64_t seed) {
#pragma omp parallel for schedule(static)
  for (int64_t g = 0; g < n_groups; ++g) {
    uint8_t chosen[8];
    for (int i = 0; i < k; ++i) {
      uint32_t j = (uint32_t)(128 - k + i);
      uint64_t d = sm64_draw(seed, 16 * (uint64_t)g + (uint64_t)i);
      uint32_t t = (uint32_t)(((d >> 32) * (uint64_t)(j + 1)) >> 32);
      for (int q = 0; q < i; ++q)
        if (chosen[q] == t) { t = j; break; }
      chosen[i] = (uint8_t)t;
    }
    for (int i = 1; i < k; ++i) { /* insertion sort, k <= 8 */
      uint8_t v = chosen[i]; int q = i - 1;
      while (q >= 0 && chosen[q] > v) { chosen[q + 1] = chosen[q]; --q; }
      chosen[q + 1] = v;
    }
    uint64_t sb = sm64_draw(seed, 16 * (uint64_t)g + 15);
    for (int i = 0; i < k; ++i) {
      pos[g * k + i] = chosen[i];
      sign[g * k + i] = (int8_t)(((sb >> i) & 1) ? -1 : 1);
    }
  }
}
