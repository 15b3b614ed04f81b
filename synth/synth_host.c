/*
 * Host side of the synthetic-input generator: fills host buffers with the
 * same values the device fill (synth_dev.cu) writes into HBM.
 * Built with gcc -O2 -ffp-contract=off so no multiply-add is fused.
 */
#include "synth_core.h"
#include <stddef.h>

/* Fill elements [i0, i0+n) of stream (seed, a, b, tensor) into dst. */
int sy_host_fill(void* dst, uint64_t i0, uint64_t n, int kind, uint64_t seed,
                 uint32_t a, uint32_t b, uint32_t tensor, double p0, double p1) {
  if (!dst && n) return -1;
  uint64_t key = sy_key(seed, a, b, tensor);
  if (sy_kind_bytes(kind) == 2) {
    uint16_t* o = (uint16_t*)dst;
#pragma omp parallel for schedule(static) if (n > 65536)
    for (int64_t i = 0; i < (int64_t)n; ++i)
      o[i] = (uint16_t)sy_element(kind, key, i0 + (uint64_t)i, p0, p1);
  } else {
    uint32_t* o = (uint32_t*)dst;
#pragma omp parallel for schedule(static) if (n > 65536)
    for (int64_t i = 0; i < (int64_t)n; ++i)
      o[i] = sy_element(kind, key, i0 + (uint64_t)i, p0, p1);
  }
  return 0;
}

uint64_t sy_host_key(uint64_t seed, uint32_t a, uint32_t b, uint32_t tensor) {
  return sy_key(seed, a, b, tensor);
}

uint64_t sy_host_draw(uint64_t key, uint64_t i) { return sy_draw(key, i); }

double sy_host_normal(uint64_t key, uint64_t i) { return sy_normal(key, i); }
double sy_host_ln(double u) { return sy_ln(u); }
double sy_host_cos2pi(double v) { return sy_cos2pi(v); }
