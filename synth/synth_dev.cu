/*
 * Device side of the synthetic-input generator: fills HBM with exactly the
 * values synth_host.c produces on the CPU (compiled with --fmad=false so that
 * every double operation is a separately rounded IEEE operation).
 *
 * A "family" fill writes the same tensor kind for a run of experts laid out
 * with a fixed byte stride: expert e's tensor starts at base + e*stride and
 * takes its values from stream (seed, a, b0 + e, tensor).
 */
#include "synth_core.h"
#include <cuda_runtime.h>

__global__ void sy_fill_family_kernel(char* base, uint64_t stride, uint64_t n_per,
                                      uint32_t n_members, int kind, uint64_t seed,
                                      uint32_t a, uint32_t b0, uint32_t tensor,
                                      double p0, double p1) {
  const uint64_t total = n_per * (uint64_t)n_members;
  const int eb = sy_kind_bytes(kind);
  uint32_t cur_m = 0xFFFFFFFFu;
  uint64_t key = 0;
  for (uint64_t t = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (uint64_t)gridDim.x * blockDim.x) {
    uint32_t m = (uint32_t)(t / n_per);
    uint64_t i = t - (uint64_t)m * n_per;
    if (m != cur_m) { cur_m = m; key = sy_key(seed, a, b0 + m, tensor); }
    uint32_t v = sy_element(kind, key, i, p0, p1);
    char* dst = base + (uint64_t)m * stride + i * (uint64_t)eb;
    if (eb == 2) *(uint16_t*)dst = (uint16_t)v;
    else *(uint32_t*)dst = v;
  }
}

extern "C" int sy_dev_fill_family(void* base, uint64_t stride_bytes, uint64_t n_per,
                                  uint32_t n_members, int kind, uint64_t seed, uint32_t a,
                                  uint32_t b0, uint32_t tensor, double p0, double p1,
                                  void* stream) {
  if (n_per == 0 || n_members == 0) return 0;
  if (!base) return -1;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  uint64_t total = n_per * (uint64_t)n_members;
  uint64_t want = (total + 255) / 256;
  unsigned grid = (unsigned)(want < (uint64_t)sms * 16 ? want : (uint64_t)sms * 16);
  sy_fill_family_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(
      (char*)base, stride_bytes, n_per, n_members, kind, seed, a, b0, tensor, p0, p1);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}
