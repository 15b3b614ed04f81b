// qe_device.cuh -- device building blocks of the sm_100a kernels:
// bf16 decode, bounded waits, mbarrier / bulk-copy wrappers and the
// dequant-dot cores of the 4-bit and 2-bit matvecs.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "qe_internal.h"

#define QE_DEV __device__ __forceinline__

namespace qe {

QE_DEV float bf16f(uint32_t h16) { return __uint_as_float(h16 << 16); }

QE_DEV uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

QE_DEV uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// ------------------------------------------------------------ global sync

QE_DEV unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

QE_DEV void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Record the first device-side error in the workspace status word.
QE_DEV void set_error(int* err, int code) { atomicCAS(err, 0, code); }

// Spin (bounded) until *ctr >= target.  Returns false on timeout or if the
// CTA-wide abort flag is raised.
QE_DEV bool wait_geq(const unsigned* ctr, unsigned target, uint64_t deadline,
                     volatile int* abort_flag) {
  unsigned spins = 0;
  while (ld_acquire(ctr) < target) {
    if (*abort_flag) return false;
    if ((++spins & 15u) == 0 && gtimer() > deadline) return false;
    __nanosleep(32);
  }
  return true;
}

// ------------------------------------------------------------- mbarriers

QE_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

QE_DEV void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

QE_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

QE_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

QE_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.
QE_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t deadline, volatile int* abort_flag) {
  unsigned spins = 0;
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if ((++spins & 7u) == 0 && gtimer() > deadline) return false;
  }
  return true;
}

// ------------------------------------------------------------ bulk copies

// L2 policy: streamed expert weights are read once per token, so they are
// marked evict-first and do not push the router or activations out of L2.
QE_DEV uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Global -> shared bulk copy (no tensor map, no multicast); completion is
// counted in bytes on `bar`.  dst, src and bytes must be 16-byte multiples.
QE_DEV void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

// -------------------------------------------------------- warp reductions

QE_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

QE_DEV double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

QE_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Sum R per-lane values over the warp at once (R a power of two <= 32).
// Stage o halves the live values: lanes with bit o set keep the upper half.
// Afterwards the total of value i sits in every lane whose bits
// (lane>>4, lane>>3, ...) spell i in binary (most significant first);
// reduced_row_of_lane() gives that index.
template <int R>
QE_DEV float warp_reduce_rows(float (&v)[R], int lane) {
  int live = R;
  int o = 16;
#pragma unroll
  for (; live > 1; o >>= 1) {
    const bool up = (lane & o) != 0;
    const int half = live / 2;
#pragma unroll
    for (int i = 0; i < R / 2; ++i) {
      if (i < half) {
        float keep = up ? v[i + half] : v[i];
        float send = up ? v[i] : v[i + half];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    live = half;
  }
  float s = v[0];
  for (; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

template <int R>
QE_DEV int reduced_row_of_lane(int lane) {
  int row = 0;
  int o = 16;
#pragma unroll
  for (int live = R; live > 1; live >>= 1, o >>= 1) row = row * 2 + ((lane & o) ? 1 : 0);
  return row;
}

template <int R>
QE_DEV int lane_of_reduced_row(int row) {
  // first lane holding row `row`
  int lane = 0;
  int o = 16;
  int bit = R / 2;
#pragma unroll
  for (int live = R; live > 1; live >>= 1, o >>= 1, bit >>= 1) lane |= (row & bit) ? o : 0;
  return lane;
}

// ------------------------------------------------------- dequant-dot cores
//
// A q field is turned into a float without a conversion instruction: the
// word is masked so the field keeps its place below bit 23, and the masked
// word read as a float is the subnormal q * 2^(p-149), p = the field's bit
// offset.  The activation is pre-scaled per column by 2^(89-p-E) (see
// xscale_q4 / xscale_q2), so every product is exactly q*x*2^(-60-E) before
// the single fp32 rounding of the fused multiply-add.  Two products go
// through one packed f32x2 FMA.  Fields above bit 22 are first shifted down
// by 12.  Per group the dot product is then
//   sum_c (q_c*s + b) x_c = s * 2^(60+E) * acc + b * sum_c x_c.
// Subnormal operands and results must not be flushed: never build these
// kernels with -ftz=true or --use_fast_math.

// Field offset p of column j (0..7) of a 4-bit word after the mapping above.
QE_DEV int q4_field_pos(int j) { return j < 5 ? 4 * j : 4 * j - 12; }
// Field offset p of column j (0..15) of a 2-bit word.
QE_DEV int q2_field_pos(int j) { return j < 11 ? 2 * j : 2 * j - 12; }

QE_DEV float f_of(uint32_t u) { return __uint_as_float(u); }

// One uint4 of 4-bit weights (32 columns) against pre-scaled x' (16 float2).
QE_DEV float2 dot32_q4(const uint4 w, const float2* xs, float2 acc) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t v = ws[i];
    const uint32_t hv = v >> 12;
    acc = __ffma2_rn(make_float2(f_of(v & 0xFu), f_of(v & 0xF0u)), xs[4 * i + 0], acc);
    acc = __ffma2_rn(make_float2(f_of(v & 0xF00u), f_of(v & 0xF000u)), xs[4 * i + 1], acc);
    acc = __ffma2_rn(make_float2(f_of(v & 0xF0000u), f_of(hv & 0xF00u)), xs[4 * i + 2], acc);
    acc = __ffma2_rn(make_float2(f_of(hv & 0xF000u), f_of(hv & 0xF0000u)), xs[4 * i + 3], acc);
  }
  return acc;
}

// One uint4 of 2-bit weights (64 columns, one group) against x' (32 float2).
QE_DEV float2 dot64_q2(const uint4 w, const float2* xs, float2 acc) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t v = ws[i];
    const uint32_t hv = v >> 12;
    const float2* x = xs + 8 * i;
    acc = __ffma2_rn(make_float2(f_of(v & 0x3u), f_of(v & 0xCu)), x[0], acc);
    acc = __ffma2_rn(make_float2(f_of(v & 0x30u), f_of(v & 0xC0u)), x[1], acc);
    acc = __ffma2_rn(make_float2(f_of(v & 0x300u), f_of(v & 0xC00u)), x[2], acc);
    acc = __ffma2_rn(make_float2(f_of(v & 0x3000u), f_of(v & 0xC000u)), x[3], acc);
    acc = __ffma2_rn(make_float2(f_of(v & 0x30000u), f_of(v & 0xC0000u)), x[4], acc);
    acc = __ffma2_rn(make_float2(f_of(v & 0x300000u), f_of(hv & 0xC00u)), x[5], acc);
    acc = __ffma2_rn(make_float2(f_of(hv & 0x3000u), f_of(hv & 0xC000u)), x[6], acc);
    acc = __ffma2_rn(make_float2(f_of(hv & 0x30000u), f_of(hv & 0xC0000u)), x[7], acc);
  }
  return acc;
}

// Vector exponent E = exponent(amax) - 30, clamped to [-38, 60]: x' stays
// below 2^121 and the products q*x*2^(-60-E) stay near 2^-30 * q, far from
// both overflow and the subnormal range, for any |x| in [2^-68, 2^90).
QE_DEV int xscale_exponent(float amax) {
  if (!(amax > 0.0f)) return 0;
  int e = ((int)((__float_as_uint(amax) >> 23) & 0xFF)) - 127;
  int E = e - 30;
  return E < -38 ? -38 : (E > 60 ? 60 : E);
}

// x' of column c for 4-bit / 2-bit matrices.
QE_DEV float xprime_q4(float x, int c, int E) {
  return x * __int_as_float((127 + 89 - q4_field_pos(c & 7) - E) << 23);
}
QE_DEV float xprime_q2(float x, int c, int E) {
  return x * __int_as_float((127 + 89 - q2_field_pos(c & 15) - E) << 23);
}
// 2^(60+E): turns acc back into sum q*x.
QE_DEV float acc_scale(int E) { return __int_as_float((127 + 60 + E) << 23); }

}  // namespace qe
