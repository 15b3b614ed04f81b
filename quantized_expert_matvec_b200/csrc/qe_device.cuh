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

// 16-byte asynchronous global -> shared copy (LDGSTS), L2 evict-first.
QE_DEV void cp_async16(void* dst, const void* src, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "l"(pol)
               : "memory");
}
QE_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
QE_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

QE_DEV void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p)); }
QE_DEV void prefetch_l1(const void* p) { asm volatile("prefetch.global.L1 [%0];" ::"l"(p)); }

// Named barrier over `count` threads (non-aligned form: counts threads).
QE_DEV void named_barrier(int id, int count) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Copy `bytes` (a multiple of 16) from global to shared with the 32 lanes of
// a warp, 16 bytes per lane per step.
QE_DEV void warp_copy_async(void* dst, const void* src, uint32_t bytes, int lane, uint64_t pol) {
  unsigned char* d = (unsigned char*)dst;
  const unsigned char* s = (const unsigned char*)src;
  for (uint32_t o = (uint32_t)lane * 16u; o < bytes; o += 512u) cp_async16(d + o, s + o, pol);
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
// xprime_q4 / xprime_q2), so every product is exactly q*x*2^(-60-E) before
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

// Eight 4-bit columns of one word against their x' (4 float2).
QE_DEV float2 dot8_q4(const uint32_t v, const float2* x, float2 acc) {
  const uint32_t hv = v >> 12;
  acc = __ffma2_rn(make_float2(f_of(v & 0xFu), f_of(v & 0xF0u)), x[0], acc);
  acc = __ffma2_rn(make_float2(f_of(v & 0xF00u), f_of(v & 0xF000u)), x[1], acc);
  acc = __ffma2_rn(make_float2(f_of(v & 0xF0000u), f_of(hv & 0xF00u)), x[2], acc);
  acc = __ffma2_rn(make_float2(f_of(hv & 0xF000u), f_of(hv & 0xF0000u)), x[3], acc);
  return acc;
}

// Sixteen 2-bit columns of one word against their x' (8 float2).
QE_DEV float2 dot16_q2(const uint32_t v, const float2* x, float2 acc) {
  const uint32_t hv = v >> 12;
  acc = __ffma2_rn(make_float2(f_of(v & 0x3u), f_of(v & 0xCu)), x[0], acc);
  acc = __ffma2_rn(make_float2(f_of(v & 0x30u), f_of(v & 0xC0u)), x[1], acc);
  acc = __ffma2_rn(make_float2(f_of(v & 0x300u), f_of(v & 0xC00u)), x[2], acc);
  acc = __ffma2_rn(make_float2(f_of(v & 0x3000u), f_of(v & 0xC000u)), x[3], acc);
  acc = __ffma2_rn(make_float2(f_of(v & 0x30000u), f_of(v & 0xC0000u)), x[4], acc);
  acc = __ffma2_rn(make_float2(f_of(v & 0x300000u), f_of(hv & 0xC00u)), x[5], acc);
  acc = __ffma2_rn(make_float2(f_of(hv & 0x3000u), f_of(hv & 0xC000u)), x[6], acc);
  acc = __ffma2_rn(make_float2(f_of(hv & 0x30000u), f_of(hv & 0xC0000u)), x[7], acc);
  return acc;
}

// Two words of 2-bit weights (32 columns) against x' (16 float2).
QE_DEV float2 dot32_q2(const uint2 w, const float2* xs, float2 acc) {
  float2 a2 = make_float2(0.f, 0.f);
  acc = dot16_q2(w.x, xs, acc);
  a2 = dot16_q2(w.y, xs + 8, a2);
  return make_float2(acc.x + a2.x, acc.y + a2.y);
}

// One uint4 of 4-bit weights (32 columns) against x' (16 float2); two
// accumulators so consecutive FMAs do not wait on each other.
QE_DEV float2 dot32_q4(const uint4 w, const float2* xs, float2 acc) {
  float2 a2 = make_float2(0.f, 0.f);
  acc = dot8_q4(w.x, xs, acc);
  a2 = dot8_q4(w.y, xs + 4, a2);
  acc = dot8_q4(w.z, xs + 8, acc);
  a2 = dot8_q4(w.w, xs + 12, a2);
  return make_float2(acc.x + a2.x, acc.y + a2.y);
}

// One uint4 of 2-bit weights (64 columns, one group) against x' (32 float2).
QE_DEV float2 dot64_q2(const uint4 w, const float2* xs, float2 acc) {
  float2 a2 = make_float2(0.f, 0.f);
  acc = dot16_q2(w.x, xs, acc);
  a2 = dot16_q2(w.y, xs + 8, a2);
  acc = dot16_q2(w.z, xs + 16, acc);
  a2 = dot16_q2(w.w, xs + 24, a2);
  return make_float2(acc.x + a2.x, acc.y + a2.y);
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
// Shared-memory layout of x' in the fused kernel.  A lane reads the whole
// uint4 chunk of columns it works on (32 columns for 4-bit, 64 for 2-bit) as
// float4 pieces; stored linearly, the 32 lanes of a warp would hit the same
// banks (chunks are 128 or 256 bytes apart).  Piece i of chunk ch is stored
// at position i ^ (ch & 7), so lanes ch..ch+7 reading piece i touch eight
// different 16-byte bank groups.
QE_DEV int swz_q4(int c) {
  const int ch = c >> 5;
  return (ch << 5) | ((((c >> 2) & 7) ^ (ch & 7)) << 2) | (c & 3);
}
QE_DEV int swz_q2(int c) {
  const int ch = c >> 6;
  return (ch << 6) | ((((c >> 2) & 15) ^ (ch & 7)) << 2) | (c & 3);
}

// The 32 x' values of columns [32*lc, 32*lc+32) from a swizzled buffer, as
// 16 float2 (4-bit form: whole chunk lc; 2-bit form: half lc&1 of chunk lc/2).
QE_DEV void load_xs32_q4(const float* xp, int lc, float2 (&xs)[16]) {
  const float4* src = (const float4*)(xp + lc * 32);
  const int sw = lc & 7;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 v = src[i ^ sw];
    xs[2 * i] = make_float2(v.x, v.y);
    xs[2 * i + 1] = make_float2(v.z, v.w);
  }
}
QE_DEV void load_xs32_q2(const float* xp, int lc, float2 (&xs)[16]) {
  const int ch = lc >> 1, half = lc & 1;
  const float4* src = (const float4*)(xp + ch * 64);
  const int sw = ch & 7;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 v = src[(half * 8 + i) ^ sw];
    xs[2 * i] = make_float2(v.x, v.y);
    xs[2 * i + 1] = make_float2(v.z, v.w);
  }
}

// 2^(60+E): turns acc back into sum q*x.
QE_DEV float acc_scale(int E) { return __int_as_float((127 + 60 + E) << 23); }

}  // namespace qe
