// qe_device.cuh -- device building blocks of the sm_100a kernels:
// bf16 decode, bounded waits, mbarrier and asynchronous-copy wrappers and the
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
QE_DEV unsigned long long atom_add_release_u64(unsigned long long* p, unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.release.gpu.global.add.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}

QE_DEV unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait until a 64-bit counter reaches target; false if the deadline
// passed or the CTA's abort flag was raised.
QE_DEV bool wait_geq64(const unsigned long long* ctr, unsigned long long target, uint64_t deadline,
                       volatile int* abort_flag) {
  unsigned spins = 0;
  while (ld_acquire_u64(ctr) < target) {
    if (*abort_flag) return false;
    if ((++spins & 15u) == 0 && gtimer() > deadline) return false;
  }
  return true;
}

QE_DEV bool wait_geq(const unsigned* ctr, unsigned target, uint64_t deadline,
                     volatile int* abort_flag) {
  unsigned spins = 0;
  while (ld_acquire(ctr) < target) {
    if (*abort_flag) return false;
    if ((++spins & 15u) == 0 && gtimer() > deadline) return false;
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

// ---------------------------------------------------- asynchronous copies

// L2 policy: streamed expert weights are read once per token, so they are
// marked evict-first and do not push the router or activations out of L2.
QE_DEV uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 16-byte asynchronous global -> shared copy (LDGSTS), L2 evict-first.
QE_DEV void cp_async16(void* dst, const void* src, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "l"(pol)
               : "memory");
}

// 8- and 4-byte asynchronous copies (cached form; dst and src aligned to the size).
QE_DEV void cp_async8(void* dst, const void* src, uint64_t pol) {
  asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], 8, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "l"(pol)
               : "memory");
}
QE_DEV void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
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

// Same as warp_reduce_rows with max instead of sum.
template <int R>
QE_DEV float warp_reduce_rows_max(float (&v)[R], int lane) {
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
        v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, o));
      }
    }
    live = half;
  }
  float s = v[0];
  for (; o > 0; o >>= 1) s = fmaxf(s, __shfl_xor_sync(0xffffffffu, s, o));
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
// the single fp32 rounding of the fused multiply-add.  Per group the dot
// product is then
//   sum_c (q_c*s + b) x_c = s * 2^(60+E) * acc + b * sum_c x_c.
// Subnormal operands and results must not be flushed: never build these
// kernels with -ftz=true or --use_fast_math.
//
// Pair form.  Two adjacent packed words are one 64-bit value P (an aligned
// register pair), and one 64-bit AND with the field mask repeated in both
// halves yields the same field of both words: a ready operand pair of one
// packed f32x2 FMA, with no register moves.  Fields that reach bit 23 or
// above are taken from P >> 12, where they sit at bits 8..19 (a 64-bit
// shift: the bits the high word pushes into the low half land at bit 20 and
// above, where no mask of the shifted value looks).  The x'
// of a 32-column chunk is therefore stored in pair order: pair k holds the
// columns of field k of both words of a word pair (see xperm_q4 / xperm_q2).

// Field offset p of field j (0..7) of a 4-bit word after the mapping above.
QE_DEV int q4_field_pos(int j) { return j < 5 ? 4 * j : 4 * j - 12; }
// Field offset p of field j (0..15) of a 2-bit word.
QE_DEV int q2_field_pos(int j) { return j < 11 ? 2 * j : 2 * j - 12; }

QE_DEV float f_of(uint32_t u) { return __uint_as_float(u); }

QE_DEV float2 f2_of(unsigned long long v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}

// acc += (P & M) * x as one packed FMA (P: two words, M: the mask in both halves).
#define QE_QFMA2(acc, P, M, x) (acc) = __ffma2_rn(f2_of((P) & (M)), (x), (acc))

QE_DEV constexpr unsigned long long rep2(unsigned m) { return ((unsigned long long)m << 32) | m; }

// One 32-column chunk of 4-bit weights (words 0..3 as two 64-bit pairs)
// against its 16 x' pairs; pair 8h + j holds columns 16h + j and 16h + 8 + j.
// Two accumulators so consecutive FMAs do not wait on each other.
QE_DEV float2 dot32_q4(const ulonglong2 w, const float2* xs, float2 acc) {
  float2 a2 = make_float2(0.f, 0.f);
  const unsigned long long s0 = w.x >> 12, s1 = w.y >> 12;
  QE_QFMA2(acc, w.x, rep2(0xFu), xs[0]);
  QE_QFMA2(a2, w.y, rep2(0xFu), xs[8]);
  QE_QFMA2(acc, w.x, rep2(0xF0u), xs[1]);
  QE_QFMA2(a2, w.y, rep2(0xF0u), xs[9]);
  QE_QFMA2(acc, w.x, rep2(0xF00u), xs[2]);
  QE_QFMA2(a2, w.y, rep2(0xF00u), xs[10]);
  QE_QFMA2(acc, w.x, rep2(0xF000u), xs[3]);
  QE_QFMA2(a2, w.y, rep2(0xF000u), xs[11]);
  QE_QFMA2(acc, w.x, rep2(0xF0000u), xs[4]);
  QE_QFMA2(a2, w.y, rep2(0xF0000u), xs[12]);
  QE_QFMA2(acc, s0, rep2(0xF00u), xs[5]);
  QE_QFMA2(a2, s1, rep2(0xF00u), xs[13]);
  QE_QFMA2(acc, s0, rep2(0xF000u), xs[6]);
  QE_QFMA2(a2, s1, rep2(0xF000u), xs[14]);
  QE_QFMA2(acc, s0, rep2(0xF0000u), xs[7]);
  QE_QFMA2(a2, s1, rep2(0xF0000u), xs[15]);
  return make_float2(acc.x + a2.x, acc.y + a2.y);
}

// One 32-column chunk of 2-bit weights (two words as one 64-bit pair)
// against its 16 x' pairs; pair j holds columns j and 16 + j.
QE_DEV float2 dot32_q2(const unsigned long long w, const float2* xs, float2 acc) {
  float2 a2 = make_float2(0.f, 0.f);
  const unsigned long long s = w >> 12;
  QE_QFMA2(acc, w, rep2(0x3u), xs[0]);
  QE_QFMA2(a2, w, rep2(0xCu), xs[1]);
  QE_QFMA2(acc, w, rep2(0x30u), xs[2]);
  QE_QFMA2(a2, w, rep2(0xC0u), xs[3]);
  QE_QFMA2(acc, w, rep2(0x300u), xs[4]);
  QE_QFMA2(a2, w, rep2(0xC00u), xs[5]);
  QE_QFMA2(acc, w, rep2(0x3000u), xs[6]);
  QE_QFMA2(a2, w, rep2(0xC000u), xs[7]);
  QE_QFMA2(acc, w, rep2(0x30000u), xs[8]);
  QE_QFMA2(a2, w, rep2(0xC0000u), xs[9]);
  QE_QFMA2(acc, w, rep2(0x300000u), xs[10]);
  QE_QFMA2(a2, s, rep2(0xC00u), xs[11]);
  QE_QFMA2(acc, s, rep2(0x3000u), xs[12]);
  QE_QFMA2(a2, s, rep2(0xC000u), xs[13]);
  QE_QFMA2(acc, s, rep2(0x30000u), xs[14]);
  QE_QFMA2(a2, s, rep2(0xC0000u), xs[15]);
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

// x' of column c for 4-bit / 2-bit matrices (c's field is c mod 8 / 16).
QE_DEV float xprime_q4(float x, int c, int E) {
  return x * __int_as_float((127 + 89 - q4_field_pos(c & 7) - E) << 23);
}
QE_DEV float xprime_q2(float x, int c, int E) {
  return x * __int_as_float((127 + 89 - q2_field_pos(c & 15) - E) << 23);
}

// Position of column c in the pair order of its 32-column chunk.
// 4-bit: column 16h + 8e + j -> 2(8h + j) + e; 2-bit: column 16e + j -> 2j + e.
QE_DEV int xperm_q4(int c) {
  const int m = c & 31;
  return (c & ~31) | ((m >> 4) << 4) | ((m & 7) << 1) | ((m >> 3) & 1);
}
QE_DEV int xperm_q2(int c) {
  const int m = c & 31;
  return (c & ~31) | ((m & 15) << 1) | (m >> 4);
}

// Shared-memory copies of x' also swizzle the eight 16-byte pieces of a
// chunk: piece i of chunk ch sits at i ^ (ch & 7), so lanes reading piece i
// of consecutive chunks touch eight different bank groups.  Global copies
// keep the pair order unswizzled; a float4 piece moves as a whole.
QE_DEV int xswz(int pos) {
  const int ch = pos >> 5;
  return (ch << 5) | ((((pos >> 2) & 7) ^ (ch & 7)) << 2) | (pos & 3);
}
QE_DEV int swz_q4(int c) { return xswz(xperm_q4(c)); }
QE_DEV int swz_q2(int c) { return xswz(xperm_q2(c)); }

// The 16 x' pairs of 32-column chunk lc from a swizzled buffer (either form).
QE_DEV void load_xs32(const float* xp, int lc, float2 (&xs)[16]) {
  const float4* src = (const float4*)(xp + lc * 32);
  const int sw = lc & 7;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 v = src[i ^ sw];
    xs[2 * i] = make_float2(v.x, v.y);
    xs[2 * i + 1] = make_float2(v.z, v.w);
  }
}
QE_DEV void load_xs32_q4(const float* xp, int lc, float2 (&xs)[16]) { load_xs32(xp, lc, xs); }
QE_DEV void load_xs32_q2(const float* xp, int lc, float2 (&xs)[16]) { load_xs32(xp, lc, xs); }

// 2^(60+E): turns acc back into sum q*x.
QE_DEV float acc_scale(int E) { return __int_as_float((127 + 60 + E) << 23); }

}  // namespace qe
