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

// try_wait that may suspend the thread for up to `ns` nanoseconds while the
// phase is incomplete (it resumes as soon as the phase completes).
QE_DEV bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Each try
// suspends the thread in hardware (up to 10 us, resuming as soon as the
// phase completes), so waiting warps take no issue slots from working ones.
QE_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t deadline, volatile int* abort_flag) {
  while (!mbar_try_wait_sleep(bar, parity, 10000u)) {
    if (*abort_flag || gtimer() > deadline) return false;
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
QE_DEV void cp_async8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
QE_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until every cp.async this thread has issued has landed (committed or not).
QE_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Arrive on an mbarrier once every cp.async this thread has issued so far
// has landed (the arrival is counted now and completed then, so the
// barrier's expected count is unchanged).
QE_DEV void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// The same arrival counted against the barrier's expected count (its init
// count must include it).
QE_DEV void cp_async_mbar_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
template <int N>
QE_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
// Programmatic dependent launch: wait until the kernels this one depends on
// have finished and their memory is visible (returns at once when the
// launch had no such dependency), and let the next kernel of the stream
// start its own prologue.
QE_DEV void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
QE_DEV void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
QE_DEV void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p)); }
QE_DEV void prefetch_l1(const void* p) { asm volatile("prefetch.global.L1 [%0];" ::"l"(p)); }

// 1-D bulk copy (TMA engine) of `bytes` (a multiple of 16; both addresses
// 16-byte aligned) from global to this CTA's shared memory; its completion
// counts `bytes` against the transaction count of mbarrier `bar`.  No
// multicast: the copy lands in the issuing CTA only.
QE_DEV void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

// Arrive on `bar` and raise its expected transaction count by `bytes`.
QE_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Tagged records: an aligned 64-bit word {32-bit value, 32-bit tag of the
// launch that wrote it}.  A reader that sees the tag it expects in a word
// also sees that launch's value in it (single-copy atomicity of an aligned
// 64-bit access), so records need no fence or flag; a 16-byte access moves
// two of them (each word still atomic on its own).
QE_DEV unsigned long long rec_word(uint32_t value, uint32_t tag) { return ((unsigned long long)tag << 32) | value; }
QE_DEV uint32_t rec_tag(unsigned long long w) { return (uint32_t)(w >> 32); }
QE_DEV uint32_t rec_val(unsigned long long w) { return (uint32_t)w; }
QE_DEV void st_rec(unsigned long long* p, unsigned long long w) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
QE_DEV unsigned long long ld_rec(const unsigned long long* p) {
  unsigned long long w;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return w;
}
QE_DEV void st_rec2(unsigned long long* p, unsigned long long a, unsigned long long b) {
  asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(p), "l"(a), "l"(b) : "memory");
}
QE_DEV void ld_rec2(const unsigned long long* p, unsigned long long& a, unsigned long long& b) {
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}

QE_DEV unsigned ld_relaxed_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
QE_DEV void st_relaxed_u32(unsigned* p, unsigned v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Named barrier over `count` threads (non-aligned form: counts threads).
QE_DEV void named_barrier(int id, int count) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Arrive at named barrier `id` without waiting (a producer: its earlier
// memory accesses are ordered before the waiters' later ones).
QE_DEV void named_barrier_arrive(int id, int count) {
  asm volatile("barrier.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
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

// Sum R per-lane values (float or double) over the warp at once (R a power
// of two <= 32).
// Stage o halves the live values: lanes with bit o set keep the upper half.
// Afterwards the total of value i sits in every lane whose bits
// (lane>>4, lane>>3, ...) spell i in binary (most significant first);
// reduced_row_of_lane() gives that index.
template <int R, typename T>
QE_DEV T warp_reduce_rows(T (&v)[R], int lane) {
  int live = R;
  int o = 16;
#pragma unroll
  for (; live > 1; o >>= 1) {
    const bool up = (lane & o) != 0;
    const int half = live / 2;
#pragma unroll
    for (int i = 0; i < R / 2; ++i) {
      if (i < half) {
        T keep = up ? v[i + half] : v[i];
        T send = up ? v[i] : v[i + half];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    live = half;
  }
  T s = v[0];
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

// ------------------------------------------------ integer dequant-dot cores
//
// The activation vector v is held as 22-bit fixed point under one power-of-
// two scale per vector: v_c = vi_c * 2^(e-22), |vi_c| < 2^22, where e is the
// least exponent with max|v| < 2^e (fixed_scale_exponent).  vi is split into
// three byte limbs, vi = b2 * 2^16 + b1 * 2^8 + b0 (b2 signed, b1 and b0
// unsigned).  A packed word of q fields is spread into bytes with masks (two
// LOP3 and a shift per eight 4-bit fields) and dp4a multiplies four q bytes
// with four limb bytes, accumulating exactly in int32.  Per 32-column chunk
// and row the three limb sums give
//   sum_c q_c vi_c = A2 * 2^16 + A1 * 2^8 + A0,
// and the group's affine term is then  s * 2^(e-22) * that + b * sum_c v_c.
// Everything before the final fp32 combination is exact integer arithmetic,
// and the fixed point keeps 22 bits below max|v|.  This costs 0.375 integer
// ops and 0.75 dp4a per weight, against one mask per weight for a float
// operand per q field.  Integers below 2^22 in magnitude move to and from
// fp32 by adding 1.5 * 2^23 (round to nearest, exact), so neither direction
// uses the slow conversion unit.
//
// Byte order of the limb words of one 32-column chunk:
//   4-bit: word r = 2w + h (w = packed word 0..3, h = 0 even fields, 1 odd
//          fields): byte i holds column 8w + 2i + h;
//   2-bit: word r = 4w + t (w = packed word 0..1, t = shift 0..3): byte i
//          holds column 16w + 4i + t.

struct XLimbs {
  int b2[8];       // signed high limbs
  unsigned b1[8];  // unsigned middle limbs
  unsigned b0[8];  // unsigned low limbs
};

QE_DEV int dp4a_us(unsigned a, int b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
QE_DEV int dp4a_uu(unsigned a, unsigned b, int c) {
  int d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
QE_DEV unsigned prmt(unsigned a, unsigned b, unsigned sel) {
  unsigned d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
constexpr int kMagicBits = 0x4B400000;
// Nearest integer of f, |f| < 2^22.
QE_DEV int round_small(float f) { return __float_as_int(f + kMagic) - kMagicBits; }
// i as a float, |i| < 2^22 (exact).
QE_DEV float small_to_float(int i) { return __int_as_float(i + kMagicBits) - kMagic; }

// Least e with max|v| < 2^e (amax = max|v|), kept where both 2^(22-e) and
// 2^(e-22) are normal floats; 0 for an all-zero vector.
QE_DEV int fixed_scale_exponent(float amax) {
  if (!(amax > 0.0f)) return 0;
  const int e = ((int)((__float_as_uint(amax) >> 23) & 0xFF)) - 127 + 1;
  return e < -100 ? -100 : (e > 120 ? 120 : e);
}
QE_DEV float pow2f(int k) { return __int_as_float((127 + k) << 23); }  // 2^k, |k| <= 126

// The limbs of one 32-column chunk under exponent e; also returns the sum of
// the 32 raw values (column order).  src is the chunk's 32 floats in shared
// memory with its eight 16-byte pieces swizzled (piece i at i ^ sw, sw = the
// chunk's index & 7, as xswz lays them out), so the lanes of a warp reading
// consecutive chunks spread over all banks.
template <int BITS>
QE_DEV float build_limbs(const float* src, int sw, int e, XLimbs& x) {
  const float in = pow2f(22 - e);
  int vi[32];
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 f = ((const float4*)src)[i ^ sw];
    sum += f.x; sum += f.y; sum += f.z; sum += f.w;
    vi[4 * i] = round_small(f.x * in);
    vi[4 * i + 1] = round_small(f.y * in);
    vi[4 * i + 2] = round_small(f.z * in);
    vi[4 * i + 3] = round_small(f.w * in);
  }
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    unsigned v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      v[i] = (unsigned)vi[BITS == 4 ? 8 * (r >> 1) + 2 * i + (r & 1) : 16 * (r >> 2) + 4 * i + (r & 3)];
    // byte k of v[0..3] into bytes 0..3 of limb word k
    const unsigned t01 = prmt(v[0], v[1], 0x5140u), t23 = prmt(v[2], v[3], 0x5140u);
    const unsigned s01 = prmt(v[0], v[1], 0x0062u), s23 = prmt(v[2], v[3], 0x0062u);
    x.b0[r] = prmt(t01, t23, 0x5410u);
    x.b1[r] = prmt(t01, t23, 0x7632u);
    x.b2[r] = (int)prmt(s01, s23, 0x5410u);
  }
  return sum;
}

// The limbs of one 32-column chunk held in registers (v[c] = column c) under
// exponent e.
template <int BITS>
QE_DEV void build_limbs_reg(const float (&v)[32], int e, XLimbs& x) {
  const float in = pow2f(22 - e);
  int vi[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) vi[c] = round_small(v[c] * in);
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    unsigned w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w[i] = (unsigned)vi[BITS == 4 ? 8 * (r >> 1) + 2 * i + (r & 1) : 16 * (r >> 2) + 4 * i + (r & 3)];
    const unsigned t01 = prmt(w[0], w[1], 0x5140u), t23 = prmt(w[2], w[3], 0x5140u);
    const unsigned s01 = prmt(w[0], w[1], 0x0062u), s23 = prmt(w[2], w[3], 0x0062u);
    x.b0[r] = prmt(t01, t23, 0x5410u);
    x.b1[r] = prmt(t01, t23, 0x7632u);
    x.b2[r] = (int)prmt(s01, s23, 0x5410u);
  }
}

QE_DEV float limb_sum(int a2, int a1, int a0) {
  return fmaf(small_to_float(a2), 65536.0f, fmaf(small_to_float(a1), 256.0f, small_to_float(a0)));
}

// sum_c q_c vi_c of one 32-column chunk of 4-bit weights (words 0..3).
QE_DEV float idot32_q4(const uint4 w, const XLimbs& x) {
  int a2 = 0, a1 = 0, a0 = 0;
  const unsigned ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const unsigned lo = ws[j] & 0x0F0F0F0Fu, hi = (ws[j] >> 4) & 0x0F0F0F0Fu;
    a2 = dp4a_us(lo, x.b2[2 * j], a2);
    a1 = dp4a_uu(lo, x.b1[2 * j], a1);
    a0 = dp4a_uu(lo, x.b0[2 * j], a0);
    a2 = dp4a_us(hi, x.b2[2 * j + 1], a2);
    a1 = dp4a_uu(hi, x.b1[2 * j + 1], a1);
    a0 = dp4a_uu(hi, x.b0[2 * j + 1], a0);
  }
  return limb_sum(a2, a1, a0);
}

// Same for 2-bit weights (words 0..1).
QE_DEV float idot32_q2(const uint2 w, const XLimbs& x) {
  int a2 = 0, a1 = 0, a0 = 0;
  const unsigned ws[2] = {w.x, w.y};
#pragma unroll
  for (int j = 0; j < 2; ++j) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const unsigned q = (ws[j] >> (2 * t)) & 0x03030303u;
      a2 = dp4a_us(q, x.b2[4 * j + t], a2);
      a1 = dp4a_uu(q, x.b1[4 * j + t], a1);
      a0 = dp4a_uu(q, x.b0[4 * j + t], a0);
    }
  }
  return limb_sum(a2, a1, a0);
}

template <int BITS>
QE_DEV float idot32(const unsigned char* w, const XLimbs& x) {
  if (BITS == 4) return idot32_q4(*(const uint4*)w, x);
  return idot32_q2(*(const uint2*)w, x);
}

}  // namespace qe
