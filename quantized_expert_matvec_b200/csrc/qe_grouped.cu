// qe_grouped.cu -- batched layer step (T tokens per step): the (token, k)
// assignments are grouped by expert so each selected expert's weights are
// streamed from HBM once per token pass and reused by all of its tokens.
//
//   group kernel  : counting sort of the T*K assignments by expert (stable:
//                   ascending assignment id inside an expert); active experts
//                   ordered by descending token count
//   gate/up kernel: persistent CTAs take items (expert, kRowsA rows of gate
//                   and of up) from a shared counter; an item is cut into
//                   segments of at most kTile tokens.  The CTA stages the x'
//                   of the segment's tokens in shared memory; each warp takes
//                   units of two output rows (two gate rows and the two up
//                   rows: four matrix rows) and each lane a 32-column chunk
//                   of them per step.  A packed word pair is masked once and
//                   multiplied into the accumulators of every token, and each
//                   x' piece read from shared memory serves the four rows.
//                   h = silu(g) u and the running max |h| per assignment go
//                   to global memory.
//   down kernel   : the same over items (expert, kRowsB rows of down), units
//                   of four rows, with h of the segment's tokens staged in
//                   x' form -> y[assignment][H]
//   combine       : out[t] = sum_k w[t,k] y[t*K+k] (+ x[t])
//
// Each warp streams its packed words through a ring of kSlots steps in shared
// memory, filled by asynchronous copies with one commit group per step: the
// slot of a step is refilled with the step kSlots ahead as soon as it has
// been used, and at the end of a segment the refills already fetch the next
// segment's first steps, so the loads run across the staging of the next
// segment's activations.  With the loads hidden, the kernels are bound by
// instruction issue (one mask per weight, one multiply-add per weight and
// token), not by the bytes they stream.
#include <math.h>

#include "qe_device.cuh"

namespace qe {

constexpr int kGWarps = 16;
constexpr int kGThreads = kGWarps * 32;
constexpr int kTile = 4;     // tokens sharing one pass over the weights
constexpr int kRowsA = 256;  // gate/up rows (of gate and of up) per item
constexpr int kRowsB = 1024; // down rows per item
constexpr int kSlots = 3;    // steps of packed words in flight per warp
constexpr bool kTcEnabled = false;  // see launch_grouped

// Round a count of 4-byte elements up to a multiple of 4 (16 bytes).
static __host__ __device__ __forceinline__ int al4(int n) { return (n + 3) & ~3; }

// -------------------------------------------------------------- grouping
// One CTA of 1024 threads (E <= 1024).  Also zeroes the per-assignment |h|
// maxima and the two work counters of the expert kernels.
__global__ void __launch_bounds__(1024) group_kernel(const int32_t* __restrict__ idx, int A, int E, int* count,
                                                     int* start, int* list, int* order, int* ctl,
                                                     unsigned* hamax, int tc_min, int* err) {
  __shared__ int cnt[kMaxE];
  __shared__ int cur[kMaxE];
  __shared__ int wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
  for (int a = tid; a < A; a += blockDim.x) hamax[a] = 0u;
  // [0] active experts, [1] gate/up work, [2] down work, [3] experts with at
  // least tc_min tokens (tensor-core gate/up; they lead `order`), [4] its work
  if (tid < 8) ctl[tid] = 0;
  __syncthreads();
  for (int a = tid; a < A; a += blockDim.x) {
    const int e = idx[a];
    if (e < 0 || e >= E) { set_error(err, QE_ERR_INVALID_ARG); continue; }
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  // exclusive scan of the counts (thread e holds expert e)
  const int c = tid < E ? cnt[tid] : 0;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    wsum[lane] = v;  // inclusive over warps
  }
  __syncthreads();
  const int excl = incl - c + (warp > 0 ? wsum[warp - 1] : 0);
  if (tid < E) {
    start[tid] = excl;
    cur[tid] = excl;
    count[tid] = c;
    if (c > 0) {
      // rank among active experts: more tokens first, then lower index
      int rank = 0;
      for (int f = 0; f < E; ++f) {
        const int cf = cnt[f];
        rank += (cf > c) || (cf == c && f < tid);
      }
      order[rank] = tid;
      atomicAdd(&ctl[0], 1);
      if (tc_min > 0 && c >= tc_min) atomicAdd(&ctl[3], 1);
    }
  }
  if (tid == 0) start[E] = wsum[31];
  __syncthreads();
  for (int a = tid; a < A; a += blockDim.x) {
    const int e = idx[a];
    if (e < 0 || e >= E) continue;
    list[atomicAdd(&cur[e], 1)] = a;
  }
  __syncthreads();
  // ascending assignment order inside each expert (lists are short)
  if (tid < E) {
    int* l = list + excl;
    for (int i = 1; i < c; ++i) {
      const int v = l[i];
      int j = i - 1;
      while (j >= 0 && l[j] > v) { l[j + 1] = l[j]; --j; }
      l[j + 1] = v;
    }
  }
}

struct GroupedKParams {
  int H, I, K, T;
  int tile;           // tokens per pass of this kernel (1, 2 or 4)
  const qe_expert* experts;
  const float* xp4;   // [T][H] x' (pair order, unswizzled)
  const float* xp2;
  const float* xsum;  // [T][H/32]
  const int* xexp;    // [T]
  const int* count;
  const int* start;
  const int* list;
  const int* order;
  int* ctl;           // [0] active experts, [1] gate/up work, [2] down work, [3] tensor-core experts
  float* h;           // [T*K][I]
  unsigned* hamax;    // [T*K]
  float* y;           // [T*K][H]
  int* err;
};

// Packed words and scales/biases are copied with 16-, 8- and 4-byte
// asynchronous copies, so every pointer of a descriptor must be 16-byte
// aligned (the library's documented contract).
static __device__ __forceinline__ bool qmat_ok(const qe_qmat& m, int bits) {
  return m.bits == bits && m.wq && m.scales && m.biases && ((uintptr_t)m.wq & 15) == 0 &&
         ((uintptr_t)m.scales & 15) == 0 && ((uintptr_t)m.biases & 15) == 0;
}

// One segment of an item: rows [r0, r0 + nrows) of expert e against tokens
// [t0, t0 + nt) of the expert's assignment list.  m0/m1 are gate/up for the
// gate/up kernel, m0 is down for the down kernel.
struct GSeg {
  int valid, e, bits, r0, nrows, t0, nt;
  qe_qmat m0, m1;
};

// Per-warp ring of kSlots steps in shared memory.  A step is, for each lane,
// the packed 32-column chunk of four matrix rows (16 bytes each; 8 at 2-bit,
// layout [slot][row][lane], each lane reads what it copied) and the bf16
// scales and biases of the step's groups.  When a row holds a multiple of 8
// groups the scale/bias runs are 16-byte aligned and lanes 0..15 copy the
// step's 16 groups of each row and array in one 16-byte copy each (layout
// [slot][row][scale|bias][16 entries]); otherwise every lane copies the
// 4-byte word holding its own group's entry ([slot][row][scale|bias][lane]).
constexpr int kRingWords = kSlots * 4 * 32 * 16;
constexpr int kRingSb = kSlots * 4 * 2 * 32 * 4;
constexpr int kRingWarp = kRingWords + kRingSb;  // 9 KiB

// Staged x' vectors keep each 32-column chunk in pair order and pad it to
// 36 floats: lane L's chunk then starts 36 L floats in, so the eight
// 16-byte pieces of a chunk are read at fixed offsets from one address and
// the lanes of a quarter warp fall on distinct bank groups.
constexpr int kXPad = 36;
static __host__ __device__ __forceinline__ int xs_stride(int C) { return (C / 32) * kXPad; }

// Token-pass width for nt live tokens: 1, 2 or 4.
static __host__ __device__ __forceinline__ int nt_pad(int nt) { return nt <= 1 ? 1 : (nt <= 2 ? 2 : 4); }

// Units of four matrix rows in a segment: gate/up takes output rows in pairs
// (gate and up of each), down takes four rows.
template <int MODE>
static __device__ __forceinline__ int seg_units(const GSeg& s) { return MODE == 0 ? s.nrows / 2 : s.nrows / 4; }

// Steps of warp `warp` in segment s: its units warp, warp + kGWarps, ...
// times cpl chunks per lane and row.
template <int MODE>
static __device__ __forceinline__ int seg_steps(const GSeg& s, int warp, int cpl) {
  const int u = seg_units<MODE>(s);
  return u > warp ? ((u - warp + kGWarps - 1) / kGWarps) * cpl : 0;
}

// Row of matrix row m (0..3) of unit q.
template <int MODE>
static __device__ __forceinline__ int unit_row(const GSeg& s, int q, int m) {
  return MODE == 0 ? s.r0 + 2 * q + (m & 1) : s.r0 + 4 * q + m;
}

// Issue the copies of step (k, c) of this warp in segment s -- chunk c of
// the lanes in the warp's k-th unit -- into ring slot (rw, rsb) (C = columns
// of the matrices; lanes past the last chunk copy nothing).  The caller
// commits the group.
template <int MODE>
static __device__ __forceinline__ void issue_step(const GSeg& s, int C, int k, int c, int warp, int lane,
                                                  unsigned char* rw, uint32_t* rsb, bool coop, uint64_t pol) {
  const int q = warp + kGWarps * k;
  const int lc = 32 * c + lane;
  const int bits = s.bits;
  const size_t rowb = (size_t)C * bits / 8;
  const int gpr = C / kGroup;
#pragma unroll
  for (int m = 0; m < 4 && lc < C / 32; ++m) {
    const qe_qmat& mat = (MODE == 0 && m >= 2) ? s.m1 : s.m0;
    const int row = unit_row<MODE>(s, q, m);
    const unsigned char* rp = (const unsigned char*)mat.wq + (size_t)row * rowb;
    if (bits == 4) cp_async16(rw + (m * 32 + lane) * 16, rp + (size_t)lc * 16, pol);
    else cp_async8(rw + (m * 32 + lane) * 16, rp + (size_t)lc * 8, pol);
    if (!coop) {
      // the 4-byte word holding group gi's entry (gi rounded down to even;
      // the arrays hold an even number of entries, so the word is in bounds)
      const size_t gi2 = ((size_t)row * gpr + (lc >> 1)) & ~(size_t)1;
      cp_async4(rsb + (m * 2 + 0) * 32 + lane, mat.scales + gi2);
      cp_async4(rsb + (m * 2 + 1) * 32 + lane, mat.biases + gi2);
    }
  }
  if (coop && lane < 16) {
    // piece lane = (row m, array a, half h): groups 16c + 8h .. +7 of row m
    const int m = lane >> 2, a = (lane >> 1) & 1, h = lane & 1;
    const int g0 = 16 * c + 8 * h;
    if (g0 < gpr) {
      const qe_qmat& mat = (MODE == 0 && m >= 2) ? s.m1 : s.m0;
      const uint16_t* src = (a ? mat.biases : mat.scales) + (size_t)unit_row<MODE>(s, q, m) * gpr + g0;
      cp_async16((unsigned char*)rsb + (m * 2 + a) * 32 + h * 16, src, pol);
    }
  }
}

// Field f of both words of a word pair P (S = P >> 12), as the float pair
// fed to the multiply-add: fields that reach bit 23 come from S, so no field
// touches the exponent bits.
template <int BITS>
static __device__ __forceinline__ float2 field_pair(unsigned long long P, unsigned long long S, int f) {
  if (BITS == 4) return f2_of(f < 5 ? (P & rep2(0xFu << (4 * f))) : (S & rep2(0xFu << (4 * f - 12))));
  return f2_of(f < 11 ? (P & rep2(3u << (2 * f))) : (S & rep2(3u << (2 * f - 12))));
}

// Piece i (0..7) of a chunk: x' pairs 2i and 2i+1.  4-bit: fields 2(i&3),
// 2(i&3)+1 of word pair i>>2; 2-bit: fields 2i, 2i+1 of the one word pair.
template <int BITS>
static __device__ __forceinline__ void piece_masks(const ulonglong2 w, int i, float2& m0, float2& m1) {
  const unsigned long long P = (BITS == 4 && i >= 4) ? w.y : w.x, S = P >> 12;
  const int f = BITS == 4 ? 2 * (i & 3) : 2 * i;
  m0 = field_pair<BITS>(P, S, f);
  m1 = field_pair<BITS>(P, S, f + 1);
}

// One step: chunk lc of the four matrix rows in ring slot (rw, rsb) against
// the NT staged token vectors (x' padded, [NT][xs_stride(C)]); v[m*NT + t]
// gets row m, token t.  par[m] = parity of the chunk's group index in row m
// (which half of the copied 4-byte scale/bias word is the chunk's; per-lane
// copies only).
template <int BITS, int NT>
static __device__ __forceinline__ void compute_step(const unsigned char* rw, const uint32_t* rsb, const int (&par)[4],
                                                    bool coop, const float* xs, const float* sums, const float* xk,
                                                    int C, int lc, int lane, float (&v)[4 * NT]) {
  const int nch = C / 32;
  if (lc >= nch) return;
  ulonglong2 w[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const unsigned char* src = rw + (m * 32 + lane) * 16;
    if (BITS == 4) {
      w[m] = *(const ulonglong2*)src;
    } else {
      w[m].x = *(const unsigned long long*)src;
      w[m].y = 0ull;
    }
  }
  float2 acc[4][NT];
#pragma unroll
  for (int m = 0; m < 4; ++m)
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[m][t] = make_float2(0.f, 0.f);
  const float4* xb = (const float4*)(xs + lc * kXPad);
  const int ts = xs_stride(C) / 4;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float4 xp[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) xp[t] = xb[t * ts + i];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      float2 m0, m1;
      piece_masks<BITS>(w[m], i, m0, m1);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        acc[m][t] = __ffma2_rn(m0, make_float2(xp[t].x, xp[t].y), acc[m][t]);
        acc[m][t] = __ffma2_rn(m1, make_float2(xp[t].z, xp[t].w), acc[m][t]);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    float sc, bi;
    if (coop) {
      const uint16_t* e = (const uint16_t*)rsb + (m * 2) * 16 + ((lc >> 1) & 15);
      sc = __uint_as_float((uint32_t)e[0] << 16);
      bi = __uint_as_float((uint32_t)e[16] << 16);
    } else {
      const uint32_t sw2 = rsb[(m * 2 + 0) * 32 + lane], bw2 = rsb[(m * 2 + 1) * 32 + lane];
      sc = __uint_as_float(par[m] ? (sw2 & 0xFFFF0000u) : (sw2 << 16));
      bi = __uint_as_float(par[m] ? (bw2 & 0xFFFF0000u) : (bw2 << 16));
    }
#pragma unroll
    for (int t = 0; t < NT; ++t)
      v[m * NT + t] += sc * xk[t] * (acc[m][t].x + acc[m][t].y) + bi * sums[t * nch + lc];
  }
}

// End of unit q: reduce v over the warp and write the unit's results.
// Gate/up: h = silu(g) u for output rows 2q, 2q+1, and |h| into the
// segment's maxima; down: y of rows 4q..4q+3.
template <int MODE, int NT>
static __device__ __forceinline__ void unit_epilogue(const GroupedKParams& p, const GSeg& s, const int* asg, int q,
                                                     float (&v)[4 * NT], unsigned* hmax, int lane) {
  const float sv = warp_reduce_rows<4 * NT>(v, lane);
  const int ri = reduced_row_of_lane<4 * NT>(lane);  // m * NT + t
  const int m = ri / NT, t = ri - m * NT;
  const bool first = lane == lane_of_reduced_row<4 * NT>(ri);
  if (MODE == 0) {
    // lanes holding g of (row, token) fetch u of the same pair
    const float uv = __shfl_sync(0xffffffffu, sv, lane_of_reduced_row<4 * NT>(m < 2 ? ri + 2 * NT : ri));
    if (m < 2 && t < s.nt && first) {
      const float hv = sv / (1.0f + expf(-sv)) * uv;
      p.h[(size_t)asg[t] * p.I + unit_row<0>(s, q, m)] = hv;
      atomicMax(&hmax[t], __float_as_uint(fabsf(hv)));
    }
  } else {
    if (t < s.nt && first) p.y[(size_t)asg[t] * p.H + unit_row<1>(s, q, m)] = sv;
  }
}

// All steps of this warp in segment S.  Before step l the warp waits until
// at most kSlots-1 copy groups are pending (step l's group is complete);
// after it the slot is refilled with step l + kSlots and one group is
// committed (empty if there is nothing to copy), so the groups stay in step
// order.  Past the end of S the refills fetch the next segment N, whose
// steps start at the next multiple of kSlots.  Steps run through (unit k,
// chunk c) with counters, the computed step and the refilled one apart.
template <int MODE, int BITS, int NT>
static __device__ __forceinline__ void run_segment(const GroupedKParams& p, const GSeg& Ssm, const GSeg& N,
                                                   const int* asg, int C, int cpl, const float* xs,
                                                   const float* sums, const float* xk, unsigned* hmax,
                                                   unsigned char* ring, int warp, int lane, uint64_t pol) {
  const GSeg S = Ssm;  // the segment's fields in registers
  const int nst = seg_steps<MODE>(S, warp, cpl);
  const int nstp = (nst + kSlots - 1) / kSlots * kSlots;
  const int nstN = N.valid ? seg_steps<MODE>(N, warp, cpl) : 0;
  const int gpr = C / kGroup;
  const bool coop = (gpr & 7) == 0;
  float v[4 * NT];
#pragma unroll
  for (int i = 0; i < 4 * NT; ++i) v[i] = 0.f;
  int kc = 0, cc = 0;                          // step being computed
  int ki = kSlots / cpl, ci = kSlots % cpl;    // step being refilled
  for (int l0 = 0; l0 < nstp; l0 += kSlots) {
#pragma unroll
    for (int j = 0; j < kSlots; ++j) {
      unsigned char* rw = ring + j * (4 * 32 * 16);
      uint32_t* rsb = (uint32_t*)(ring + kRingWords) + j * (4 * 2 * 32);
      const int l = l0 + j;
      cp_async_wait<kSlots - 1>();
      __syncwarp();  // the slot's shared scale/bias copies are visible to every lane
      if (l < nst) {
        const int q = warp + kGWarps * kc, lc = 32 * cc + lane;
        int par[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) par[m] = coop ? 0 : (unit_row<MODE>(S, q, m) * gpr + (lc >> 1)) & 1;
        compute_step<BITS, NT>(rw, rsb, par, coop, xs, sums, xk, C, lc, lane, v);
        if (cc == cpl - 1) {
          unit_epilogue<MODE, NT>(p, S, asg, q, v, hmax, lane);
#pragma unroll
          for (int i = 0; i < 4 * NT; ++i) v[i] = 0.f;
          cc = 0;
          ++kc;
        } else {
          ++cc;
        }
      }
      const int ln = l + kSlots;
      __syncwarp();  // every lane is done with the slot before it is refilled
      if (ln < nst) {
        issue_step<MODE>(S, C, ki, ci, warp, lane, rw, rsb, coop, pol);
        if (++ci == cpl) {
          ci = 0;
          ++ki;
        }
      } else if (ln >= nstp && ln - nstp < nstN) {
        const int lN = ln - nstp, kN = lN / cpl;
        issue_step<MODE>(N, C, kN, lN - kN * cpl, warp, lane, rw, rsb, coop, pol);
      }
      cp_async_commit();
    }
  }
  if (nstp == 0) {
    // no steps here: the slots take N's first steps (the groups of the
    // empty steps that were meant for S are complete)
#pragma unroll
    for (int j = 0; j < kSlots; ++j) {
      unsigned char* rw = ring + j * (4 * 32 * 16);
      uint32_t* rsb = (uint32_t*)(ring + kRingWords) + j * (4 * 2 * 32);
      if (j < nstN) issue_step<MODE>(N, C, j / cpl, j % cpl, warp, lane, rw, rsb, coop, pol);
      cp_async_commit();
    }
  }
}

// Thread 0: the segment after `prev` (the next token pass of the same item,
// else the first pass of the next item from the shared counter), with its
// assignments and tokens.
template <int MODE>
static __device__ void next_segment(const GroupedKParams& p, const GSeg& prev, GSeg& out, int* asg, int* toks) {
  int e = -1, t0 = 0;
  GSeg s = prev;
  if (prev.valid && prev.t0 + p.tile < p.count[prev.e]) {
    e = prev.e;
    t0 = prev.t0 + p.tile;
  } else {
    const int R = MODE == 0 ? p.I : p.H;
    const int rows = MODE == 0 ? kRowsA : kRowsB;
    const int ipe = (R + rows - 1) / rows;
    const int n_tc = MODE == 0 ? p.ctl[3] : 0;  // experts done by the tensor-core kernel
    const int n_items = (p.ctl[0] - n_tc) * ipe;
    for (;;) {
      const int item = atomicAdd(&p.ctl[MODE == 0 ? 1 : 2], 1);
      if (item >= n_items) {
        out.valid = 0;
        return;
      }
      e = p.order[n_tc + item / ipe];
      const qe_expert ex = p.experts[e];
      const int bits = MODE == 0 ? ex.gate.bits : ex.down.bits;
      const bool ok = (bits == 4 || bits == 2) &&
                      (MODE == 0 ? qmat_ok(ex.gate, bits) && qmat_ok(ex.up, bits) && qmat_ok(ex.down, bits)
                                 : qmat_ok(ex.down, bits));
      if (!ok) {
        set_error(p.err, QE_ERR_INVALID_ARG);
        continue;
      }
      s.bits = bits;
      s.r0 = (item % ipe) * rows;
      s.nrows = min(rows, R - s.r0);
      s.m0 = MODE == 0 ? ex.gate : ex.down;
      s.m1 = ex.up;
      break;
    }
  }
  s.valid = 1;
  s.e = e;
  s.t0 = t0;
  s.nt = min(p.tile, p.count[e] - t0);
  const int base = p.start[e] + t0;
  for (int t = 0; t < s.nt; ++t) {
    const int a = p.list[base + t];
    asg[t] = a;
    toks[t] = a / p.K;
  }
  out = s;
}

// Stage the segment's token vectors in x' form (swizzled), their 32-column
// sums and accumulator scales; padding tokens up to nt_pad(nt) are zero.
template <int MODE>
static __device__ void stage_segment(const GroupedKParams& p, const GSeg& s, const int* asg, const int* toks,
                                     float* xs, float* sums, float* xk, int* hexp) {
  const int ntp = nt_pad(s.nt), nt = s.nt;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (MODE == 0) {
    const int H = p.H;
    const float* src = s.bits == 4 ? p.xp4 : p.xp2;
    for (int i = tid; i < ntp * (H / 4); i += kGThreads) {
      const int t = i / (H / 4), c = (i - t * (H / 4)) * 4;
      const float4 v = t < nt ? *(const float4*)(src + (size_t)toks[t] * H + c) : make_float4(0.f, 0.f, 0.f, 0.f);
      *(float4*)(xs + t * xs_stride(H) + (c >> 5) * kXPad + (c & 31)) = v;  // pair order; pieces move whole
    }
    for (int i = tid; i < ntp * (H / 32); i += kGThreads) {
      const int t = i / (H / 32), c = i - t * (H / 32);
      sums[i] = t < nt ? p.xsum[(size_t)toks[t] * (H / 32) + c] : 0.f;
    }
    if (tid < ntp) xk[tid] = tid < nt ? acc_scale(p.xexp[toks[tid]]) : 0.f;
  } else {
    const int I = p.I;
    if (tid < ntp) {
      const int Eh = tid < nt ? xscale_exponent(__uint_as_float(__ldcg(&p.hamax[asg[tid]]))) : 0;
      hexp[tid] = Eh;
      xk[tid] = tid < nt ? acc_scale(Eh) : 0.f;
    }
    __syncthreads();
    for (int i = tid; i < ntp * I; i += kGThreads) {
      const int t = i / I, c = i - t * I;
      const float hv = t < nt ? __ldcg(p.h + (size_t)asg[t] * I + c) : 0.f;
      const int pos = s.bits == 4 ? xperm_q4(c) : xperm_q2(c);
      xs[t * xs_stride(I) + (pos >> 5) * kXPad + (pos & 31)] =
          s.bits == 4 ? xprime_q4(hv, c, hexp[t]) : xprime_q2(hv, c, hexp[t]);
    }
    for (int i = warp; i < ntp * (I / 32); i += kGWarps) {
      const int t = i / (I / 32), ch = i - t * (I / 32);
      const float sm = t < nt ? warp_sum(__ldcg(p.h + (size_t)asg[t] * I + ch * 32 + lane)) : 0.f;
      if (lane == 0) sums[i] = sm;
    }
  }
}

template <int MODE, int BITS>
static __device__ __forceinline__ void run_segment_nt(const GroupedKParams& p, const GSeg& S, const GSeg& N,
                                                      const int* asg, int C, int cpl, const float* xs,
                                                      const float* sums, const float* xk, unsigned* hmax,
                                                      unsigned char* ring, int warp, int lane, uint64_t pol) {
  const int ntp = nt_pad(S.nt);
  if (ntp == 1) run_segment<MODE, BITS, 1>(p, S, N, asg, C, cpl, xs, sums, xk, hmax, ring, warp, lane, pol);
  else if (ntp == 2) run_segment<MODE, BITS, 2>(p, S, N, asg, C, cpl, xs, sums, xk, hmax, ring, warp, lane, pol);
  else run_segment<MODE, BITS, 4>(p, S, N, asg, C, cpl, xs, sums, xk, hmax, ring, warp, lane, pol);
}

// Dynamic shared memory: the warps' rings, then x' of `tile` tokens, their
// 32-column sums and scales.
static __host__ __device__ __forceinline__ size_t expert_smem(int C, int tile) {
  return (size_t)kGWarps * kRingWarp + 4 * ((size_t)tile * xs_stride(C) + al4(tile * (C / 32)) + al4(tile));
}

// MODE 0: gate/up (C = H columns); MODE 1: down (C = I columns).
template <int MODE>
__global__ void __launch_bounds__(kGThreads, 1) grouped_expert_kernel(const GroupedKParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int C = MODE == 0 ? p.H : p.I;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* ring = smem + (size_t)warp * kRingWarp;
  float* xs = (float*)(smem + (size_t)kGWarps * kRingWarp);  // [tile][xs_stride(C)]
  float* sums = xs + p.tile * xs_stride(C);                    // [tile][C/32]
  float* xk = sums + al4(p.tile * (C / 32));                   // [tile]
  __shared__ GSeg s_seg[2];
  __shared__ int s_asg[2][kTile], s_tok[2][kTile], s_hexp[kTile];
  __shared__ unsigned s_hmax[2][kTile];
  const int cpl = (C / 32 + 31) / 32;  // chunks per lane and row
  const uint64_t pol = policy_evict_first();
  if (threadIdx.x == 0) {
    GSeg none;
    none.valid = 0;
    next_segment<MODE>(p, none, s_seg[0], s_asg[0], s_tok[0]);
    if (s_seg[0].valid) next_segment<MODE>(p, s_seg[0], s_seg[1], s_asg[1], s_tok[1]);
    else s_seg[1].valid = 0;
  }
  __syncthreads();
  {
    const int nst = s_seg[0].valid ? seg_steps<MODE>(s_seg[0], warp, cpl) : 0;
#pragma unroll
    for (int j = 0; j < kSlots; ++j) {
      if (j < nst)
        issue_step<MODE>(s_seg[0], C, j / cpl, j % cpl, warp, lane, ring + j * (4 * 32 * 16),
                         (uint32_t*)(ring + kRingWords) + j * (4 * 2 * 32), ((C / kGroup) & 7) == 0, pol);
      cp_async_commit();
    }
  }
  int cur = 0;
  while (s_seg[cur].valid) {
    const GSeg& S = s_seg[cur];
    const GSeg& N = s_seg[cur ^ 1];
    if (threadIdx.x < kTile) s_hmax[cur][threadIdx.x] = 0u;
    stage_segment<MODE>(p, S, s_asg[cur], s_tok[cur], xs, sums, xk, s_hexp);
    __syncthreads();
    if (S.bits == 4)
      run_segment_nt<MODE, 4>(p, S, N, s_asg[cur], C, cpl, xs, sums, xk, s_hmax[cur], ring, warp, lane, pol);
    else
      run_segment_nt<MODE, 2>(p, S, N, s_asg[cur], C, cpl, xs, sums, xk, s_hmax[cur], ring, warp, lane, pol);
    __syncthreads();
    if (threadIdx.x == 0) {
      if (MODE == 0)
        for (int t = 0; t < S.nt; ++t) atomicMax(&p.hamax[s_asg[cur][t]], s_hmax[cur][t]);
      // the buffer of S takes the segment after N
      if (N.valid) next_segment<MODE>(p, N, s_seg[cur], s_asg[cur], s_tok[cur]);
      else s_seg[cur].valid = 0;
    }
    cur ^= 1;
  }
  cp_async_wait<0>();
}

// Largest token pass (4, 2 or 1) whose shared memory fits.
static int expert_tile(int C, size_t avail) {
  for (int t = kTile; t >= 1; t >>= 1)
    if (expert_smem(C, t) <= avail) return t;
  return 0;
}

cudaError_t launch_grouped(const GroupedParams& gp, cudaStream_t s) {
  const int A = gp.T * gp.K;
  if (A == 0) return cudaSuccess;
  int* ctl = gp.grp_count + gp.E;  // the workspace reserves E + 8 ints
  // The tensor-core gate/up kernel (qe_tc.cu) is not launched: at hidden 4096
  // with 2-bit experts it stopped with an illegal instruction whose cause is
  // not found yet, so groups of every size take the CUDA-core path.
  const bool tc = kTcEnabled && tc_eligible(gp.H, gp.I) && gp.xh != nullptr;
  group_kernel<<<1, 1024, 0, s>>>(gp.idx, A, gp.E, gp.grp_count, gp.grp_start, gp.grp_list, gp.grp_order, ctl,
                                  gp.hamax, tc ? tc_min_tokens() : 0, gp.err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (tc && (e = launch_tc_gateup(gp, ctl, gp.budget_ns, s)) != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static int attr_dev = -1;
  static size_t avail = 0;
  if (attr_dev != dev) {
    int optin = 0;
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaFuncAttributes fa{}, fb{};
    if ((e = cudaFuncGetAttributes(&fa, grouped_expert_kernel<0>)) != cudaSuccess) return e;
    if ((e = cudaFuncGetAttributes(&fb, grouped_expert_kernel<1>)) != cudaSuccess) return e;
    const size_t st = fa.sharedSizeBytes > fb.sharedSizeBytes ? fa.sharedSizeBytes : fb.sharedSizeBytes;
    avail = (size_t)optin > st ? (size_t)optin - st : 0;
    if ((e = cudaFuncSetAttribute(grouped_expert_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)avail)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(grouped_expert_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)avail)) != cudaSuccess)
      return e;
    attr_dev = dev;
  }
  GroupedKParams p{};
  p.H = gp.H; p.I = gp.I; p.K = gp.K; p.T = gp.T;
  p.experts = gp.experts;
  p.xp4 = gp.xp4; p.xp2 = gp.xp2; p.xsum = gp.xsum; p.xexp = gp.xexp;
  p.count = gp.grp_count; p.start = gp.grp_start; p.list = gp.grp_list; p.order = gp.grp_order; p.ctl = ctl;
  p.h = gp.h; p.hamax = gp.hamax; p.y = gp.y; p.err = gp.err;
  const int ta = expert_tile(gp.H, avail), tb = expert_tile(gp.I, avail);
  if (ta == 0 || tb == 0) return cudaErrorInvalidConfiguration;
  p.tile = ta;
  grouped_expert_kernel<0><<<sms, kGThreads, expert_smem(gp.H, ta), s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  p.tile = tb;
  grouped_expert_kernel<1><<<sms, kGThreads, expert_smem(gp.I, tb), s>>>(p);
  return cudaGetLastError();
}

}  // namespace qe
