// qe_fused_plan.h -- where the single-token layer kernel puts its share of the
// selected experts in shared memory, and which bulk copies fill it.
//
// Host and device use the same functions: the kernel to issue its copies and
// to address what it reads, the library's plan probe (a host function the CPU
// tests call) to check every copy and every read against the buffers.
//
// Work split over a grid of G CTAs for one token:
//   - gate/up: CTA c takes rows [c*I/G, (c+1)*I/G) of the gate and up matrix
//     of EVERY selected expert (a "row pair" is gate row r with up row r: the
//     two dot products that make h_r = silu(g_r) * u_r);
//   - down: CTA c owns output rows [c*H/G, (c+1)*H/G) and computes them for
//     every selected expert, then combines them.
// Per expert k, the CTA's slot holds (4-bit sizes; a 2-bit expert uses part):
//   gate/up slot: its gate rows back to back (np_max row slots of gu_row
//                 bytes), its up rows likewise, then four segment slots
//                 (gate scales, gate biases, up scales, up biases) of gu_sc
//                 bytes;
//   down slot:    the owned down rows back to back (no_max rows), then two
//                 segment slots (scales, biases) of d_sc bytes.
// A bulk copy (TMA engine) costs tens of nanoseconds of issue whatever its
// size, so every run of consecutive rows is ONE bulk copy: per expert, the
// gate rows, the up rows and the four gate/up scale/bias runs (on its
// gate/up mbarrier), the down rows and the two down scale/bias runs (on its
// down mbarrier), each mbarrier counting the bytes of its copies.  (Copying
// the short scale/bias runs with cp.async instead stalls the issuing warp
// behind the bulk traffic already queued at the SM.)
// A scale/bias run of consecutive rows starts wherever the rows start; its
// copy is widened to 16-byte boundaries (every segment is 16-byte aligned
// and a multiple of 16 bytes long, so the widened copy stays inside it) and
// the reader adds the start's offset within its 16 bytes.
#pragma once

#include <stdint.h>

#include "qe_internal.h"

#ifdef __CUDACC__
#define QE_HD __host__ __device__ __forceinline__
#else
#define QE_HD inline
#endif

namespace qe {

struct FusedCta {
  int r_lo, np;  // gate/up rows [r_lo, r_lo + np) of every expert
  int o_lo, no;  // output rows [o_lo, o_lo + no)
};

// 32-bit arithmetic: c <= 256 and H, I <= 4096 in this kernel (a 64-bit
// division is a long instruction sequence on the GPU).
QE_HD FusedCta fused_cta(int H, int I, int G, int c) {
  FusedCta t;
  t.r_lo = c * I / G;
  t.np = (c + 1) * I / G - t.r_lo;
  t.o_lo = c * H / G;
  t.no = (c + 1) * H / G - t.o_lo;
  return t;
}

// Device addresses of one expert's nine segments, as integers.
struct ExpertAddr {
  uint64_t gwq, uwq, dwq, gs, gb, us, ub, ds, db;
  int bits;
};

QE_HD ExpertAddr expert_addr(const qe_expert& e) {
  ExpertAddr a;
  a.gwq = (uint64_t)(uintptr_t)e.gate.wq;
  a.uwq = (uint64_t)(uintptr_t)e.up.wq;
  a.dwq = (uint64_t)(uintptr_t)e.down.wq;
  a.gs = (uint64_t)(uintptr_t)e.gate.scales;
  a.gb = (uint64_t)(uintptr_t)e.gate.biases;
  a.us = (uint64_t)(uintptr_t)e.up.scales;
  a.ub = (uint64_t)(uintptr_t)e.up.biases;
  a.ds = (uint64_t)(uintptr_t)e.down.scales;
  a.db = (uint64_t)(uintptr_t)e.down.biases;
  a.bits = e.gate.bits;
  return a;
}

// ------------------------------------------------------ shared-memory slots

QE_HD int gu_slot(const FusedGeometry& g, int k) { return g.off_gu + k * g.gu_bytes; }
// m = 0: the gate rows, 1: the up rows of expert k
QE_HD int gu_mat_off(const FusedGeometry& g, int k, int m) { return gu_slot(g, k) + m * g.np_max * g.gu_row; }
// s = 0 gate scales, 1 gate biases, 2 up scales, 3 up biases
QE_HD int gu_sc_off(const FusedGeometry& g, int k, int s) {
  return gu_slot(g, k) + 2 * g.np_max * g.gu_row + s * g.gu_sc;
}
QE_HD int d_slot(const FusedGeometry& g, int k) { return g.off_down + k * g.d_bytes; }
// s = 0 scales, 1 biases
QE_HD int d_sc_off(const FusedGeometry& g, int k, int s) { return d_slot(g, k) + g.no_max * g.d_row + s * g.d_sc; }

// mbarriers: gate/up of expert k, down of expert k
QE_HD int bar_gu(int k) { return k; }
QE_HD int bar_down(int K, int k) { return K + k; }

// Offset of a run's first byte within its widened 16-byte-aligned copy.
QE_HD int run_misalign(uint64_t seg, int row0, int row_bytes) {
  return (int)((seg + (uint64_t)row0 * (uint64_t)row_bytes) & 15ull);
}

// ------------------------------------------------------------- the reads

// 32-column chunk lc of gate (m = 0) or up (m = 1) row pair j of expert k.
QE_HD int gu_word_smem(const FusedGeometry& g, int H, int k, int j, int m, int lc, int bits) {
  return gu_mat_off(g, k, m) + j * (H * bits / 8) + lc * (bits == 4 ? 16 : 8);
}
// bf16 entry gi of row pair j in segment s; mis = run_misalign of that run.
QE_HD int gu_scale_smem(const FusedGeometry& g, int H, int k, int s, int mis, int j, int gi) {
  return gu_sc_off(g, k, s) + mis + j * (H / 32) + gi * 2;
}
// 32-column chunk lc of owned down row i of expert k.
QE_HD int d_word_smem(const FusedGeometry& g, int I, int k, int i, int lc, int bits) {
  return d_slot(g, k) + i * (I * bits / 8) + lc * (bits == 4 ? 16 : 8);
}
QE_HD int d_scale_smem(const FusedGeometry& g, int I, int k, int s, int mis, int i, int gi) {
  return d_sc_off(g, k, s) + mis + i * (I / 32) + gi * 2;
}

// ------------------------------------------------------------- the copies

struct FusedCopy {
  int dst;        // shared-memory offset
  uint64_t src;   // global address
  uint32_t bytes;
  int bar;        // the mbarrier that counts the copy's bytes
};

QE_HD int gu_copies(const FusedCta& t) { return t.np > 0 ? 6 : 0; }
QE_HD int d_copies(const FusedCta& t) { return t.no > 0 ? 3 : 0; }
// Copies of one CTA: all gate/up copies (expert by expert: gate rows, up
// rows, the four scale/bias runs), then all down copies.
QE_HD int fused_ncopies(int K, const FusedCta& t) { return K * (gu_copies(t) + d_copies(t)); }

QE_HD FusedCopy widened(uint64_t seg, int row0, int nrows, int row_bytes) {
  const uint64_t s0 = seg + (uint64_t)row0 * (uint64_t)row_bytes;
  const uint64_t s1 = s0 + (uint64_t)nrows * (uint64_t)row_bytes;
  FusedCopy c;
  c.src = s0 & ~15ull;
  c.bytes = (uint32_t)(((s1 + 15ull) & ~15ull) - c.src);
  c.dst = 0;
  c.bar = 0;
  return c;
}

// Copy u of expert k: u < gu_copies(t) is a gate/up copy, the next
// d_copies(t) are its down copies.
QE_HD FusedCopy fused_expert_copy(const FusedGeometry& g, int H, int I, int K, const FusedCta& t, int k,
                                  const ExpertAddr& a, int u) {
  FusedCopy c;
  if (u < gu_copies(t)) {
    if (u >= 2) {
      const int sidx = u - 2;
      const uint64_t seg = sidx == 0 ? a.gs : sidx == 1 ? a.gb : sidx == 2 ? a.us : a.ub;
      c = widened(seg, t.r_lo, t.np, H / 32);
      c.dst = gu_sc_off(g, k, sidx);
    } else {
      const uint64_t rowb = (uint64_t)H * (uint64_t)a.bits / 8;
      c.dst = gu_mat_off(g, k, u);
      c.src = (u ? a.uwq : a.gwq) + (uint64_t)t.r_lo * rowb;
      c.bytes = (uint32_t)(rowb * (uint64_t)t.np);
    }
    c.bar = bar_gu(k);
    return c;
  }
  u -= gu_copies(t);
  if (u == 0) {
    const uint64_t rowb = (uint64_t)I * (uint64_t)a.bits / 8;
    c.dst = d_slot(g, k);
    c.src = a.dwq + (uint64_t)t.o_lo * rowb;
    c.bytes = (uint32_t)(rowb * (uint64_t)t.no);
  } else {
    c = widened(u == 1 ? a.ds : a.db, t.o_lo, t.no, I / 32);
    c.dst = d_sc_off(g, k, u - 1);
  }
  c.bar = bar_down(K, k);
  return c;
}

// Copy v of the CTA in issue order (0 <= v < fused_ncopies).
QE_HD FusedCopy fused_copy_at(const FusedGeometry& g, int H, int I, int K, const FusedCta& t, const ExpertAddr* a,
                              int v) {
  const int ng = gu_copies(t), nd = d_copies(t);
  if (v < K * ng) return fused_expert_copy(g, H, I, K, t, v / ng, a[v / ng], v % ng);
  v -= K * ng;
  return fused_expert_copy(g, H, I, K, t, v / nd, a[v / nd], ng + v % nd);
}

// Bytes mbarrier b is armed with: the sum over the copies that complete on
// it (0 if none does).
QE_HD uint32_t fused_bar_bytes(const FusedGeometry& g, int H, int I, int K, const FusedCta& t, const ExpertAddr* a,
                               int b) {
  const int k = b < K ? b : b - K;
  const int u0 = b < K ? 0 : gu_copies(t), n = b < K ? gu_copies(t) : d_copies(t);
  uint32_t sum = 0;
  for (int u = u0; u < u0 + n; ++u) sum += fused_expert_copy(g, H, I, K, t, k, a[k], u).bytes;
  return sum;
}

}  // namespace qe
