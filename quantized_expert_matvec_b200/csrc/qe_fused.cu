// qe_fused.cu -- the single-token layer step as ONE persistent kernel:
// RMSNorm -> router (fp64) -> top-K -> gate/up dequant-matvec + SwiGLU ->
// down dequant-matvec -> weighted combine (+ residual).
//
// One CTA of 16 warps per SM, launched cooperatively so every CTA is
// resident; the kernel is bound by HBM bytes and by the latency of the two
// grid-wide exchanges the step needs (all logits before top-K, all of h
// before the down matvecs).
//
// Exchanges.  The step needs two grid-wide exchanges: all logits before
// top-K, all of h before the down matvecs.  Each CTA publishes its values
// as tagged records (a 64-bit word {value, tag}; a logit takes two, written
// and read as one 16-byte access) and the readers poll exactly the records
// they need, with 16-byte relaxed loads, until every word carries this
// launch's tag: one L2 round trip both waits and delivers.  (Per-CTA flags
// or a shared counter need a fence and a second round trip, and were about
// twice as slow on B200.)  For h, every CTA also publishes one "done" record
// after its h records; readers poll those G records first and then read all
// of h once (checking every tag, re-polling the rare stale one), so waiting
// CTAs put little load on L2 while others still stream their down rows.  The
// tag is (epoch + 1) with the top bit set: every launch reads the workspace
// epoch, and CTA 0 advances it at the end, once it has seen every CTA's done
// record (so no CTA of the launch still has to read the old epoch).

// Expert streaming.  Right after top-K, warp k issues the CTA's share of
// selected expert k as 1-D bulk copies (TMA engine) into shared memory: its
// gate and up rows and their scale/bias runs first (one mbarrier), then,
// once every such warp has issued those, its down rows (another).  The
// layout and the copy list are in qe_fused_plan.h.  Nothing waits for a
// copy before all are issued, so the HBM sees the whole step's expert bytes
// at once.
//
// Gate/up: warp (row group rg, column quarter qd) keeps one 32-column chunk
// of xn per lane in registers, as 24-bit fixed-point byte limbs for the dp4a
// dequant core (qe_device.cuh), and walks the row pairs rg, rg+nrg, ... in
// arrival order; quarter sums meet in shared memory.  h records are
// published, every CTA stages all K*I of h in shared memory (the gate/up
// slots are free by then), and warp w computes the owned down rows of
// expert w % K with its lane's chunk of h as limbs in registers.  The CTA
// combines its rows (+ residual).  Every wait is bounded (QE_ERR_TIMEOUT).
#include <math.h>

#include "qe_device.cuh"
#include "qe_fused_plan.h"

namespace qe {

constexpr int kWarps = 16;                           // compute warps
constexpr int kComputeThreads = kWarps * 32;
constexpr int kFusedThreads = kComputeThreads + 32;  // + the warp that issues the copies
constexpr int kBarCompute = 1;                       // named barrier of the compute warps
constexpr int kBarHandoff = 10;                      // warp 0's descriptors, out to the other warps
// named barriers 2 .. 9: one per expert in the down phase (K <= 8 there)
constexpr int kRouterRows = 8;  // router rows one CTA owns at most: E <= 8 * grid

struct FusedMisc {
  int abort;
  unsigned tag;
  int Ex;    // fixed-point exponent of xn: max|xn| < 2^Ex
  float xK;  // 2^(Ex - 22)
  int idx[kMaxK];
  float wk[kMaxK];
  int gu_cnt[kMaxK];      // gate/up warps done with expert k
  int mis_gu[kMaxK][4];   // offsets of the gate/up scale/bias runs in their copies
  int mis_d[kMaxK][2];
  qe_expert ex[kMaxK];    // descriptors of the selected experts
  ExpertAddr ea[kMaxK];   // the same descriptors as addresses (copy plan)
  unsigned long long selkey[kMaxK];  // keys of the selected experts, in rank order
  // expert k's index and descriptor are in (ex[k] landed by cp.async):
  // count 2, the selecting lane's cp.async arrival and its own arrival
  uint64_t dbar[kMaxK];
  unsigned amax_bits;  // max |xn| (float bits)
  double redd[kWarps];
  double rpart[kRouterRows][kWarps];
};

// Optional phase trace: globaltimer stamps per CTA (qe_trace_fused).
enum {
  kTrStart, kTrRouter, kTrLogits, kTrTopK, kTrIssued, kTrFirstPair, kTrGateUp, kTrCombined, kTrDown, kTrEnd,
  kTrMerged, kTrLastGateUpData, kTrDownData, kTrBarsDone, kTrPolledAll, kTrRounds
};
#define QE_TRACE(slot) \
  do { if (p.trace) p.trace[(size_t)blockIdx.x * 16 + (slot)] = gtimer(); } while (0)

static __device__ __forceinline__ float load_x(const FusedParams& p, int c) {
  return p.x_bf16 ? bf16f(((const uint16_t*)p.x)[c]) : ((const float*)p.x)[c];
}

// x[c..c+3] as doubles (fp32 or bf16 input); c is a multiple of 4.
static __device__ __forceinline__ void load_x4(const FusedParams& p, int c, double (&v)[4]) {
  if (p.x_bf16) {
    const uint2 u = *(const uint2*)((const uint16_t*)p.x + c);
    v[0] = bf16f(u.x & 0xFFFFu); v[1] = bf16f(u.x >> 16); v[2] = bf16f(u.y & 0xFFFFu); v[3] = bf16f(u.y >> 16);
  } else {
    const float4 f = *(const float4*)((const float*)p.x + c);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  }
}

static __device__ __forceinline__ bool desc_ok(const qe_qmat& m, int bits) {
  return m.bits == bits && m.wq && m.scales && m.biases && ((uintptr_t)m.wq & 15) == 0 &&
         ((uintptr_t)m.scales & 15) == 0 && ((uintptr_t)m.biases & 15) == 0;
}

static __device__ __forceinline__ bool expert_ok(const qe_expert& ex) {
  const int bits = ex.gate.bits;
  return (bits == 4 || bits == 2) && desc_ok(ex.gate, bits) && desc_ok(ex.up, bits) && desc_ok(ex.down, bits);
}

// Order-preserving map of a double onto an unsigned 64-bit key (-0 and +0
// map to the same key, as they compare equal) and its inverse.
static __device__ __forceinline__ unsigned long long dkey(double d) {
  if (d == 0.0) d = 0.0;
  const unsigned long long u = (unsigned long long)__double_as_longlong(d);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}
static __device__ __forceinline__ double dkey_inv(unsigned long long k) {
  const unsigned long long u = (k >> 63) ? (k & 0x7FFFFFFFFFFFFFFFull) : ~k;
  return __longlong_as_double((long long)u);
}

// Place of expert e's logit record (in 64-bit words): CTA c = e % G writes
// the records of its rows r = e / G (at most 8) into its own 128-byte line.
// A line written by several CTAs while every CTA polls it slows the whole
// exchange down severalfold on B200; one writer per line avoids that.
static __device__ __forceinline__ size_t logit_rec(int e, int G) { return ((size_t)(e % G) * 8 + e / G) * 2; }

// One candidate of the two-level top-K: a key (0: none) and its expert.
struct TopKCand {
  unsigned long long key;
  unsigned idx;
  unsigned pad;
};

// Whether this lane's candidate (key, idx) is the largest key over the
// warp, the lowest index among equal keys.  Lanes without a candidate pass
// key 0 and never win.  Keys are compared by their high words first: when
// one lane alone holds the largest high word (the usual case) it wins;
// otherwise the low words, then the indices decide.
static __device__ __forceinline__ bool lane_wins_argmax(unsigned long long key, unsigned idx) {
  const unsigned hi = (unsigned)(key >> 32), lo = (unsigned)key;
  const unsigned hmax = __reduce_max_sync(0xffffffffu, hi);
  const bool top = key != 0ull && hi == hmax;
  const unsigned mt = __ballot_sync(0xffffffffu, top);
  if (__popc(mt) == 1) return top;  // the same branch for the whole warp
  const unsigned lmax = __reduce_max_sync(0xffffffffu, top ? lo : 0u);
  const bool eq = top && lo == lmax;
  const unsigned m = __ballot_sync(0xffffffffu, eq);
  if (__popc(m) == 1) return eq;
  // every lane takes part in the collective (a full-mask reduction that
  // some lanes skipped, as under a short-circuited &&, would never finish)
  const unsigned imin = __reduce_min_sync(0xffffffffu, eq ? idx : 0xffffffffu);
  return eq && idx == imin;
}

// First level of the top-K, in every compute warp: the K largest of the
// warp's keys (a lane holds up to two: experts lane + 32 w and that + 512),
// written largest first to out[0..K) (key 0 where the warp has fewer).  In
// each round the winning lane moves its second key up.
static __device__ __forceinline__ void warp_topk_local(unsigned long long kA, unsigned iA, unsigned long long kB,
                                                       unsigned iB, int K, int lane, TopKCand* out) {
  const bool sw = kB > kA;  // equal keys: iA, the lower index, first
  unsigned long long k1 = sw ? kB : kA, k2 = sw ? kA : kB;
  unsigned i1 = sw ? iB : iA, i2 = sw ? iA : iB;
  if (lane < K) out[lane] = TopKCand{0ull, 0xffffffffu, 0u};
  __syncwarp();
  for (int k = 0; k < K; ++k) {
    if (lane_wins_argmax(k1, i1)) {
      out[k] = TopKCand{k1, i1, 0u};
      k1 = k2;
      i1 = i2;
      k2 = 0ull;
    }
  }
}

// Bounded poll of N 8-byte records (p[i], or null to skip) until each
// carries `tag`; every round reloads all records still stale at once.
template <int N>
static __device__ __forceinline__ bool poll_rec(const unsigned long long* const (&p)[N], unsigned tag,
                                                uint64_t deadline, volatile int* abort_flag) {
  unsigned long long a[N];
#pragma unroll
  for (int i = 0; i < N; ++i) a[i] = p[i] ? ld_rec(p[i]) : 0ull;
  for (unsigned spins = 0;; ++spins) {
    bool stale = false;
#pragma unroll
    for (int i = 0; i < N; ++i) stale |= p[i] && rec_tag(a[i]) != tag;
    if (!stale) return true;
    if (*abort_flag) return false;
    if ((spins & 7u) == 7u && gtimer() > deadline) return false;
#pragma unroll
    for (int i = 0; i < N; ++i)
      if (p[i] && rec_tag(a[i]) != tag) a[i] = ld_rec(p[i]);
  }
}

// Bounded poll of N 16-byte record pairs (p[i] 16-byte aligned, or null to
// skip) until both words of each carry `tag`; every round reloads all pairs
// still stale at once (one L2 round trip per round).
template <int N>
static __device__ __forceinline__ bool poll_rec2(const unsigned long long* const (&p)[N], unsigned tag,
                                                 uint64_t deadline, volatile int* abort_flag,
                                                 unsigned long long (&a)[N], unsigned long long (&b)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) {
    a[i] = b[i] = 0ull;
    if (p[i]) ld_rec2(p[i], a[i], b[i]);
  }
  for (unsigned spins = 0;; ++spins) {
    bool stale = false;
#pragma unroll
    for (int i = 0; i < N; ++i) stale |= p[i] && (rec_tag(a[i]) != tag || rec_tag(b[i]) != tag);
    if (!stale) return true;
    if (*abort_flag) return false;
    if ((spins & 7u) == 7u && gtimer() > deadline) return false;
#pragma unroll
    for (int i = 0; i < N; ++i)
      if (p[i] && (rec_tag(a[i]) != tag || rec_tag(b[i]) != tag)) ld_rec2(p[i], a[i], b[i]);
  }
}

static __device__ __forceinline__ float ld_bf16(const unsigned char* p) { return bf16f(*(const uint16_t*)p); }

// A gate/up warp has finished its row pairs of expert k: count it, and the
// last of the CTA's gate/up warps to do so turns the quarter sums of expert
// k's rows into h = silu(g) * u and publishes them as tagged records.
// (Unlike the logits, giving each CTA its own lines here measured slower:
// the readers' loads of h_k, coalesced four lines a warp in this layout,
// weigh more than the writers sharing a line.)
static __device__ __forceinline__ void gateup_expert_done(const FusedParams& p, const FusedCta& t, FusedMisc* misc,
                                                          const float* gred, int k, int ngu, int lane,
                                                          unsigned tag) {
  const FusedGeometry& g = p.g;
  __threadfence_block();  // this warp's quarter sums before its count
  __syncwarp();
  int last = 0;
  if (lane == 0) last = atomicAdd(&misc->gu_cnt[k], 1) == ngu - 1;
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __threadfence_block();
  for (int j = lane; j < t.np; j += 32) {
    const int P = k * t.np + j;
    float gs = 0.f, us = 0.f;
    for (int q = 0; q < g.nq; ++q) {
      gs += gred[(P * g.nq + q) * 2];
      us += gred[(P * g.nq + q) * 2 + 1];
    }
    const float hv = gs / (1.0f + expf(-gs)) * us;
    st_rec(&p.rec_h[(size_t)k * p.I + t.r_lo + j], rec_word(__float_as_uint(hv), tag));
  }
}

// kPB row pairs (gate row j and up row j) of expert k at a time: pair i is
// j0 + nrg*i.  The body has no branch (a pair past np is computed on pair
// j0 and dropped), so the compiler interleaves the pairs' loads and dp4a
// chains.  acc[2i] / acc[2i+1]: this lane's 32-column part of the gate /
// up dot of pair i.
constexpr int kPB = 2;
template <int BITS>
static __device__ __forceinline__ void gateup_batch(const FusedGeometry& g, int H, int k, int j0, int np,
                                                    const FusedMisc* misc, const XLimbs& xl, float xsl, float xK,
                                                    const unsigned char* smem, int lc, bool live,
                                                    float (&acc)[2 * kPB]) {
  const int lcs = live ? lc : 0, gi = lcs >> 1;
#pragma unroll
  for (int i = 0; i < kPB; ++i) {
    const int jr = j0 + g.nrg * i;
    const bool valid = jr < np && live;
    const int j = jr < np ? jr : j0;
    const float ag = idot32<BITS>(smem + gu_word_smem(g, H, k, j, 0, lcs, BITS), xl);
    const float au = idot32<BITS>(smem + gu_word_smem(g, H, k, j, 1, lcs, BITS), xl);
    const float sg = ld_bf16(smem + gu_scale_smem(g, H, k, 0, misc->mis_gu[k][0], j, gi));
    const float bg = ld_bf16(smem + gu_scale_smem(g, H, k, 1, misc->mis_gu[k][1], j, gi));
    const float su = ld_bf16(smem + gu_scale_smem(g, H, k, 2, misc->mis_gu[k][2], j, gi));
    const float bu = ld_bf16(smem + gu_scale_smem(g, H, k, 3, misc->mis_gu[k][3], j, gi));
    acc[2 * i] = valid ? sg * xK * ag + bg * xsl : 0.f;
    acc[2 * i + 1] = valid ? su * xK * au + bu * xsl : 0.f;
  }
}

// Gate/up phase of one warp: row group rg = warp / nq, column quarter
// qd = warp % nq, this lane's 32-column chunk lc = 32 qd + lane.  Expert by
// expert (the order their bytes arrive in), the warp waits for the
// expert's copies, takes its row pairs rg, rg + nrg, ... in batches of kPB
// (one transposed warp reduction per batch leaves each pair's two quarter
// sums in gred), and reports the expert done.  Once the last expert's
// bytes are in, a warp has at most one batch left.  The x limbs are
// rebuilt when the bits change from one expert to the next.
static __device__ __forceinline__ void gateup_phase(const FusedParams& p, const FusedCta& t, FusedMisc* misc,
                                                    uint64_t* bars, const float* xn_s, float* gred,
                                                    unsigned char* smem, uint64_t deadline, int warp, int lane,
                                                    unsigned tag) {
  const FusedGeometry& g = p.g;
  const int H = p.H, K = p.K, np = t.np;
  volatile int* abort_flag = &misc->abort;
  const int ngu = g.nq * g.nrg;
  const int qd = warp % g.nq, rg = warp / g.nq;
  const int lc = qd * 32 + lane;
  const bool live = lc < H / 32;
  const float xK = misc->xK;
  XLimbs xl;
  float xsl = 0.f;  // sum of this lane's 32 columns of xn
  int xl_bits = 0;
  for (int k = 0; k < K; ++k) {
    if (rg < np) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars[bar_gu(k)], 0, deadline, abort_flag))) {
        set_error(&p.ctl->err, QE_ERR_TIMEOUT);
        misc->abort = 1;
        return;
      }
      if (warp == 1 && lane == 0 && k == 0) QE_TRACE(kTrFirstPair);
      if (warp == 1 && lane == 0 && k == K - 1) QE_TRACE(kTrLastGateUpData);
      if (__any_sync(0xffffffffu, *abort_flag != 0)) return;  // one decision per warp
      const int bits = misc->ex[k].gate.bits;
      if (bits != xl_bits) {
        if (live) xsl = bits == 4 ? build_limbs<4>(xn_s + 32 * lc, lc & 7, misc->Ex, xl)
                                  : build_limbs<2>(xn_s + 32 * lc, lc & 7, misc->Ex, xl);
        xl_bits = bits;
      }
#pragma unroll 1
      for (int j0 = rg; j0 < np; j0 += g.nrg * kPB) {
        float acc[2 * kPB];
        if (bits == 4) gateup_batch<4>(g, H, k, j0, np, misc, xl, xsl, xK, smem, lc, live, acc);
        else gateup_batch<2>(g, H, k, j0, np, misc, xl, xsl, xK, smem, lc, live, acc);
        // batch row 2i = gate, 2i + 1 = up of pair j0 + nrg*i
        const float r = warp_reduce_rows<2 * kPB>(acc, lane);
        const int row = reduced_row_of_lane<2 * kPB>(lane);
        const int j = j0 + g.nrg * (row >> 1);
        if (lane == lane_of_reduced_row<2 * kPB>(row) && j < np)
          gred[((k * np + j) * g.nq + qd) * 2 + (row & 1)] = r;
      }
    }
    gateup_expert_done(p, t, misc, gred, k, ngu, lane, tag);
  }
}

// Down phase of one warp, after its gate/up: expert k = warp / nwk, one of
// the nwk = 16 / K warps of that expert (wi = warp % nwk).  The warp waits
// until its own CTA has finished expert k's gate/up (the expert's gate/up
// slot is then free and holds nothing anyone still reads), the nwk warps
// poll h_k's records together and stage h_k into that slot (16-byte pieces
// swizzled per 32-column chunk), meet at a named barrier, and compute the
// owned down rows wi, wi + nwk, ... of expert k in batches of 8 with this
// lane's 32-column chunk of h_k as limbs.
template <int BITS>
static __device__ __forceinline__ bool down_phase(const FusedParams& p, const FusedCta& t, FusedMisc* misc,
                                                  uint64_t* bars, float* ycomb, unsigned char* smem,
                                                  uint64_t deadline, int warp, int lane, unsigned tag) {
  const FusedGeometry& g = p.g;
  const int I = p.I, K = p.K;
  volatile int* abort_flag = &misc->abort;
  const int nwk = kWarps / K, k = warp / nwk, wi = warp - k * nwk;
  const int ngu = g.nq * g.nrg;
  // Steps 1-2 may give up (abort flag, wait budget), but every warp of the
  // expert still reaches the named barrier after them exactly once: a warp
  // that left early would leave its partners waiting there for good.
  bool ok = !*abort_flag;
  // 1. this CTA is done with expert k's gate/up
  if (ok) {
    volatile int* cnt = &misc->gu_cnt[k];
    for (unsigned spins = 0; *cnt < ngu; ++spins) {
      __nanosleep(64);
      if ((spins & 15u) == 15u && (*abort_flag || gtimer() > deadline)) {
        ok = false;
        break;
      }
    }
    __threadfence_block();
  }
  ok = __all_sync(0xffffffffu, ok);
  // 2. stage h_k: this warp takes record pairs q = wi*32 + lane + 32*nwk*i,
  // four at a time, all loads in flight together; the records carry their
  // own tag, so the poll both waits for the producing CTAs and delivers
  float* hst = (float*)(smem + gu_slot(g, k));
  const unsigned long long* hrec = p.rec_h + (size_t)k * I;
  for (int q0 = wi * 32 + lane; q0 < I / 2 && ok; q0 += 4 * 32 * nwk) {
    const unsigned long long* rp[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = q0 + 32 * nwk * i;
      rp[i] = q < I / 2 ? hrec + 2 * q : nullptr;
    }
    unsigned long long a[4], b[4];
    ok = poll_rec2<4>(rp, tag, deadline, abort_flag, a, b);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (rp[i])
        *(float2*)(hst + xswz(2 * (q0 + 32 * nwk * i))) =
            make_float2(__uint_as_float(rec_val(a[i])), __uint_as_float(rec_val(b[i])));
  }
  ok = __all_sync(0xffffffffu, ok);
  if (nwk > 1) named_barrier(2 + k, 32 * nwk);  // k < 8 when nwk > 1
  else __syncwarp();
  if (!ok) return false;
  // 4. this lane's chunk of h_k, the expert's exponent from the warp's max
  const bool live = lane < I / 32;
  float v[32];
  float amax = 0.f, hs = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
    if (live) f = ((const float4*)(hst + 32 * lane))[i ^ (lane & 7)];
    v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    hs += v[i];
    amax = fmaxf(amax, fabsf(v[i]));
  }
  const int e = fixed_scale_exponent(warp_max(amax));
  const float hK = pow2f(e - 22);
  XLimbs hl;
  build_limbs_reg<BITS>(v, e, hl);
  if (t.no == 0) return true;
  if (!__all_sync(0xffffffffu, mbar_wait(&bars[bar_down(K, k)], 0, deadline, abort_flag))) return false;
  if (warp == 0 && lane == 0) QE_TRACE(kTrDownData);
  // 5. rows ri = wi + nwk*i of batch b0, one transposed reduction per batch
  const int gi = lane >> 1;
  const int ms0 = misc->mis_d[k][0], ms1 = misc->mis_d[k][1];
#pragma unroll 1
  for (int b0 = wi; b0 < t.no; b0 += nwk * 8) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      acc[i] = 0.f;
      const int ri = b0 + nwk * i;
      if (live && ri < t.no) {
        const float a = idot32<BITS>(smem + d_word_smem(g, I, k, ri, lane, BITS), hl);
        const float s = ld_bf16(smem + d_scale_smem(g, I, k, 0, ms0, ri, gi));
        const float b = ld_bf16(smem + d_scale_smem(g, I, k, 1, ms1, ri, gi));
        acc[i] = s * hK * a + b * hs;
      }
    }
    const float r = warp_reduce_rows<8>(acc, lane);
    const int row = reduced_row_of_lane<8>(lane);
    const int ri = b0 + nwk * row;
    if (lane == lane_of_reduced_row<8>(row) && ri < t.no) ycomb[k * g.no_max + ri] = r;
  }
  return true;
}

__global__ void __launch_bounds__(kFusedThreads, 1) qe_fused_layer_kernel(const FusedParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const FusedGeometry& g = p.g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int H = p.H, E = p.E, K = p.K, I = p.I;
  const FusedCta t = fused_cta(H, I, G, cta);
  const bool given = p.given_idx != nullptr;

  FusedMisc* misc = (FusedMisc*)(smem + g.off_misc);
  volatile int* abort_flag = &misc->abort;
  uint64_t* bars = (uint64_t*)(smem + g.off_bar);
  float* xn_s = (float*)(smem + g.off_xn);      // raw x, then xn; pieces swizzled per chunk (xswz)
  float* gred = (float*)(smem + g.off_gred);    // [K*np_max][nq][2] quarter sums
  float* ycomb = (float*)(smem + g.off_ycomb);  // [K][no_max]
  WsControl* ctl = p.ctl;

  // Prologue, which may run while the previous kernel of the stream is
  // still finishing (programmatic dependent launch): shared-memory set-up
  // and a prefetch of this CTA's router rows into L2 (a hint that reads
  // nothing back), then the wait for the previous kernel's memory.
  if (tid == 0) {
    misc->abort = 0;
    misc->amax_bits = 0u;
    for (int b = 0; b < g.nbar; ++b) mbar_init(&bars[b], 1);
    for (int k = 0; k < K; ++k) mbar_init(&misc->dbar[k], 2);
    fence_mbar_init();
  }
  if (tid < kMaxK) misc->gu_cnt[tid] = 0;
  if (!given) {
    const int nrows_pf = E > cta ? (E - cta + G - 1) / G : 0, lines = H / 32;  // 128-byte lines per row
    for (int i = tid; i < nrows_pf * lines; i += kFusedThreads)
      prefetch_l2(p.router_w + (size_t)(cta + G * (i / lines)) * H + 32 * (i % lines));
  }
  grid_dependency_wait();
  grid_launch_dependents();
  const uint64_t deadline = gtimer() + p.budget_ns;
  unsigned epoch = 0;
  if (tid == 0) {
    epoch = ld_relaxed_u32(&ctl->epoch);  // used once the router loads are in flight
    QE_TRACE(kTrStart);
  }

  // Every warp of the CTA agrees on `issued` (the copies went out): warp 0
  // from its lanes' checks, the others from the abort flag it sets before
  // the hand-off barrier.
  bool issued = false;
  unsigned tag = 0;    // this launch's record tag (compute warps)
  unsigned armed = 0;  // copy warp: bit k, expert k's copies were issued
  if (warp < kWarps) {
    // ------------------------------------------------------------- routing
    // The router dot s_e = sum_c W[e,c] x_c gamma_c does not depend on the
    // RMSNorm scale, so it runs on the same x loads as the sum of squares; the
    // logit is s_e * rinv (+ offset_e), in fp64.  CTA c owns rows c, c+G, ...;
    // thread t covers float4 columns t and t + 512 of each of them.
    const int nrows = (!given && E > cta) ? (E - cta + G - 1) / G : 0;
    const int nf4 = H / 4;
    {
      // the first (usually only) batch of router rows is requested before x
      float4 wv[4][2];
      auto load_rows = [&](int r0) {
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
          for (int s = 0; s < 2; ++s) {
            const int f = tid + s * kComputeThreads;
            wv[m][s] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r0 + m < nrows && f < nf4)
              wv[m][s] = __ldg((const float4*)(p.router_w + (size_t)(cta + G * (r0 + m)) * H) + f);
          }
      };
      load_rows(0);
      double xg[2][4];
      double ss = 0.0;
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int f = tid + s * kComputeThreads;
#pragma unroll
        for (int i = 0; i < 4; ++i) xg[s][i] = 0.0;
        if (f < nf4) {
          load_x4(p, 4 * f, xg[s]);
          ss += xg[s][0] * xg[s][0] + xg[s][1] * xg[s][1] + xg[s][2] * xg[s][2] + xg[s][3] * xg[s][3];
          // raw x for RMSNorm pass 2
          *(float4*)(xn_s + xswz(4 * f)) = make_float4((float)xg[s][0], (float)xg[s][1], (float)xg[s][2], (float)xg[s][3]);
          if (p.gamma) {
            const float4 gm = *(const float4*)(p.gamma + 4 * f);
            xg[s][0] *= (double)gm.x; xg[s][1] *= (double)gm.y; xg[s][2] *= (double)gm.z; xg[s][3] *= (double)gm.w;
          }
        }
      }
      // one transposed warp reduction per batch of 4 rows; the first batch
      // also carries the sum of squares (value 4 of 8)
      for (int r0 = 0; r0 == 0 || r0 < nrows; r0 += 4) {
        if (r0 > 0) load_rows(r0);
        double a[8];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          a[m] = 0.0;  // rows past nrows were loaded as zeros
#pragma unroll
          for (int s = 0; s < 2; ++s) {
            a[m] = fma((double)wv[m][s].x, xg[s][0], a[m]);
            a[m] = fma((double)wv[m][s].y, xg[s][1], a[m]);
            a[m] = fma((double)wv[m][s].z, xg[s][2], a[m]);
            a[m] = fma((double)wv[m][s].w, xg[s][3], a[m]);
          }
        }
        a[4] = r0 == 0 ? ss : 0.0;
        a[5] = a[6] = a[7] = 0.0;
        const double r = warp_reduce_rows<8>(a, lane);
        const int row = reduced_row_of_lane<8>(lane);
        if (lane == lane_of_reduced_row<8>(row)) {
          if (row < 4 && r0 + row < nrows) misc->rpart[r0 + row][warp] = r;
          if (row == 4 && r0 == 0) misc->redd[warp] = r;
        }
      }
    }
    if (tid == 0) {
      const unsigned tg = 0x80000000u | ((epoch + 1u) & 0x7FFFFFFFu);
      misc->tag = tg;
      st_rec(&p.rec_done[(size_t)cta * kDoneStride], rec_word(0u, tg));  // this CTA has read the epoch
    }
    named_barrier(kBarCompute, kComputeThreads);
    if (tid == 0) QE_TRACE(kTrRouter);
    tag = misc->tag;
    double rinv;
    {
      double tot = 0.0;
      for (int w = 0; w < kWarps; ++w) tot += misc->redd[w];
      rinv = 1.0 / sqrt(tot / (double)H + (double)p.eps);
    }
    if (tid < nrows && cta != p.skip_cta) {
      double sl = 0.0;
      for (int w = 0; w < kWarps; ++w) sl += misc->rpart[tid][w];
      const int e = cta + G * tid;
      const unsigned long long key = dkey(sl * rinv + (p.offset ? (double)p.offset[e] : 0.0));
      st_rec2(&p.rec_logit[logit_rec(e, G)], rec_word((uint32_t)key, tag), rec_word((uint32_t)(key >> 32), tag));
    }
    // RMSNorm pass 2 (fp32 suffices: xn feeds the expert matvecs, not the
    // routing) and max |xn|
    {
      const float rinv_f = (float)rinv;
      float amax = 0.f;
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int f = tid + s * kComputeThreads;
        if (f < nf4) {
          float4 v = *(const float4*)(xn_s + xswz(4 * f));
          float4 gm = make_float4(1.f, 1.f, 1.f, 1.f);
          if (p.gamma) gm = *(const float4*)(p.gamma + 4 * f);
          v.x = v.x * rinv_f * gm.x; v.y = v.y * rinv_f * gm.y; v.z = v.z * rinv_f * gm.z; v.w = v.w * rinv_f * gm.w;
          *(float4*)(xn_s + xswz(4 * f)) = v;
          amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
        }
      }
      amax = warp_max(amax);
      if (lane == 0) atomicMax(&misc->amax_bits, __float_as_uint(amax));  // non-negative: ordered as integers
    }

    // ---------------------------------------------------------------- top-K
    // Two levels.  Thread t polls the records of experts t and t + 512, and
    // its warp takes the K largest of its keys at once (warp_topk_local);
    // after the barrier warp 0 merges the 16 sorted lists: lane w holds the
    // head of warp w's list, and in each of K rounds the winning lane takes
    // its head and moves to its next one.  Equal keys: the lower expert
    // index, at both levels.  As each winner is known its descriptor is
    // requested (cp.async) into shared memory.
    TopKCand* cand = (TopKCand*)(smem + g.off_cand);  // [kWarps][K]
    if (!given) {
      const unsigned iA = (unsigned)tid, iB = (unsigned)(tid + kComputeThreads);
      const bool hasA = (int)iA < E, hasB = (int)iB < E;
      const unsigned long long* const rp[2] = {hasA ? &p.rec_logit[logit_rec(iA, G)] : nullptr,
                                               hasB ? &p.rec_logit[logit_rec(iB, G)] : nullptr};
      unsigned long long lo[2], hi[2];
      if (!poll_rec2<2>(rp, tag, deadline, abort_flag, lo, hi)) {
        set_error(&ctl->err, QE_ERR_TIMEOUT);
        misc->abort = 1;
      }
      if (tid == 0) QE_TRACE(kTrLogits);
      // a key of 0 stands for "none"; the one key a real logit could map to
      // 0 (a negative NaN with every payload bit set) is raised to 1
      unsigned long long kA = ((unsigned long long)rec_val(hi[0]) << 32) | rec_val(lo[0]);
      unsigned long long kB = ((unsigned long long)rec_val(hi[1]) << 32) | rec_val(lo[1]);
      kA = hasA ? (kA ? kA : 1ull) : 0ull;
      kB = hasB ? (kB ? kB : 1ull) : 0ull;
      warp_topk_local(kA, iA, kB, iB, K, lane, cand + warp * K);
    }
    named_barrier(kBarCompute, kComputeThreads);
    if (warp == 0 && !*abort_flag) {
      // the compute warps need only xn's exponent to start: hand off now;
      // each expert's descriptor follows through its dbar mbarrier
      if (lane == 0) {
        misc->Ex = fixed_scale_exponent(__uint_as_float(misc->amax_bits));
        misc->xK = pow2f(misc->Ex - 22);
      }
      __syncwarp();
      named_barrier_arrive(kBarHandoff, kFusedThreads);
      issued = true;
      // expert k is decided: record it, fetch its descriptor into ex[k]
      // (cp.async), arrive twice on dbar[k]
      auto publish = [&](int k, int e) {
        misc->idx[k] = e;
        if (e >= 0 && e < E) {
          const unsigned char* src = (const unsigned char*)(p.experts + e);
          unsigned char* dst = (unsigned char*)&misc->ex[k];
#pragma unroll
          for (int q = 0; q < (int)sizeof(qe_expert); q += 8) cp_async8(dst + q, src + q);
        }
        cp_async_mbar_arrive_noinc(&misc->dbar[k]);
        mbar_arrive(&misc->dbar[k]);
      };
      if (given) {
        // routing decided beforehand: take its experts and weights as they are
        if (lane < K) {
          misc->wk[lane] = p.given_w[lane];
          publish(lane, p.given_idx[lane]);
        }
      } else {
        if (lane == 0) QE_TRACE(kTrPolledAll);
        const TopKCand* cl = cand + lane * K;
        int h = 0;
        TopKCand c = lane < kWarps ? cl[0] : TopKCand{0ull, 0xffffffffu, 0u};
        for (int k = 0; k < K; ++k) {
          if (lane_wins_argmax(c.key, c.idx)) {
            misc->selkey[k] = c.key;
            publish(k, (int)c.idx);
            ++h;
            c = h < K ? cl[h] : TopKCand{0ull, 0xffffffffu, 0u};
          }
        }
        if (lane == 0) QE_TRACE(kTrRounds);
        __syncwarp();
        // renormalised softmax over the K kept logits (sum in k order); the
        // weights are needed at the combine only
        const double lmax = dkey_inv(misc->selkey[0]);
        const float ev = lane < K ? expf((float)(dkey_inv(misc->selkey[lane]) - lmax)) : 0.0f;
        float sum = 0.0f;
        for (int k = 0; k < K; ++k) sum += __shfl_sync(0xffffffffu, ev, k);
        if (lane < K) misc->wk[lane] = ev / sum;
      }
      __syncwarp();
      if (cta == 0 && lane < K) {
        if (p.topk_idx) p.topk_idx[lane] = misc->idx[lane];
        if (p.topk_w) p.topk_w[lane] = misc->wk[lane];
      }
      if (lane == 0) QE_TRACE(kTrMerged);
    } else {
      named_barrier(kBarHandoff, kFusedThreads);
      issued = !*abort_flag;
    }

    // ------------------------------------------ gate/up and down, pipelined
    // Every warp does its gate/up pairs, then down rows of expert
    // warp / (16 / K) as soon as that expert is ready; the last warp to finish
    // an expert's pairs publishes its h.  Experts stream in one after the
    // other and each group of warps works on its own expert, so the exchange
    // and the down rows of the early experts overlap the later ones' data.
    if (issued) {
      bool ok = true;
      if (warp < g.nq * g.nrg) {
        gateup_phase(p, t, misc, bars, xn_s, gred, smem, deadline, warp, lane, tag);
        if (warp == 0 && lane == 0) QE_TRACE(kTrGateUp);
      }
      if (warp < K * (kWarps / K)) {  // every warp of an expert calls it (named barrier inside)
        // the expert's descriptor (a warp without gate/up rows has not
        // waited for it yet)
        const int kd = warp / (kWarps / K);
        mbar_wait(&misc->dbar[kd], 0, deadline, abort_flag);
        ok = misc->ex[kd].down.bits == 4
                 ? down_phase<4>(p, t, misc, bars, ycomb, smem, deadline, warp, lane, tag)
                 : down_phase<2>(p, t, misc, bars, ycomb, smem, deadline, warp, lane, tag);
        if (!ok && lane == 0 && !*abort_flag) {
          set_error(&ctl->err, QE_ERR_TIMEOUT);
          misc->abort = 1;
        }
      }
    }
    named_barrier(kBarCompute, kComputeThreads);
    if (tid == 0) QE_TRACE(kTrDown);

    // ----------------------------------------------- combine of owned rows
    if (issued && !*abort_flag) {
      for (int i = tid; i < t.no; i += kComputeThreads) {
        const int r = t.o_lo + i;
        float acc = 0.f;
        for (int k = 0; k < K; ++k) acc += misc->wk[k] * ycomb[k * g.no_max + i];
        if (p.add_residual) acc += load_x(p, r);
        p.out[r] = acc;
      }
    }
    if (tid == 0) QE_TRACE(kTrCombined);
  } else {
    // ---------------------------------------------------- the copy warp
    named_barrier(kBarHandoff, kFusedThreads);
    issued = !*abort_flag;
    if (issued) {
      // Expert by expert, as warp 0 decides them: wait for the descriptor,
      // check it, write what the compute warps read of it, arm the expert's
      // gate/up mbarrier and issue its gate/up copies (lane u takes copy u:
      // gate rows, up rows, the four scale/bias runs).  Then the down copies
      // of every expert.  Each expert's gate/up bytes are ahead of the next
      // expert's, and all of them ahead of the down rows.  A bulk copy's
      // issue waits while the SM's queue of copies is full, so this warp
      // keeps issuing for most of the stream; nothing else waits on it.
      const uint64_t pol = policy_evict_first();
      const int ng = gu_copies(t), nd = d_copies(t);
      for (int k = 0; k < K; ++k) {
        if (!__all_sync(0xffffffffu, mbar_wait(&misc->dbar[k], 0, deadline, abort_flag))) {
          if (lane == 0) {
            set_error(&ctl->err, QE_ERR_TIMEOUT);
            __threadfence_block();
            misc->abort = 1;
          }
          break;
        }
        const int e = misc->idx[k];
        qe_expert ex{};
        bool ok = e >= 0 && e < E;
        if (ok) {
          ex = misc->ex[k];
          ok = expert_ok(ex);
        }
        if (!ok) {  // the same decision in every lane
          if (lane == 0) {
            set_error(&ctl->err, QE_ERR_INVALID_ARG);
            __threadfence_block();  // the error word before the flag others act on
            misc->abort = 1;
          }
          break;
        }
        const ExpertAddr ak = expert_addr(ex);
        if (lane == 0) {
          misc->ea[k] = ak;
          misc->mis_gu[k][0] = run_misalign(ak.gs, t.r_lo, H / 32);
          misc->mis_gu[k][1] = run_misalign(ak.gb, t.r_lo, H / 32);
          misc->mis_gu[k][2] = run_misalign(ak.us, t.r_lo, H / 32);
          misc->mis_gu[k][3] = run_misalign(ak.ub, t.r_lo, H / 32);
          misc->mis_d[k][0] = run_misalign(ak.ds, t.o_lo, I / 32);
          misc->mis_d[k][1] = run_misalign(ak.db, t.o_lo, I / 32);
          // releases the writes above to the warps that wait on the barrier
          if (ng) mbar_arrive_expect_tx(&bars[bar_gu(k)], fused_bar_bytes(g, H, I, K, t, misc->ea, bar_gu(k)));
        }
        __syncwarp();
        if (lane < ng) {
          const FusedCopy c = fused_expert_copy(g, H, I, K, t, k, ak, lane);
          bulk_g2s(smem + c.dst, (const void*)(uintptr_t)c.src, c.bytes, &bars[c.bar], pol);
        }
        armed |= 1u << k;
        if (k == 0 && lane == 0) QE_TRACE(kTrTopK);
      }
      for (int k = 0; k < K && nd; ++k) {
        if (!(armed >> k & 1u)) break;
        if (lane == 0)
          mbar_arrive_expect_tx(&bars[bar_down(K, k)], fused_bar_bytes(g, H, I, K, t, misc->ea, bar_down(K, k)));
        __syncwarp();
        if (lane < nd) {
          const FusedCopy c = fused_expert_copy(g, H, I, K, t, k, misc->ea[k], ng + lane);
          bulk_g2s(smem + c.dst, (const void*)(uintptr_t)c.src, c.bytes, &bars[c.bar], pol);
        }
      }
      if (lane == 0) QE_TRACE(kTrIssued);
    }
    // CTA 0 advances the launch epoch at the end: check here, off the
    // compute warps' path, that every CTA has read it (its "read the epoch"
    // record, lanes polling CTAs lane, lane + 32, ...).  Every CTA writes
    // that record right after its router whatever happens later, so this
    // wait does not end early on an abort: an epoch advanced before a CTA
    // read it would hand that CTA the next launch's tag.
    if (cta == 0) {
      const unsigned tg = misc->tag;  // written before the hand-off
      for (int c0 = 0; c0 < G; c0 += 8 * 32) {
        const unsigned long long* rp[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int c = c0 + lane + 32 * i;
          rp[i] = c < G ? &p.rec_done[(size_t)c * kDoneStride] : nullptr;
        }
        volatile int no_abort = 0;
        if (!poll_rec<8>(rp, tg, deadline, &no_abort)) {
          set_error(&ctl->err, QE_ERR_TIMEOUT);
          misc->abort = 1;
        }
      }
    }
  }
  // no copy may still be landing when the CTA exits (they all have, unless
  // a wait gave up): wait for every armed mbarrier, bounded
  if (warp == kWarps && issued) {
    volatile int no_abort = 0;
    const uint64_t dl2 = gtimer() + p.budget_ns;
    for (int b = lane; b < g.nbar; b += 32) {
      const int k = b < K ? b : b - K;
      if ((armed >> k & 1u) && fused_bar_bytes(g, H, I, K, t, misc->ea, b)) mbar_wait(&bars[b], 0, dl2, &no_abort);
    }
  }
  // the descriptor copies warp 0 started (normally long landed)
  if (warp == 0) cp_async_wait_all();
  if (warp == kWarps && lane == 0) QE_TRACE(kTrBarsDone);
  __syncthreads();
  if (tid == 0) {
    // every CTA has read the epoch (CTA 0 saw every CTA's record, or gave
    // up after the wait budget): advance it for the next launch
    if (cta == 0) st_relaxed_u32(&ctl->epoch, tag & 0x7FFFFFFFu);
    QE_TRACE(kTrEnd);
  }
}

// ------------------------------------------------------------ host side

static int align_up(int v, int a) { return (v + a - 1) / a * a; }

int fused_geometry(int H, int E, int K, int I, int sms, int smem_optin, FusedGeometry* out) {
  FusedGeometry g{};
  // one 32-column chunk per lane: a gate/up row in at most 4 warps, a down
  // row in one
  if (H % 64 != 0 || I % 64 != 0 || H > 4096 || I > 1024) return QE_ERR_UNSUPPORTED;
  if (K < 1 || K > kMaxK || E > 2 * kComputeThreads) return QE_ERR_UNSUPPORTED;
  if (sms < 1 || sms > kMaxGrid || E > kRouterRows * sms) return QE_ERR_UNSUPPORTED;
  g.grid = sms;
  g.nq = (H / 32 + 31) / 32;
  g.nrg = kWarps / g.nq;
  g.np_max = (I + sms - 1) / sms;
  g.no_max = (H + sms - 1) / sms;
  g.gu_row = H / 2;
  g.gu_sc = align_up(g.np_max * (H / 32) + 30, 16);
  g.gu_bytes = 2 * g.np_max * g.gu_row + 4 * g.gu_sc;
  if (g.gu_bytes < 4 * I) g.gu_bytes = 4 * I;  // h_k is staged in expert k's slot
  g.d_row = I / 2;
  g.d_sc = align_up(g.no_max * (I / 32) + 30, 16);
  g.d_bytes = g.no_max * g.d_row + 2 * g.d_sc;
  g.nbar = 2 * K;
  int off = 0;
  g.off_misc = off; off = align_up(off + (int)sizeof(FusedMisc), 128);
  g.off_bar = off; off = align_up(off + 8 * g.nbar, 128);
  g.off_xn = off; off = align_up(off + 4 * H, 128);
  g.off_cand = off; off = align_up(off + (int)sizeof(TopKCand) * kWarps * K, 128);  // top-K candidates
  g.off_gred = off; off = align_up(off + 4 * 2 * g.nq * K * g.np_max, 128);
  g.off_ycomb = off; off = align_up(off + 4 * K * g.no_max, 128);
  g.off_gu = off;
  off = align_up(off + K * g.gu_bytes, 128);
  g.off_down = off;
  off += K * g.d_bytes;
  g.smem_bytes = align_up(off, 128);
  if (g.smem_bytes > smem_optin) return QE_ERR_UNSUPPORTED;
  *out = g;
  return QE_OK;
}

cudaError_t launch_fused_layer(const FusedParams& p, cudaStream_t s) {
  static int attr_dev = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (attr_dev != dev) {
    int optin = 0;
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    e = cudaFuncSetAttribute(qe_fused_layer_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e != cudaSuccess) return e;
    attr_dev = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.g.grid);
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = p.g.smem_bytes;
  cfg.stream = s;
  // Every CTA must be resident at once (one per SM; the CTAs wait on one
  // another with bounded waits).  No cooperative attribute: with it the
  // launch does not overlap the previous kernel's tail.  Programmatic
  // dependent launch lets the CTAs start their prologue on SMs the
  // previous kernel has left, before that kernel has finished.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, qe_fused_layer_kernel, p);
}

}  // namespace qe

// ---------------------------------------------------------------------------
// Host probe of the single-token kernel's plan (no GPU involved): geometry,
// the bulk copies of CTA `cta` and the shared-memory offset of every read
// the kernel makes from them, computed by the same functions the kernel
// uses.  The CPU tests check the copies against the buffers and every read
// against the copies.
extern "C" QE_API int qe_fused_plan_probe(int H, int E, int K, int I, int sms, int smem_optin, int cta,
                                          const int* bits, const uint64_t* seg /* [K][9] */, int* geom /* [64] */,
                                          long long* copies /* [max_copies][4] */, int max_copies,
                                          long long* reads /* [max_reads][6] */, int max_reads) {
  using namespace qe;
  FusedGeometry g;
  const int rc = fused_geometry(H, E, K, I, sms, smem_optin, &g);
  if (rc != QE_OK) return rc;
  const int gv[24] = {g.grid, g.nq, g.nrg, g.np_max, g.no_max, g.gu_row, g.gu_sc, g.gu_bytes,
                      g.d_row, g.d_sc, g.d_bytes, g.nbar, g.off_xn, g.off_cand, g.off_misc, g.off_bar,
                      g.off_gred, g.off_ycomb, g.off_gu, g.off_down, g.smem_bytes, 0, 0, 0};
  for (int i = 0; i < 24; ++i) geom[i] = gv[i];
  const FusedCta t = fused_cta(H, I, sms, cta);
  ExpertAddr a[kMaxK];
  for (int k = 0; k < K; ++k) {
    const uint64_t* s = seg + 9 * k;
    a[k] = ExpertAddr{s[0], s[1], s[2], s[3], s[4], s[5], s[6], s[7], s[8], bits[k]};
  }
  const int nc = fused_ncopies(K, t);
  if (nc > max_copies) return QE_ERR_INVALID_ARG;
  for (int v = 0; v < nc; ++v) {
    const FusedCopy c = fused_copy_at(g, H, I, K, t, a, v);
    copies[4 * v] = c.dst;
    copies[4 * v + 1] = (long long)c.src;
    copies[4 * v + 2] = c.bytes;
    copies[4 * v + 3] = c.bar;
  }
  for (int b = 0; b < 40; ++b) geom[24 + b] = b < g.nbar ? (int)fused_bar_bytes(g, H, I, K, t, a, b) : 0;
  // reads: {kind, k, a, b, smem offset, bytes}; kind 0 gate/up word (a =
  // 2j + m, b = chunk), 1 gate/up scale/bias (a = 4j + s, b = group),
  // 2 down word (a = row, b = chunk), 3 down scale/bias (a = 2i + s, b = group)
  int nr = 0;
  auto put = [&](int kind, int k, int x, int y, int off, int bytes) {
    if (nr < max_reads) {
      long long* r = reads + 6 * nr;
      r[0] = kind; r[1] = k; r[2] = x; r[3] = y; r[4] = off; r[5] = bytes;
    }
    ++nr;
  };
  for (int k = 0; k < K; ++k) {
    const int b = a[k].bits;
    const uint64_t sg[4] = {a[k].gs, a[k].gb, a[k].us, a[k].ub};
    for (int j = 0; j < t.np; ++j)
      for (int m = 0; m < 2; ++m)
        for (int lc = 0; lc < H / 32; ++lc) put(0, k, 2 * j + m, lc, gu_word_smem(g, H, k, j, m, lc, b), b == 4 ? 16 : 8);
    for (int j = 0; j < t.np; ++j)
      for (int s = 0; s < 4; ++s)
        for (int gi = 0; gi < H / 64; ++gi)
          put(1, k, 4 * j + s, gi, gu_scale_smem(g, H, k, s, run_misalign(sg[s], t.r_lo, H / 32), j, gi), 2);
    for (int i = 0; i < t.no; ++i)
      for (int lc = 0; lc < I / 32; ++lc) put(2, k, i, lc, d_word_smem(g, I, k, i, lc, b), b == 4 ? 16 : 8);
    const uint64_t sd[2] = {a[k].ds, a[k].db};
    for (int i = 0; i < t.no; ++i)
      for (int s = 0; s < 2; ++s)
        for (int gi = 0; gi < I / 64; ++gi)
          put(3, k, 2 * i + s, gi, d_scale_smem(g, I, k, s, run_misalign(sd[s], t.o_lo, I / 32), i, gi), 2);
  }
  geom[21] = nc;
  geom[22] = nr;
  geom[23] = t.r_lo;
  return nr > max_reads ? QE_ERR_INVALID_ARG : QE_OK;
}
