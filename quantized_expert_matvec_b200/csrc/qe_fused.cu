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

constexpr int kWarps = 16;
constexpr int kFusedThreads = kWarps * 32;
constexpr int kRouterRows = 8;  // router rows one CTA owns at most: E <= 8 * grid

struct FusedMisc {
  int abort;
  unsigned tag;
  int Ex;    // fixed-point exponent of xn: max|xn| < 2^Ex
  float xK;  // 2^(Ex - 22)
  int ubits; // bits shared by all K selected experts (4 or 2), 0 if mixed
  int idx[kMaxK];
  float wk[kMaxK];
  int hexp[kMaxK];  // fixed-point exponent of h_k
  float hK[kMaxK];  // 2^(hexp - 22)
  unsigned hamax[kMaxK];  // max |h_k| as float bits
  int mis_gu[kMaxK][4];   // offsets of the gate/up scale/bias runs in their copies
  int mis_d[kMaxK][2];
  qe_expert ex[kMaxK];
  ExpertAddr ea[kMaxK];   // the same descriptors as addresses (copy plan)
  unsigned long long selkey[kMaxK];  // keys of the selected experts, in rank order
  float redf[kWarps];
  double redd[kWarps];
  double rpart[kRouterRows][kWarps];
};

// Optional phase trace: globaltimer stamps per CTA (qe_trace_fused).
enum {
  kTrStart, kTrRouter, kTrLogits, kTrTopK, kTrIssued, kTrFirstPair, kTrGateUp, kTrHStaged, kTrDown, kTrEnd,
  kTrMerged, kTrLastGateUpData, kTrDownData, kTrHPolled, kTrPolledAll, kTrRounds
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

// Largest key over the warp, the lowest index among equal keys.  Lanes
// without a candidate pass idx 0xffffffff.  Returns the winning index.
static __device__ __forceinline__ unsigned warp_argmax_key(unsigned long long key, unsigned idx) {
  const bool has = idx != 0xffffffffu;
  const unsigned hi = (unsigned)(key >> 32), lo = (unsigned)key;
  const unsigned hmax = __reduce_max_sync(0xffffffffu, has ? hi : 0u);
  const bool top = has && hi == hmax;
  const unsigned lmax = __reduce_max_sync(0xffffffffu, top ? lo : 0u);
  return __reduce_min_sync(0xffffffffu, (top && lo == lmax) ? idx : 0xffffffffu);
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

// Gate/up phase of one warp: row group rg = warp / nq, column quarter
// qd = warp % nq, this lane's 32-column chunk lc = 32 qd + lane.  The warp
// takes the row pairs P = rg, rg + nrg, ... of the flattened (expert, row)
// list in batches of kPB (one transposed warp reduction per batch: warp
// shuffles are a scarce resource when all 16 warps reduce), waits for an
// expert's mbarrier when it first meets that expert, and leaves each pair's
// two quarter sums in gred.  BITS is the bits of every selected expert, or
// 0 when they differ (each pair then picks its core).
constexpr int kPB = 4;
template <int BITS>
static __device__ __forceinline__ void gateup_phase(const FusedParams& p, const FusedCta& t, FusedMisc* misc,
                                                    uint64_t* bars, const float* xn_s, float* gred,
                                                    unsigned char* smem, uint64_t deadline, int warp, int lane) {
  const FusedGeometry& g = p.g;
  const int H = p.H, K = p.K;
  volatile int* abort_flag = &misc->abort;
  const int qd = warp % g.nq, rg = warp / g.nq;
  const int lc = qd * 32 + lane;
  const bool live = lc < H / 32;
  const int gi = lc >> 1;
  const int npairs = K * t.np;
  const float xK = misc->xK;
  XLimbs xl;
  float xsl = 0.f;  // sum of this lane's 32 columns of xn
  int xl_bits = 0;
  int have_k = -1;  // experts [0, have_k] have landed
#pragma unroll 1
  for (int p0 = rg; p0 < npairs; p0 += g.nrg * kPB) {
    if (__any_sync(0xffffffffu, *abort_flag != 0)) break;  // one decision per warp
    float acc[2 * kPB];
#pragma unroll
    for (int i = 0; i < kPB; ++i) {
      acc[2 * i] = acc[2 * i + 1] = 0.f;
      const int P = p0 + g.nrg * i;
      if (P < npairs) {  // uniform over the warp
        const int k = P / t.np, j = P - k * t.np;
        const int bits = BITS ? BITS : misc->ex[k].gate.bits;
        if (bits != xl_bits) {
          if (live) xsl = bits == 4 ? build_limbs<4>(xn_s + 32 * lc, lc & 7, misc->Ex, xl)
                                    : build_limbs<2>(xn_s + 32 * lc, lc & 7, misc->Ex, xl);
          xl_bits = bits;
        }
        if (k > have_k) {
          if (!__all_sync(0xffffffffu, mbar_wait(&bars[bar_gu(k)], 0, deadline, abort_flag))) {
            set_error(&p.ctl->err, QE_ERR_TIMEOUT);
            misc->abort = 1;
            break;
          }
          have_k = k;
          if (warp == 0 && lane == 0 && P == 0) QE_TRACE(kTrFirstPair);
          if (warp == 0 && lane == 0 && k == K - 1) QE_TRACE(kTrLastGateUpData);
        }
        if (live) {
          const unsigned char* wg = smem + gu_word_smem(g, H, k, j, 0, lc, bits);
          const unsigned char* wu = smem + gu_word_smem(g, H, k, j, 1, lc, bits);
          float ag, au;
          if (BITS) {
            ag = idot32<BITS ? BITS : 4>(wg, xl);
            au = idot32<BITS ? BITS : 4>(wu, xl);
          } else if (bits == 4) {
            ag = idot32<4>(wg, xl);
            au = idot32<4>(wu, xl);
          } else {
            ag = idot32<2>(wg, xl);
            au = idot32<2>(wu, xl);
          }
          const float sg = ld_bf16(smem + gu_scale_smem(g, H, k, 0, misc->mis_gu[k][0], j, gi));
          const float bg = ld_bf16(smem + gu_scale_smem(g, H, k, 1, misc->mis_gu[k][1], j, gi));
          const float su = ld_bf16(smem + gu_scale_smem(g, H, k, 2, misc->mis_gu[k][2], j, gi));
          const float bu = ld_bf16(smem + gu_scale_smem(g, H, k, 3, misc->mis_gu[k][3], j, gi));
          acc[2 * i] = sg * xK * ag + bg * xsl;
          acc[2 * i + 1] = su * xK * au + bu * xsl;
        }
      }
    }
    // batch row 2i = gate, 2i + 1 = up of pair p0 + nrg*i
    const float r = warp_reduce_rows<2 * kPB>(acc, lane);
    const int row = reduced_row_of_lane<2 * kPB>(lane);
    const int P = p0 + g.nrg * (row >> 1);
    if (lane == lane_of_reduced_row<2 * kPB>(row) && P < npairs) gred[(P * g.nq + qd) * 2 + (row & 1)] = r;
  }
}

// Down phase of one warp: expert k = warp % K, its owned rows wi, wi + nwk,
// ... (wi = warp / K, nwk = warps per expert), one row at a time, with this
// lane's 32-column chunk of h_k as limbs in registers; row results go to
// ycomb.
template <int BITS>
static __device__ __forceinline__ void down_phase(const FusedParams& p, const FusedCta& t, FusedMisc* misc,
                                                  uint64_t* bars, const float* hst, float* ycomb,
                                                  unsigned char* smem, uint64_t deadline, int warp, int lane) {
  const FusedGeometry& g = p.g;
  const int K = p.K, I = p.I;
  volatile int* abort_flag = &misc->abort;
  const int k = warp % K, wi = warp / K, nwk = kWarps / K;
  const bool live = lane < I / 32;
  const int gi = lane >> 1;
  XLimbs hl;
  float hs = 0.f;
  const int ch = k * (I / 32) + lane;  // this lane's chunk of the staged h
  if (live) hs = build_limbs<BITS>(hst + 32 * ch, ch & 7, misc->hexp[k], hl);
  const float hK = misc->hK[k];
  const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[bar_down(K, k)], 0, deadline, abort_flag));
  if (warp == 0 && lane == 0) QE_TRACE(kTrDownData);
  if (!ok) {
    set_error(&p.ctl->err, QE_ERR_TIMEOUT);
    misc->abort = 1;
    return;
  }
  const int ms0 = misc->mis_d[k][0], ms1 = misc->mis_d[k][1];
  // batches of 8 rows: ri = b0 + nwk * i, one transposed reduction each
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
}

__global__ void __launch_bounds__(kFusedThreads, 1) qe_fused_layer_kernel(const FusedParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const FusedGeometry& g = p.g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int H = p.H, E = p.E, K = p.K, I = p.I;
  const uint64_t deadline = gtimer() + p.budget_ns;
  const FusedCta t = fused_cta(H, I, G, cta);
  const bool given = p.given_idx != nullptr;

  FusedMisc* misc = (FusedMisc*)(smem + g.off_misc);
  volatile int* abort_flag = &misc->abort;
  uint64_t* bars = (uint64_t*)(smem + g.off_bar);
  float* xn_s = (float*)(smem + g.off_xn);      // raw x, then xn; pieces swizzled per chunk (xswz)
  float* gred = (float*)(smem + g.off_gred);    // [K*np_max][nq][2] quarter sums
  float* ycomb = (float*)(smem + g.off_ycomb);  // [K][no_max]
  WsControl* ctl = p.ctl;

  unsigned epoch = 0;
  if (tid == 0) {
    epoch = ld_relaxed_u32(&ctl->epoch);  // used once the router loads are in flight
    misc->abort = 0;
    for (int b = 0; b < g.nbar; ++b) mbar_init(&bars[b], 1);
    fence_mbar_init();
    QE_TRACE(kTrStart);
  }
  if (tid < kMaxK) misc->hamax[tid] = 0u;

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
          const int f = tid + s * kFusedThreads;
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
      const int f = tid + s * kFusedThreads;
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
    for (int r0 = 0; r0 < nrows; r0 += 4) {
      if (r0 > 0) load_rows(r0);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        double a = 0.0;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          a = fma((double)wv[m][s].x, xg[s][0], a);
          a = fma((double)wv[m][s].y, xg[s][1], a);
          a = fma((double)wv[m][s].z, xg[s][2], a);
          a = fma((double)wv[m][s].w, xg[s][3], a);
        }
        if (r0 + m < nrows) {  // uniform over the CTA
          a = warp_sum_d(a);
          if (lane == 0) misc->rpart[r0 + m][warp] = a;
        }
      }
    }
    ss = warp_sum_d(ss);
    if (lane == 0) misc->redd[warp] = ss;
  }
  if (tid == 0) misc->tag = 0x80000000u | ((epoch + 1u) & 0x7FFFFFFFu);
  __syncthreads();
  if (tid == 0) QE_TRACE(kTrRouter);
  const unsigned tag = misc->tag;
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
    st_rec2(&p.rec_logit[2 * e], rec_word((uint32_t)key, tag), rec_word((uint32_t)(key >> 32), tag));
  }
  // RMSNorm pass 2 (fp32 suffices: xn feeds the expert matvecs, not the
  // routing) and max |xn|
  {
    const float rinv_f = (float)rinv;
    float amax = 0.f;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int f = tid + s * kFusedThreads;
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
    if (lane == 0) misc->redf[warp] = amax;
  }

  // ---------------------------------------------------------------- top-K
  // Thread t polls the records of experts t and t + 512 and stages their
  // keys in the expert slots (unused until the copies are issued); warp 0
  // then takes the top K in K rounds: each lane scans its keys (experts
  // lane, lane + 32, ...) for the largest one not yet taken, and a warp
  // arg-max picks the winner (equal keys: the lower expert index).
  unsigned long long* keys = (unsigned long long*)(smem + g.off_gu);  // [E]
  if (!given) {
    const unsigned iA = (unsigned)tid, iB = (unsigned)(tid + kFusedThreads);
    const bool hasA = (int)iA < E, hasB = (int)iB < E;
    const unsigned long long* const rp[2] = {hasA ? &p.rec_logit[2 * iA] : nullptr,
                                             hasB ? &p.rec_logit[2 * iB] : nullptr};
    unsigned long long lo[2], hi[2];
    if (!poll_rec2<2>(rp, tag, deadline, abort_flag, lo, hi)) {
      set_error(&ctl->err, QE_ERR_TIMEOUT);
      misc->abort = 1;
    }
    if (hasA) keys[iA] = ((unsigned long long)rec_val(hi[0]) << 32) | rec_val(lo[0]);
    if (hasB) keys[iB] = ((unsigned long long)rec_val(hi[1]) << 32) | rec_val(lo[1]);
    if (tid == 0) QE_TRACE(kTrLogits);
  }
  __syncthreads();
  if (warp == 0 && !*abort_flag) {
    if (given) {
      // routing decided beforehand: take its experts and weights as they are
      if (lane < K) {
        const int e = p.given_idx[lane];
        misc->idx[lane] = e;
        misc->wk[lane] = p.given_w[lane];
      }
    } else {
      if (lane == 0) QE_TRACE(kTrPolledAll);
      unsigned taken = 0;  // bit j: expert lane + 32 j is selected
      for (int k = 0; k < K; ++k) {
        unsigned bi = 0xffffffffu;
        unsigned long long bk = 0;
        for (int j = 0, e = lane; e < E; ++j, e += 32) {
          const unsigned long long v = keys[e];
          if (!(taken >> j & 1u) && (bi == 0xffffffffu || v > bk)) {
            bk = v;
            bi = (unsigned)e;
          }
        }
        const unsigned win = warp_argmax_key(bk, bi);
        if (bi != 0xffffffffu && bi == win) {
          misc->idx[k] = (int)win;
          misc->selkey[k] = bk;
          taken |= 1u << ((win - lane) / 32);
        }
      }
      if (lane == 0) QE_TRACE(kTrRounds);
      __syncwarp();
      // renormalised softmax over the K kept logits (sum in k order)
      const double lmax = dkey_inv(misc->selkey[0]);
      const float ev = lane < K ? expf((float)(dkey_inv(misc->selkey[lane]) - lmax)) : 0.0f;
      float s = 0.0f;
      for (int k = 0; k < K; ++k) s += __shfl_sync(0xffffffffu, ev, k);
      if (lane < K) misc->wk[lane] = ev / s;
    }
    __syncwarp();
    if (lane == 0) QE_TRACE(kTrMerged);
    if (lane < K) {
      const int e = misc->idx[lane];
      if (cta == 0 && p.topk_idx) p.topk_idx[lane] = e;
      if (cta == 0 && p.topk_w) p.topk_w[lane] = misc->wk[lane];
      qe_expert ex{};
      bool ok = e >= 0 && e < E;
      if (ok) {
        ex = p.experts[e];
        ok = expert_ok(ex);
      }
      if (!ok) {
        set_error(&ctl->err, QE_ERR_INVALID_ARG);
        misc->abort = 1;
      }
      misc->ex[lane] = ex;
      const ExpertAddr a = expert_addr(ex);
      misc->ea[lane] = a;
      misc->mis_gu[lane][0] = run_misalign(a.gs, t.r_lo, H / 32);
      misc->mis_gu[lane][1] = run_misalign(a.gb, t.r_lo, H / 32);
      misc->mis_gu[lane][2] = run_misalign(a.us, t.r_lo, H / 32);
      misc->mis_gu[lane][3] = run_misalign(a.ub, t.r_lo, H / 32);
      misc->mis_d[lane][0] = run_misalign(a.ds, t.o_lo, I / 32);
      misc->mis_d[lane][1] = run_misalign(a.db, t.o_lo, I / 32);
      // arm this expert's two mbarriers with the bytes their copies bring
      if (ok) {
        const uint32_t ngu = fused_bar_bytes(g, H, I, K, t, misc->ea, bar_gu(lane));
        const uint32_t nd = fused_bar_bytes(g, H, I, K, t, misc->ea, bar_down(K, lane));
        if (ngu) mbar_arrive_expect_tx(&bars[bar_gu(lane)], ngu);
        if (nd) mbar_arrive_expect_tx(&bars[bar_down(K, lane)], nd);
      }
    }
    if (lane == 0) {
      float m = 0.f;
      for (int w = 0; w < kWarps; ++w) m = fmaxf(m, misc->redf[w]);
      misc->Ex = fixed_scale_exponent(m);
      misc->xK = pow2f(misc->Ex - 22);
      int ub = misc->ex[0].gate.bits;
      for (int k = 1; k < K; ++k)
        if (misc->ex[k].gate.bits != ub) ub = 0;
      misc->ubits = ub;
    }
  }
  // the keys' generic stores and loads come before the bulk copies' writes
  // into the same shared memory
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  if (tid == 0) QE_TRACE(kTrTopK);

  // ------------------------------------------------------- issue the copies
  // Every warp first copies scale/bias runs with cp.async (so they are ahead
  // of the bulk traffic), then warp k < K issues expert k's bulk row copies:
  // gate and up rows, and, after every such warp has issued those, its down
  // rows.  The CTA barrier below waits for the scale/bias runs.
  bool issued = false;
  if (!*abort_flag) {
    issued = true;
    const uint64_t pol = policy_evict_first();
    // run r = 6k + u: u < 4 gate/up scale/bias segment u, u = 4, 5 down scales, biases
    for (int r = warp; r < 6 * K; r += kWarps) {
      const int k = r / 6, u = r - 6 * k;
      if (u < 4 ? t.np > 0 : t.no > 0) {
        const FusedCopy c =
            fused_expert_copy(g, H, I, K, t, k, misc->ea[k], u < 4 ? 2 + u : gu_copies(t) + u - 3);
        const unsigned char* src = (const unsigned char*)(uintptr_t)c.src;
        for (uint32_t o = 16u * lane; o < c.bytes; o += 512u) cp_async16(smem + c.dst + o, src + o, pol);
      }
    }
    cp_async_commit();
    if (warp < K) {
      const ExpertAddr& a = misc->ea[warp];
      if (lane < 2 && t.np > 0) {
        const FusedCopy c = fused_expert_copy(g, H, I, K, t, warp, a, lane);
        bulk_g2s(smem + c.dst, (const void*)(uintptr_t)c.src, c.bytes, &bars[c.bar], pol);
      }
      named_barrier(1, 32 * K);
      if (lane == 0 && t.no > 0) {
        const FusedCopy c = fused_expert_copy(g, H, I, K, t, warp, a, gu_copies(t));
        bulk_g2s(smem + c.dst, (const void*)(uintptr_t)c.src, c.bytes, &bars[c.bar], pol);
      }
      if (tid == 0) QE_TRACE(kTrIssued);
    }
    cp_async_wait<0>();
  }
  __syncthreads();

  // ------------------------------------------------------------- gate/up
  if (issued && warp < g.nq * g.nrg && t.np > 0) {
    const int ub = misc->ubits;
    if (ub == 4) gateup_phase<4>(p, t, misc, bars, xn_s, gred, smem, deadline, warp, lane);
    else if (ub == 2) gateup_phase<2>(p, t, misc, bars, xn_s, gred, smem, deadline, warp, lane);
    else gateup_phase<0>(p, t, misc, bars, xn_s, gred, smem, deadline, warp, lane);
  }
  __syncthreads();
  if (tid == 0) QE_TRACE(kTrGateUp);
  // h = silu(g) * u of this CTA's row pairs, then this CTA's h flag
  if (issued && !*abort_flag) {
    for (int P = tid; P < K * t.np; P += kFusedThreads) {
      float gs = 0.f, us = 0.f;
      for (int q = 0; q < g.nq; ++q) {
        gs += gred[(P * g.nq + q) * 2];
        us += gred[(P * g.nq + q) * 2 + 1];
      }
      const float hv = gs / (1.0f + expf(-gs)) * us;
      const int k = P / t.np, j = P - k * t.np;
      st_rec(&p.rec_h[(size_t)k * I + t.r_lo + j], rec_word(__float_as_uint(hv), tag));
    }
  }

  // ------------------------------------------------ stage all of h
  // This CTA's done record goes out after its h records (same threads'
  // stores, behind a barrier); thread c < G polls CTA c's done record, then
  // every thread reads its share of h (two records per 16-byte load) into
  // the gate/up slots (free by now), re-polling any record still stale, and
  // the CTA finds max |h_k| itself.
  float* hst = (float*)(smem + g.off_gu);  // [K][I], 16-byte pieces swizzled per 32-column chunk (xswz)
  if (issued && !*abort_flag) {
    __syncthreads();
    if (tid == 0) st_rec(&p.rec_done[kDoneStride * cta], rec_word(0u, tag));
    bool ok = true;
    if (tid < G) {
      unsigned long long w = ld_rec(&p.rec_done[kDoneStride * tid]);
      for (unsigned spins = 0; rec_tag(w) != tag; ++spins) {
        if (*abort_flag || ((spins & 7u) == 7u && gtimer() > deadline)) {
          ok = false;
          break;
        }
        w = ld_rec(&p.rec_done[kDoneStride * tid]);
      }
    }
    if (!ok) {
      set_error(&ctl->err, QE_ERR_TIMEOUT);
      misc->abort = 1;
    }
    __syncthreads();
    if (tid == 0) QE_TRACE(kTrHPolled);
    if (!*abort_flag) {
      const int npair = K * I / 2;
      for (int b0 = 0; b0 < npair; b0 += 4 * kFusedThreads) {
        const unsigned long long* rp[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int q = b0 + tid + m * kFusedThreads;
          rp[m] = q < npair ? &p.rec_h[2 * q] : nullptr;
        }
        unsigned long long a[4], b[4];
        ok = poll_rec2<4>(rp, tag, deadline, abort_flag, a, b) && ok;
        float mv[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int q = b0 + tid + m * kFusedThreads;
          float2 v = make_float2(0.f, 0.f);
          if (q < npair) {
            v = make_float2(__uint_as_float(rec_val(a[m])), __uint_as_float(rec_val(b[m])));
            *(float2*)(hst + xswz(2 * q)) = v;
          }
          mv[m] = fmaxf(fabsf(v.x), fabsf(v.y));
        }
        // the 32 lanes of a warp hold 64 consecutive values of one expert for
        // each m: one transposed max over the four
        const float am = warp_reduce_rows_max<4>(mv, lane);
        const int m = reduced_row_of_lane<4>(lane);
        const int q0 = b0 + warp * 32 + m * kFusedThreads;
        if (lane == lane_of_reduced_row<4>(m) && q0 < npair) atomicMax(&misc->hamax[(2 * q0) / I], __float_as_uint(am));
      }
      if (!ok) {
        set_error(&ctl->err, QE_ERR_TIMEOUT);
        misc->abort = 1;
      }
    }
  }
  __syncthreads();
  if (tid < K) {
    const int Eh = fixed_scale_exponent(__uint_as_float(misc->hamax[tid]));
    misc->hexp[tid] = Eh;
    misc->hK[tid] = pow2f(Eh - 22);
  }
  __syncthreads();
  if (tid == 0) QE_TRACE(kTrHStaged);

  // ------------------------------------------------------------------ down
  // warp w: expert k = w % K, its owned rows wi, wi + nwk, ... (wi = w / K)
  if (issued && !*abort_flag && t.no > 0 && warp < K * (kWarps / K)) {
    if (misc->ex[warp % K].down.bits == 4) down_phase<4>(p, t, misc, bars, hst, ycomb, smem, deadline, warp, lane);
    else down_phase<2>(p, t, misc, bars, hst, ycomb, smem, deadline, warp, lane);
  }
  __syncthreads();
  if (tid == 0) QE_TRACE(kTrDown);

  // ----------------------------------------------- combine of owned rows
  if (issued && !*abort_flag) {
    for (int i = tid; i < t.no; i += kFusedThreads) {
      const int r = t.o_lo + i;
      float acc = 0.f;
      for (int k = 0; k < K; ++k) acc += misc->wk[k] * ycomb[k * g.no_max + i];
      if (p.add_residual) acc += load_x(p, r);
      p.out[r] = acc;
    }
  }
  // no copy may still be landing when the CTA exits (they all have, unless
  // a wait gave up): wait for every armed mbarrier, bounded
  if (issued) {
    volatile int no_abort = 0;
    const uint64_t dl2 = gtimer() + p.budget_ns;
    for (int b = tid; b < g.nbar; b += kFusedThreads)
      if (fused_bar_bytes(g, H, I, K, t, misc->ea, b)) mbar_wait(&bars[b], 0, dl2, &no_abort);
  }
  __syncthreads();
  if (tid == 0) {
    // every CTA has read the epoch (CTA 0 saw all done records, or gave up
    // after the wait budget): advance it for the next launch
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
  if (K < 1 || K > kMaxK || E > 2 * kFusedThreads) return QE_ERR_UNSUPPORTED;
  if (sms < 1 || sms > kMaxGrid || E > kRouterRows * sms) return QE_ERR_UNSUPPORTED;
  g.grid = sms;
  g.nq = (H / 32 + 31) / 32;
  g.nrg = kWarps / g.nq;
  g.np_max = (I + sms - 1) / sms;
  g.no_max = (H + sms - 1) / sms;
  g.gu_row = H / 2;
  g.gu_sc = align_up(g.np_max * (H / 32) + 30, 16);
  g.gu_bytes = 2 * g.np_max * g.gu_row + 4 * g.gu_sc;
  g.d_row = I / 2;
  g.d_sc = align_up(g.no_max * (I / 32) + 30, 16);
  g.d_bytes = g.no_max * g.d_row + 2 * g.d_sc;
  g.nbar = 2 * K;
  int off = 0;
  g.off_misc = off; off = align_up(off + (int)sizeof(FusedMisc), 128);
  g.off_bar = off; off = align_up(off + 8 * g.nbar, 128);
  g.off_xn = off; off = align_up(off + 4 * H, 128);
  g.off_xsum = off; off = align_up(off + 4 * (H / 32), 128);
  g.off_gred = off; off = align_up(off + 4 * 2 * g.nq * K * g.np_max, 128);
  g.off_ycomb = off; off = align_up(off + 4 * K * g.no_max, 128);
  g.off_gu = off;
  // the top-K keys (8 bytes per expert) and, later, all of h are staged here too
  int gu_total = K * g.gu_bytes;
  if (gu_total < 4 * K * I) gu_total = 4 * K * I;
  if (gu_total < 8 * E) gu_total = 8 * E;
  off = align_up(off + gu_total, 128);
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
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
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
                                          const int* bits, const uint64_t* seg /* [K][9] */, int* geom /* [24] */,
                                          long long* copies /* [max_copies][4] */, int max_copies,
                                          long long* reads /* [max_reads][6] */, int max_reads) {
  using namespace qe;
  FusedGeometry g;
  const int rc = fused_geometry(H, E, K, I, sms, smem_optin, &g);
  if (rc != QE_OK) return rc;
  const int gv[24] = {g.grid, g.nq, g.nrg, g.np_max, g.no_max, g.gu_row, g.gu_sc, g.gu_bytes,
                      g.d_row, g.d_sc, g.d_bytes, g.nbar, g.off_xn, g.off_xsum, g.off_misc, g.off_bar,
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
