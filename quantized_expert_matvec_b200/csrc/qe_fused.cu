// qe_fused.cu -- the single-token layer step as ONE persistent kernel:
// RMSNorm -> router (fp64) -> top-K -> gate/up dequant-matvec + SwiGLU ->
// down dequant-matvec -> weighted combine (+ residual).
//
// One CTA per SM (16 warps), launched cooperatively so all CTAs are resident.
//
// Routing: CTA c owns router rows c, c+G, ...; each warp covers one 1/16
// column slice of them, and the same x loads feed the RMSNorm sum of squares
// (the router dot does not depend on the norm scale).  After a grid-wide
// counter, every CTA ranks all E logits itself: per-warp top-K candidates by
// redux reductions, then one merge.
//
// Expert phase.  Gate/up: the selected experts' rows are cut into items of
// RB rows of gate and of up; the four 4-warp groups take items in turn and
// each warp of a group copies (16-byte cp.async into the group's ring, one
// copy group per item) and dequantises one column quarter of every row,
// keeping the x' of its columns in registers; the four quarter sums meet in
// shared memory behind a named barrier, and h = silu(g) * u goes to global
// memory.  Each warp then loads its first down rows into registers.  A second
// grid-wide counter waits for every CTA's h rows; every CTA then reads all
// of h, finds max |h_k| itself and stages h_k in x' form in shared memory.
// Down: warp w works on expert w % K and computes full rows (RC-row blocks of
// the output rows this CTA owns); the CTA combines its rows (+ residual).
// All waits are bounded (QE_ERR_TIMEOUT).  The grid counters only grow: each
// launch adds its grid size, and a CTA's arrival ticket gives the count it
// waits for, so nothing has to be reset between launches.
#include <math.h>

#include <type_traits>

#include "qe_device.cuh"

namespace qe {

constexpr int kWarps = 16;
constexpr int kGroups = 4;  // 4-warp groups of the gate/up phase
constexpr int kRB = 4;      // rows of gate (and of up) in one gate/up item
constexpr int kRC = 4;      // rows of one down block
constexpr int kFusedThreads = kWarps * 32;
constexpr int kRouterRows = 8;  // router rows one CTA owns at most: E <= 8 * grid
constexpr int kRouterBatch = 4; // router rows accumulated together
constexpr int kChunkMax = 8;    // 32-column chunks one warp converts: H <= 8 * 32 * 16

struct FusedMisc {
  int abort;
  float xK;
  int idx[kMaxK];
  float wk[kMaxK];
  qe_expert ex[kMaxK];
  float hK[kMaxK];
  int hexp[kMaxK];  // vector exponent of h_k (x' form of the down input)
  unsigned long long route_target;  // routing counter value that completes this launch
  unsigned cand_idx[kWarps][kMaxK];
  unsigned long long cand_key[kWarps][kMaxK];
  double cand_val[kWarps][kMaxK];
  double lsel[kMaxK];
  float gred[kGroups][2][4][2 * kRB];  // gate/up partial sums [group][item parity][quarter][row]
  unsigned hamax[kMaxK];               // max |h_k| of this CTA's rows, as float bits
  unsigned long long t_lastC;
  float redf[kWarps];
  double redd[kWarps];
  double rpart[kRouterRows][kWarps];
};

// Optional phase trace: globaltimer stamps per CTA (qe_trace_fused).
enum {
  kTrStart, kTrRouterDone, kTrRouteBarrier, kTrTopK, kTrIssuedB, kTrIssuedC, kTrFirstB, kTrLastB,
  kTrHFirst, kTrHLast, kTrLastC, kTrEnd
};
#define QE_TRACE(slot) \
  do { if (p.trace) p.trace[(size_t)blockIdx.x * 64 + (slot)] = gtimer(); } while (0)

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

// Order-preserving map of a double onto an unsigned 64-bit key.
static __device__ __forceinline__ unsigned long long dkey(double d) {
  const unsigned long long u = (unsigned long long)__double_as_longlong(d);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
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

// ------------------------------------------------------- gate/up (groups)
// A gate/up item is kRB rows of gate and kRB rows of up of one expert.  The
// four warps of a group split the columns into quarters; warp qd copies and
// dequantises quarter qd of every row, so the x' of its columns stays in
// registers.  Slot layout: packed words of (quarter, matrix, row) at
// ((qd*2 + mat)*kRB + rr) * H/8, then per warp four segments [gate s | gate
// b | up s | up b] of sseg bytes at kRB*H + qd*4*sseg.  When H is a multiple
// of 2048 a segment holds only the quarter's groups of each row (H/128 bytes
// a row); otherwise it holds whole rows.

struct GateUpCtx {
  int H, gpr, nlc;  // nlc: 32-column lane chunks per quarter
  int qsc;          // segments hold quarter rows
  int sseg;         // bytes of one segment
  int srow;         // entries (uint16) per row in a segment
};

static __device__ __forceinline__ GateUpCtx make_gateup_ctx(int H) {
  GateUpCtx c;
  c.H = H;
  c.gpr = H / kGroup;
  c.nlc = H / 128;
  c.qsc = (H % 2048) == 0;
  c.srow = c.qsc ? H / 256 : c.gpr;
  c.sseg = kRB * c.srow * 2;
  return c;
}

static __device__ __forceinline__ void issue_gateup(const qe_expert& ex, int r0, unsigned char* slot, int qd,
                                                    const GateUpCtx& c, int lane, uint64_t pol) {
  const int bits = ex.gate.bits;
  const uint32_t qb = (uint32_t)(c.H * bits / 32);  // bytes of one row quarter
  const size_t rowb = (size_t)c.H * bits / 8;
  const unsigned char* gsrc = (const unsigned char*)ex.gate.wq + (size_t)r0 * rowb + qd * qb;
  const unsigned char* usrc = (const unsigned char*)ex.up.wq + (size_t)r0 * rowb + qd * qb;
#pragma unroll
  for (int rr = 0; rr < kRB; ++rr) {
    warp_copy_async(slot + ((qd * 2 + 0) * kRB + rr) * (c.H / 8), gsrc + rr * rowb, qb, lane, pol);
    warp_copy_async(slot + ((qd * 2 + 1) * kRB + rr) * (c.H / 8), usrc + rr * rowb, qb, lane, pol);
  }
  unsigned char* sd = slot + kRB * c.H + qd * 4 * c.sseg;
  const uint16_t* segsrc[4] = {ex.gate.scales, ex.gate.biases, ex.up.scales, ex.up.biases};
  if (c.qsc) {
    const int npc = c.H / 2048;  // 16-byte pieces of one quarter row
    const int per_seg = kRB * npc;
    for (int u = lane; u < 4 * per_seg; u += 32) {
      const int seg = u / per_seg, rem = u - seg * per_seg;
      const int rr = rem / npc, pc = rem - rr * npc;
      const unsigned char* src = (const unsigned char*)(segsrc[seg] + (size_t)(r0 + rr) * c.gpr + qd * (c.H / 256)) + pc * 16;
      cp_async16(sd + seg * c.sseg + rr * (c.H / 128) + pc * 16, src, pol);
    }
  } else {
#pragma unroll
    for (int seg = 0; seg < 4; ++seg)
      warp_copy_async(sd + seg * c.sseg, segsrc[seg] + (size_t)r0 * c.gpr, (uint32_t)c.sseg, lane, pol);
  }
  cp_async_commit();
}

// Partial sums of the 2*kRB rows over this warp's quarter; returns the
// warp-reduced value (row reduced_row_of_lane<2*kRB>(lane)).
template <int BITS>
static __device__ __forceinline__ float gateup_partial(const unsigned char* slot, int qd, const GateUpCtx& c,
                                                       const float* xp, const float* xs_sum, float xK,
                                                       float2 (&xs)[16], bool xs_cached, int lane) {
  float yv[2 * kRB];
#pragma unroll
  for (int i = 0; i < 2 * kRB; ++i) yv[i] = 0.f;
  const uint16_t* sc = (const uint16_t*)(slot + kRB * c.H + qd * 4 * c.sseg);
  const int segs = c.sseg / 2;  // uint16 entries per segment
  const int goff = c.qsc ? qd * (c.H / 256) : 0;
  for (int l = lane; l < c.nlc; l += 32) {
    const int lc = qd * c.nlc + l;  // 32-column chunk of the full row
    if (!xs_cached) load_xs32(xp, lc, xs);
    const int gi = (lc >> 1) - goff;
    const float xsum = xs_sum[lc];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
#pragma unroll
      for (int rr = 0; rr < kRB; ++rr) {
        const unsigned char* wp = slot + ((qd * 2 + m) * kRB + rr) * (c.H / 8);
        float2 a;
        if (BITS == 4) a = dot32_q4(*(const ulonglong2*)(wp + l * 16), xs, make_float2(0.f, 0.f));
        else a = dot32_q2(*(const unsigned long long*)(wp + l * 8), xs, make_float2(0.f, 0.f));
        const float sv = bf16f(sc[(2 * m) * segs + rr * c.srow + gi]);
        const float bv = bf16f(sc[(2 * m + 1) * segs + rr * c.srow + gi]);
        yv[m * kRB + rr] += sv * xK * (a.x + a.y) + bv * xsum;
      }
    }
  }
  return warp_reduce_rows<2 * kRB>(yv, lane);
}

// ------------------------------------------------------------ down (warps)
// A warp computes full rows of one expert's down matrix: RC-row blocks of the
// output blocks this CTA owns, up to 8 rows per batch; batch row i is row
// (i % RC) of block wi + nwk * (i / RC).  Each lane takes one 32-column chunk
// of every row; the packed words and the scale/bias pair of that chunk are
// loaded into registers (before h is ready, for the first chunk).
struct DownRows {
  ulonglong2 w[8];  // 4-bit: words 0..3; 2-bit: words 0..1 in .x
  // bf16 scale and bias, kept as loaded: combining them would make the warp
  // wait for the loads here instead of at their first use after the h barrier
  unsigned short sc[8], bi[8];
};

static __device__ __forceinline__ int down_row(int cta, int G, int RC, int wi, int nwk, int ri) {
  const int blk = ri / RC;
  return (cta + G * (wi + nwk * blk)) * RC + (ri - blk * RC);
}

static __device__ __forceinline__ void down_load(const qe_qmat& d, int cta, int G, int RC, int wi, int nwk, int b0,
                                                 int nr, int I, int lc, DownRows& R) {
  const int gpr = I / kGroup;
  const size_t rowb = (size_t)I * d.bits / 8;
  const int g = lc >> 1;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i < nr) {
      const int row = down_row(cta, G, RC, wi, nwk, b0 + i);
      const unsigned char* rp = (const unsigned char*)d.wq + (size_t)row * rowb;
      if (d.bits == 4) R.w[i] = __ldcs((const ulonglong2*)rp + lc);
      else R.w[i].x = __ldcs((const unsigned long long*)rp + lc);
      R.sc[i] = __ldg(d.scales + (size_t)row * gpr + g);
      R.bi[i] = __ldg(d.biases + (size_t)row * gpr + g);
    }
  }
}

template <int BITS>
static __device__ __forceinline__ void down_accum(const DownRows& R, int nr, int lc, const float* hpk,
                                                  const float* hsk, float hK, float (&yv)[8]) {
  float2 xs[16];
  if (BITS == 4) load_xs32_q4(hpk, lc, xs);
  else load_xs32_q2(hpk, lc, xs);
  const float xsum = hsk[lc];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i < nr) {
      const float2 a = BITS == 4 ? dot32_q4(R.w[i], xs, make_float2(0.f, 0.f))
                                 : dot32_q2(R.w[i].x, xs, make_float2(0.f, 0.f));
      yv[i] += bf16f(R.sc[i]) * hK * (a.x + a.y) + bf16f(R.bi[i]) * xsum;
    }
  }
}

__global__ void __launch_bounds__(kFusedThreads, 1) qe_fused_layer_kernel(const FusedParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const FusedGeometry& g = p.g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int H = p.H, E = p.E, K = p.K, I = p.I;
  const uint64_t deadline = gtimer() + p.budget_ns;

  FusedMisc* misc = (FusedMisc*)(smem + g.off_misc);
  volatile int* abort_flag = &misc->abort;
  float* xp4 = (float*)(smem + g.off_xp4);
  float* xp2 = (float*)(smem + g.off_xp2);
  float* xsum = (float*)(smem + g.off_xs);
  float* hp = (float*)(smem + g.off_hp);    // [K][I]
  float* hsum = (float*)(smem + g.off_hs);  // [K][I/32]
  float* ycomb = (float*)(smem + g.off_ycomb);
  WsControl* ctl = p.ctl;

  if (tid == 0) {
    misc->abort = 0;
    misc->t_lastC = 0;
    QE_TRACE(kTrStart);
    if (p.trace) p.trace[(size_t)cta * 64 + 12] = clock64();
  }
  if (tid < kMaxK) {
    misc->hexp[tid] = 0;
  }

  // ------------------------------------------------------------- routing
  // The router dot s_e = sum_c W[e,c] x_c gamma_c does not depend on the
  // RMSNorm scale, so it runs on the same loads as the sum of squares; the
  // logit is s_e * rinv (+ offset_e), all in fp64.  Warp w covers the column
  // slice [w*S, (w+1)*S), S = H/16, of each router row its CTA owns; the 16
  // slice sums are added in slice order.
  const bool given = p.given_idx != nullptr;
  const int nrows = (!given && E > cta) ? (E - cta + G - 1) / G : 0;
  {
    const int S = H / kWarps;
    double ss = 0.0;
    for (int r0 = 0; r0 < (nrows > 0 ? nrows : 1); r0 += kRouterBatch) {
      double acc[kRouterBatch];
#pragma unroll
      for (int m = 0; m < kRouterBatch; ++m) acc[m] = 0.0;
      for (int i = lane; i < S / 4; i += 32) {
        const int c = warp * S + 4 * i;
        float4 wv[kRouterBatch];
#pragma unroll
        for (int m = 0; m < kRouterBatch; ++m)
          if (r0 + m < nrows) wv[m] = __ldg((const float4*)(p.router_w + (size_t)(cta + G * (r0 + m)) * H + c));
        double xv[4];
        load_x4(p, c, xv);
        if (r0 == 0) {
          ss += xv[0] * xv[0] + xv[1] * xv[1] + xv[2] * xv[2] + xv[3] * xv[3];
          // raw x for RMSNorm pass 2 (the x' buffer is free until then)
          *(float4*)(xp4 + c) = make_float4((float)xv[0], (float)xv[1], (float)xv[2], (float)xv[3]);
        }
        if (p.gamma) {
          const float4 gm = *(const float4*)(p.gamma + c);
          xv[0] *= (double)gm.x; xv[1] *= (double)gm.y; xv[2] *= (double)gm.z; xv[3] *= (double)gm.w;
        }
#pragma unroll
        for (int m = 0; m < kRouterBatch; ++m) {
          if (r0 + m < nrows) {
            double a = acc[m];
            a = fma((double)wv[m].x, xv[0], a);
            a = fma((double)wv[m].y, xv[1], a);
            a = fma((double)wv[m].z, xv[2], a);
            a = fma((double)wv[m].w, xv[3], a);
            acc[m] = a;
          }
        }
      }
#pragma unroll
      for (int m = 0; m < kRouterBatch; ++m) {
        if (r0 + m < nrows) {
          const double t = warp_sum_d(acc[m]);
          if (lane == 0) misc->rpart[r0 + m][warp] = t;
        }
      }
    }
    if (tid == 0) QE_TRACE(56);
    ss = warp_sum_d(ss);
    if (lane == 0) misc->redd[warp] = ss;
  }
  __syncthreads();
  if (tid == 0) QE_TRACE(57);
  double rinv;
  {
    double tot = 0.0;
    for (int w = 0; w < kWarps; ++w) tot += misc->redd[w];
    rinv = 1.0 / sqrt(tot / (double)H + (double)p.eps);
  }
  if (tid < nrows) {
    double sl = 0.0;
    for (int w = 0; w < kWarps; ++w) sl += misc->rpart[tid][w];
    const int e = cta + G * tid;
    p.logit_part[e] = sl * rinv + (p.offset ? (double)p.offset[e] : 0.0);
  }
  // RMSNorm pass 2 in 32-column chunks (lane = column): xn stays in
  // registers until the vector exponent of x' is known
  // (fp32 suffices here: xn feeds the expert matvecs, not the routing)
  float xnv[kChunkMax];
  {
    const float rinv_f = (float)rinv;
    float amax = 0.f;
#pragma unroll
    for (int q = 0; q < kChunkMax; ++q) {
      const int ch = warp + kWarps * q;
      xnv[q] = 0.f;
      if (ch < H / 32) {
        const int c = ch * 32 + lane;
        const float gm = p.gamma ? p.gamma[c] : 1.0f;
        xnv[q] = xp4[c] * rinv_f * gm;
        amax = fmaxf(amax, fabsf(xnv[q]));
      }
    }
    amax = warp_max(amax);
    if (lane == 0) misc->redf[warp] = amax;
  }
  if (tid == 0) QE_TRACE(58);
  __syncthreads();
  if (tid == 0) {
    QE_TRACE(kTrRouterDone);
    if (!given) {
      // the release publishes this CTA's logits; the ticket names the count
      // that completes this launch's arrivals (a CTA told to skip its
      // arrival, a test hook, waits for the same count and times out too)
      const unsigned long long t =
          cta != p.skip_cta ? atom_add_release_u64(&ctl->route_ctr, 1ull) : ld_acquire_u64(&ctl->route_ctr);
      misc->route_target = (t / (unsigned)G + 1ull) * (unsigned)G;
    }
  }
  {
    float m = 0.f;
    for (int w = 0; w < kWarps; ++w) m = fmaxf(m, misc->redf[w]);
    const int Ex = xscale_exponent(m);
    if (tid == 0) misc->xK = acc_scale(Ex);
    {
      // the chunk sums of this warp's kChunkMax chunks in one transposed
      // reduction (chunks past the end hold 0)
      float sv[kChunkMax];
#pragma unroll
      for (int q = 0; q < kChunkMax; ++q) sv[q] = xnv[q];
      const float sm = warp_reduce_rows<kChunkMax>(sv, lane);
      const int row = reduced_row_of_lane<kChunkMax>(lane);
      const int ch = warp + kWarps * row;
      if (lane == lane_of_reduced_row<kChunkMax>(row) && ch < H / 32) xsum[ch] = sm;
    }
#pragma unroll
    for (int q = 0; q < kChunkMax; ++q) {
      const int ch = warp + kWarps * q;
      if (ch < H / 32) {
        const int c = ch * 32 + lane;
        xp4[swz_q4(c)] = xprime_q4(xnv[q], c, Ex);
        xp2[swz_q2(c)] = xprime_q2(xnv[q], c, Ex);
      }
    }
  }
  if (tid == 0) {
    if (!given && !wait_geq64(&ctl->route_ctr, misc->route_target, deadline, abort_flag)) {
      set_error(&ctl->err, QE_ERR_TIMEOUT);
      misc->abort = 1;
    }
    QE_TRACE(kTrRouteBarrier);
  }
  __syncthreads();

  // ---------------------------------------------------------------- top-K
  // Thread t ranks logits t and t+512.  Each warp finds its own top-K by K
  // rounds of warp_argmax_key (a sorted candidate list, keys and values kept
  // in shared memory); warp 0 then merges the 16 lists, one list per lane.
  if (!given && !*abort_flag) {
    const unsigned iA = (unsigned)tid, iB = (unsigned)(tid + kFusedThreads);
    bool hasA = tid < E, hasB = tid + kFusedThreads < E;
    const double vA = hasA ? __ldcg(&p.logit_part[iA]) : 0.0;
    const double vB = hasB ? __ldcg(&p.logit_part[iB]) : 0.0;
    const unsigned long long kA = dkey(vA), kB = dkey(vB);
    for (int k = 0; k < K; ++k) {
      const bool useA = hasA && (!hasB || kA >= kB);  // equal keys: A has the lower index
      const unsigned bi = (hasA || hasB) ? (useA ? iA : iB) : 0xffffffffu;
      const unsigned win = warp_argmax_key(useA ? kA : kB, bi);
      if (lane == 0) misc->cand_idx[warp][k] = win;
      if (bi != 0xffffffffu && bi == win) {
        misc->cand_key[warp][k] = useA ? kA : kB;
        misc->cand_val[warp][k] = useA ? vA : vB;
        // warm L1 with the candidate's descriptor while the rounds go on
        prefetch_l1(&p.experts[win]);
        prefetch_l1((const unsigned char*)&p.experts[win] + 64);
        if (useA) hasA = false;
        else hasB = false;
      }
    }
  }
  __syncthreads();
  if (warp == 0 && given && !*abort_flag) {
    // routing decided beforehand: take its experts and weights as they are
    if (lane < K) {
      const int e = p.given_idx[lane];
      misc->wk[lane] = p.given_w[lane];
      if (cta == 0 && p.topk_idx) p.topk_idx[lane] = e;
      if (cta == 0 && p.topk_w) p.topk_w[lane] = p.given_w[lane];
      bool ok = e >= 0 && e < E;
      qe_expert ex{};
      if (ok) {
        ex = p.experts[e];
        const int bits = ex.gate.bits;
        ok = (bits == 4 || bits == 2) && desc_ok(ex.gate, bits) && desc_ok(ex.up, bits) && desc_ok(ex.down, bits);
      }
      if (!ok) {
        set_error(&ctl->err, QE_ERR_INVALID_ARG);
        misc->abort = 1;
      }
      misc->idx[lane] = e;
      misc->ex[lane] = ex;
    }
  }
  if (warp == 0 && !given && !*abort_flag) {
    int ptr = 0;
    double myval = 0.0;
    for (int k = 0; k < K; ++k) {
      unsigned bi = 0xffffffffu;
      unsigned long long bk = 0;
      if (lane < kWarps && ptr < K) {
        bi = misc->cand_idx[lane][ptr];
        if (bi != 0xffffffffu) bk = misc->cand_key[lane][ptr];
      }
      const unsigned win = warp_argmax_key(bk, bi);
      if (bi != 0xffffffffu && bi == win) {
        misc->idx[k] = (int)win;
        myval = misc->cand_val[lane][ptr];
        ++ptr;
        misc->lsel[k] = myval;
      }
    }
    __syncwarp();
    // renormalised softmax over the K kept logits (sum in k order); lanes
    // k < K also fetch and check the K expert descriptors
    const double lmax = misc->lsel[0];
    const float ev = lane < K ? expf((float)(misc->lsel[lane] - lmax)) : 0.0f;
    float s = 0.0f;
    for (int k = 0; k < K; ++k) s += __shfl_sync(0xffffffffu, ev, k);
    if (lane < K) {
      misc->wk[lane] = ev / s;
      if (cta == 0 && p.topk_idx) p.topk_idx[lane] = misc->idx[lane];
      if (cta == 0 && p.topk_w) p.topk_w[lane] = misc->wk[lane];
      const qe_expert ex = p.experts[misc->idx[lane]];
      const int bits = ex.gate.bits;
      if (!(bits == 4 || bits == 2) || !desc_ok(ex.gate, bits) || !desc_ok(ex.up, bits) ||
          !desc_ok(ex.down, bits)) {
        set_error(&ctl->err, QE_ERR_INVALID_ARG);
        misc->abort = 1;
      }
      misc->ex[lane] = ex;
    }
  }
  __syncthreads();
  if (tid == 0) QE_TRACE(kTrTopK);

  // ---------------------------------------------------------- expert phase
  const int nBc = g.nB > cta ? (g.nB - cta + G - 1) / G : 0;
  const int own = g.nCB > cta ? (g.nCB - cta + G - 1) / G : 0;
  const int MR = g.max_own * kRC;  // rows of one expert's slice of ycomb
  // down work of this warp: expert k = warp % K, blocks wi, wi + nwk, ...
  const int ck = warp % K, wi = warp / K, nwk = (kWarps - ck + K - 1) / K;
  const int myblocks = wi < own ? (own - wi + nwk - 1) / nwk : 0;

  const qe_qmat dmat = misc->ex[ck].down;
  const int nrow = myblocks * kRC;  // down rows of this warp
  DownRows R;
  if (tid < kMaxK) misc->hamax[tid] = 0u;
  __syncthreads();

  if (!*abort_flag) {
    // ------------------------------------------------ gate/up, 4-warp groups
    const int gr = warp >> 2, qd = warp & 3;
    const int ng = nBc > gr ? (nBc - gr + kGroups - 1) / kGroups : 0;
    unsigned char* gring = smem + g.off_ring + (size_t)gr * g.nslot * g.slot;
    const GateUpCtx cx = make_gateup_ctx(H);
    const uint64_t pol = policy_evict_first();
    // item t of this group is gate/up item gi = cta + G*(gr + 4t) of the
    // grid: expert gi / nIB, rows (gi % nIB) * kRB
    auto item_k = [&](int t, int* r0) {
      const int gi = cta + G * (gr + kGroups * t);
      const int k = gi / g.nIB;
      *r0 = (gi - k * g.nIB) * kRB;
      return k;
    };
    for (int t = 0; t < g.nslot && t < ng; ++t) {
      int r0;
      const int k = item_k(t, &r0);
      issue_gateup(misc->ex[k], r0, gring + (size_t)t * g.slot, qd, cx, lane, pol);
    }
    float2 xs[16];
    int xs_bits = 0;  // bits of the x' form cached in xs (0: none)
    const bool cache = cx.nlc <= 32;  // one lane chunk of the quarter per lane
    int slot_i = 0;
    for (int t = 0; t < ng; ++t) {
      int r0;
      const int k = item_k(t, &r0);
      unsigned char* sl = gring + (size_t)slot_i * g.slot;
      // copy groups committed after this item's: the items already issued ahead
      const int later = (t + g.nslot <= ng ? g.nslot : ng - t) - 1;
      if (later >= 2) cp_async_wait<2>();
      else if (later == 1) cp_async_wait<1>();
      else cp_async_wait<0>();
      __syncwarp();
      if (threadIdx.x == 0 && t < 2) QE_TRACE(59 + 3 * t);  // item t landed (warp 0)
      const int bits = misc->ex[k].gate.bits;
      if (cache && xs_bits != bits && lane < cx.nlc) {
        if (bits == 4) load_xs32_q4(xp4, qd * cx.nlc + lane, xs);
        else load_xs32_q2(xp2, qd * cx.nlc + lane, xs);
      }
      xs_bits = bits;
      const float s = bits == 4 ? gateup_partial<4>(sl, qd, cx, xp4, xsum, misc->xK, xs, cache, lane)
                                : gateup_partial<2>(sl, qd, cx, xp2, xsum, misc->xK, xs, cache, lane);
      float* red = misc->gred[gr][t & 1][qd];
#pragma unroll
      for (int i = 0; i < 2 * kRB; ++i)
        if (lane == lane_of_reduced_row<2 * kRB>(i)) red[i] = s;
      if (threadIdx.x == 0 && t < 2) QE_TRACE(60 + 3 * t);  // item t computed (warp 0)
      named_barrier(1 + gr, 128);
      if (threadIdx.x == 0 && t == 0) QE_TRACE(61);  // group 0 past item 0
      if (qd == 0 && lane < kRB) {
        // lane rr: h of row r0 + rr = silu(g) * u from the four quarter sums
        float gv = 0.f, uv = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          gv += misc->gred[gr][t & 1][q][lane];
          uv += misc->gred[gr][t & 1][q][kRB + lane];
        }
        const float hv = gv / (1.0f + expf(-gv)) * uv;
        p.hbuf[(size_t)k * I + r0 + lane] = hv;  // published once per CTA below
      }
      __syncwarp();
      if (t + g.nslot < ng) {
        int r1;
        const int k1 = item_k(t + g.nslot, &r1);
        issue_gateup(misc->ex[k1], r1, sl, qd, cx, lane, pol);
      }
      if (++slot_i == g.nslot) slot_i = 0;
      if (*abort_flag) break;
    }
    cp_async_wait<0>();  // nothing may still be landing when the CTA exits
    if (lane == 0) QE_TRACE(16 + warp);
    // this warp's first down rows do not depend on h: load them now
    if (nrow > 0 && lane < I / 32) down_load(dmat, cta, G, kRC, wi, nwk, 0, nrow < 8 ? nrow : 8, I, lane, R);
  }

  // ------------------------------------- publish h, wait for every CTA's h
  __syncthreads();
  if (tid == 0) {
    QE_TRACE(kTrLastB);
    if (!*abort_flag) {
      // the release publishes the h rows every thread of this CTA stored
      // before the barrier above
      const unsigned long long t = atom_add_release_u64(&ctl->h_ctr, 1ull);
      if (!wait_geq64(&ctl->h_ctr, (t / (unsigned)G + 1ull) * (unsigned)G, deadline, abort_flag)) {
        set_error(&ctl->err, QE_ERR_TIMEOUT);
        misc->abort = 1;
      }
    }
    QE_TRACE(kTrHFirst);
  }
  __syncthreads();

  // stage h in x' form, all warps: chunk ch of the K*I/32 chunks.  Every CTA
  // loads all of h, so it finds max |h_k| itself (per-warp maxima, then one
  // pass over the warps).  When the chunks fit in one round of 8 per warp the
  // values stay in registers until their exponent is known; otherwise the raw
  // values go through shared memory and are rewritten in x' form in place
  // (the x' layout only permutes values inside a chunk).
  const int per = I / 32, nch = K * per;
  // every CTA reads all of h at once: start each CTA at another chunk so the
  // requests spread over the L2 slices instead of queueing on one
  const int rot = (int)(((unsigned)cta * 37u) % (unsigned)nch);
  // (k, lc) of the 8 chunks of the round of this warp that starts at ch0
  auto round_chunks = [&](int ch0, int (&kk)[8], int (&ll)[8]) {
    int ch = ch0 + rot < nch ? ch0 + rot : ch0 + rot - nch;
    int k = 0;
    while (ch >= per) { ch -= per; ++k; }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      kk[i] = k;
      ll[i] = ch;
      ch += kWarps;
      while (ch >= per) { ch -= per; ++k; }
      while (k >= K) k -= K;  // wrapped past the last expert (rotation)
    }
  };
  const bool one_round = nch <= 8 * kWarps;
  float v[8];  // one round: the values stay here until their exponent is known
  if (!*abort_flag) {
    for (int ch0 = warp; ch0 < nch; ch0 += 8 * kWarps) {
      int kk[8], ll[8];
      round_chunks(ch0, kk, ll);
      // loads issued before any of them is used
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (ch0 + i * kWarps < nch) v[i] = __ldcg(p.hbuf + (size_t)kk[i] * I + ll[i] * 32 + lane);
      // the 8 chunks' sums and maxima in one transposed reduction each
      // (chunks past the end hold 0, which changes neither)
      float sv[8], mv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (ch0 + i * kWarps >= nch) v[i] = 0.f;
        sv[i] = v[i];
        mv[i] = fabsf(v[i]);
        if (!one_round && ch0 + i * kWarps < nch) hp[(size_t)kk[i] * I + ll[i] * 32 + lane] = v[i];
      }
      const float sm = warp_reduce_rows<8>(sv, lane);
      const float am = warp_reduce_rows_max<8>(mv, lane);
      const int row = reduced_row_of_lane<8>(lane);
      if (lane == lane_of_reduced_row<8>(row) && ch0 + row * kWarps < nch) {
        int k = 0, lc = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (i == row) { k = kk[i]; lc = ll[i]; }
        hsum[(size_t)k * per + lc] = sm;
        atomicMax(&misc->hamax[k], __float_as_uint(am));
      }
    }
  }
  __syncthreads();
  if (tid < K) {
    const int Eh = xscale_exponent(__uint_as_float(misc->hamax[tid]));
    misc->hexp[tid] = Eh;
    misc->hK[tid] = acc_scale(Eh);
  }
  __syncthreads();
  if (!*abort_flag) {
    if (one_round) {
      int kk[8], ll[8];
      round_chunks(warp, kk, ll);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (warp + i * kWarps < nch) {
          const int k = kk[i], c = ll[i] * 32 + lane;
          float* hpk = hp + (size_t)k * I;
          if (misc->ex[k].down.bits == 4) hpk[swz_q4(c)] = xprime_q4(v[i], c, misc->hexp[k]);
          else hpk[swz_q2(c)] = xprime_q2(v[i], c, misc->hexp[k]);
        }
      }
    } else {
      // raw values went through shared memory: rewrite each chunk in place
      for (int ch = warp; ch < nch; ch += kWarps) {
        int k = 0, lc = ch;
        while (lc >= per) { lc -= per; ++k; }
        float* hpk = hp + (size_t)k * I;
        const int c = lc * 32 + lane;
        const float x = hpk[c];
        __syncwarp();
        if (misc->ex[k].down.bits == 4) hpk[swz_q4(c)] = xprime_q4(x, c, misc->hexp[k]);
        else hpk[swz_q2(c)] = xprime_q2(x, c, misc->hexp[k]);
      }
    }
  }
  __syncthreads();
  if (tid == 0) QE_TRACE(kTrHLast);

  // -------------------------------------------------------- down, warps
  if (!*abort_flag && nrow > 0) {
    const int k = ck;
    const float* hpk = hp + (size_t)k * I;
    const float* hsk = hsum + (size_t)k * (I / 32);
    const float hK = misc->hK[k];
    float* yk = ycomb + (size_t)k * MR;
    for (int b0 = 0; b0 < nrow; b0 += 8) {
      const int nr = nrow - b0 < 8 ? nrow - b0 : 8;
      float yv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) yv[i] = 0.f;
      for (int lc = lane; lc < I / 32; lc += 32) {
        if (!(b0 == 0 && lc == lane)) down_load(dmat, cta, G, kRC, wi, nwk, b0, nr, I, lc, R);
        if (dmat.bits == 4) down_accum<4>(R, nr, lc, hpk, hsk, hK, yv);
        else down_accum<2>(R, nr, lc, hpk, hsk, hK, yv);
      }
      const float sred = warp_reduce_rows<8>(yv, lane);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (i < nr && lane == lane_of_reduced_row<8>(i)) {
          const int ri = b0 + i, blk = ri / kRC;
          yk[(wi + nwk * blk) * kRC + (ri - blk * kRC)] = sred;
        }
      }
    }
    if (lane == 0 && p.trace) atomicMax(&misc->t_lastC, (unsigned long long)gtimer());
  }
  if (lane == 0) QE_TRACE(32 + warp);
  __syncthreads();
  if (tid == 0) QE_TRACE(48);

  // ----------------------------------------------- combine of owned rows
  if (!*abort_flag) {
    for (int lr = tid; lr < own * kRC; lr += kFusedThreads) {
      const int ob = lr / kRC;
      const int r = (cta + G * ob) * kRC + (lr - ob * kRC);
      float acc = 0.f;
      for (int k = 0; k < K; ++k) acc += misc->wk[k] * ycomb[(size_t)k * MR + lr];
      if (p.add_residual) acc += load_x(p, r);
      p.out[r] = acc;
    }
  }
  __syncthreads();
  if (tid == 0) {
    QE_TRACE(49);
    if (p.trace) p.trace[(size_t)cta * 64 + kTrLastC] = misc->t_lastC;
    QE_TRACE(kTrEnd);
    if (p.trace) p.trace[(size_t)cta * 64 + 13] = clock64();
  }
}

// ------------------------------------------------------------ host side

static int align_up(int v, int a) { return (v + a - 1) / a * a; }

int fused_geometry(int H, int E, int K, int I, int sms, int smem_optin, FusedGeometry* out) {
  FusedGeometry g{};
  // gate/up items of kRB rows in column quarters: H a multiple of 256 keeps
  // every copied quarter row and scale segment a multiple of 16 bytes
  if (H % 256 != 0 || I % kRB != 0 || H % kRC != 0) return QE_ERR_UNSUPPORTED;
  if (E > kRouterRows * sms) return QE_ERR_UNSUPPORTED;
  if (H > kChunkMax * 32 * kWarps) return QE_ERR_UNSUPPORTED;
  g.RB = kRB;
  g.RC = kRC;
  g.nIB = I / kRB;
  g.nB = K * g.nIB;
  g.nCB = H / kRC;
  g.grid = sms;
  g.max_own = (g.nCB + sms - 1) / sms;
  const int srow = (H % 2048) == 0 ? H / 256 : H / kGroup;
  g.slot = align_up(kRB * H + 4 * 4 * kRB * srow * 2, 128);
  int off = 0;
  g.off_xp4 = off; off = align_up(off + 4 * H, 128);
  g.off_xp2 = off; off = align_up(off + 4 * H, 128);
  g.off_xs = off; off = align_up(off + 4 * (H / 32), 128);
  g.off_hp = off; off = align_up(off + 4 * K * I, 128);
  g.off_hs = off; off = align_up(off + 4 * K * (I / 32), 128);
  g.off_ycomb = off; off = align_up(off + 4 * K * g.max_own * kRC, 128);
  g.off_misc = off; off = align_up(off + (int)sizeof(FusedMisc), 1024);
  g.off_ring = off;
  const int budget = smem_optin - off;
  g.nslot = budget / (kGroups * g.slot);
  if (g.nslot > 3) g.nslot = 3;
  if (g.nslot < 1) return QE_ERR_UNSUPPORTED;
  g.smem_bytes = off + g.nslot * kGroups * g.slot;
  *out = g;
  return QE_OK;
}

cudaError_t launch_fused_layer(const FusedParams& p, cudaStream_t s) {
  static bool attr_set = false;
  if (!attr_set) {
    int optin = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaError_t e = cudaFuncSetAttribute(qe_fused_layer_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e != cudaSuccess) return e;
    attr_set = true;
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
