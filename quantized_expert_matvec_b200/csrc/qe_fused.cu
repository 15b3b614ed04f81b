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
// Expert phase: the selected experts' rows are cut into items, gate/up items
// (RB rows of gate and of up) and down items (RC rows of one expert's down
// matrix, for an output block this CTA owns).  Each warp owns a private ring
// of shared-memory slots and streams its own items into it with 16-byte
// cp.async copies, so the next item is in flight while the current one is
// dequantised; there is no producer warp and no cross-warp handshake on the
// rings.  Down items need h_k = silu(g_k) * u_k in full: every gate/up item of
// expert k bumps a global counter ready[k]; the first warp of a CTA that needs
// h_k waits for the count, stages h_k in x' form in shared memory and raises
// a flag for the others.  All such waits are bounded (QE_ERR_TIMEOUT).
// The last CTA to finish resets the counters for the next launch.
#include <math.h>

#include "qe_device.cuh"

namespace qe {

constexpr int kWarps = 16;
constexpr int kFusedThreads = kWarps * 32;
constexpr int kRouterRows = 8;  // router rows one CTA owns at most: E <= 8 * grid
constexpr int kChunkMax = 16;   // 32-column chunks one warp converts: H <= 16 * 32 * 16

struct FusedMisc {
  int abort;
  float xK;
  int idx[kMaxK];
  float wk[kMaxK];
  qe_expert ex[kMaxK];
  float hK[kMaxK];
  unsigned claim[kMaxK];
  int hflag[kMaxK];
  unsigned cand_idx[kWarps][kMaxK];
  unsigned long long t_lastB, t_lastC;
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

// ------------------------------------------------------------ gate/up item
// RB rows of gate and RB rows of up of one expert, staged in a slot as
// [gate wq | up wq (at RB*H/2) | gate s | gate b | up s | up b].
template <int RB, int BITS>
static __device__ __forceinline__ void gateup_item(const unsigned char* slot, int H, const float* xp,
                                                   const float* xs_sum, float xK, float* h_out,
                                                   int lane) {
  constexpr int COLS = BITS == 4 ? 32 : 64;  // columns per uint4 chunk
  const int nch = H / COLS;
  const int row_bytes = H * BITS / 8;
  const int gpr = H / kGroup;
  const unsigned char* gw = slot;
  const unsigned char* uw = slot + RB * H / 2;
  const uint16_t* gs = (const uint16_t*)(slot + RB * H);
  const uint16_t* gb = gs + RB * gpr;
  const uint16_t* us = gb + RB * gpr;
  const uint16_t* ub = us + RB * gpr;
  float yv[2 * RB];
#pragma unroll
  for (int i = 0; i < 2 * RB; ++i) yv[i] = 0.f;
  for (int ch = lane; ch < nch; ch += 32) {
    float2 xs[COLS / 2];
    const float4* src = (const float4*)(xp + ch * COLS);
    const int sw = ch & 7;
#pragma unroll
    for (int i = 0; i < COLS / 4; ++i) {
      const float4 v = src[i ^ sw];
      xs[2 * i] = make_float2(v.x, v.y);
      xs[2 * i + 1] = make_float2(v.z, v.w);
    }
    const int g = BITS == 4 ? (ch >> 1) : ch;
    const float xsum = BITS == 4 ? xs_sum[ch] : xs_sum[2 * ch] + xs_sum[2 * ch + 1];
#pragma unroll
    for (int rr = 0; rr < RB; ++rr) {
      const uint4 wg = *(const uint4*)(gw + rr * row_bytes + ch * 16);
      const uint4 wu = *(const uint4*)(uw + rr * row_bytes + ch * 16);
      const float2 ag = BITS == 4 ? dot32_q4(wg, xs, make_float2(0.f, 0.f)) : dot64_q2(wg, xs, make_float2(0.f, 0.f));
      const float2 au = BITS == 4 ? dot32_q4(wu, xs, make_float2(0.f, 0.f)) : dot64_q2(wu, xs, make_float2(0.f, 0.f));
      yv[rr] += bf16f(gs[rr * gpr + g]) * xK * (ag.x + ag.y) + bf16f(gb[rr * gpr + g]) * xsum;
      yv[RB + rr] += bf16f(us[rr * gpr + g]) * xK * (au.x + au.y) + bf16f(ub[rr * gpr + g]) * xsum;
    }
  }
  const float s = warp_reduce_rows<2 * RB>(yv, lane);
#pragma unroll
  for (int rr = 0; rr < RB; ++rr) {
    const float gv = __shfl_sync(0xffffffffu, s, lane_of_reduced_row<2 * RB>(rr));
    const float uv = __shfl_sync(0xffffffffu, s, lane_of_reduced_row<2 * RB>(RB + rr));
    if (lane == rr) h_out[rr] = gv / (1.0f + expf(-gv)) * uv;
  }
}

// --------------------------------------------------------------- down item
// RC rows of one expert's down matrix: [wq | s (at RC*I/2) | b].
template <int RC, int BITS>
static __device__ __forceinline__ void down_item(const unsigned char* slot, int I, const float* hp,
                                                 const float* hsum, float hK, float* y_out, int lane) {
  constexpr int COLS = BITS == 4 ? 32 : 64;
  const int nch = I / COLS;
  const int row_bytes = I * BITS / 8;
  const int gpr = I / kGroup;
  const uint16_t* ds = (const uint16_t*)(slot + RC * I / 2);
  const uint16_t* db = ds + RC * gpr;
  float yv[RC];
#pragma unroll
  for (int i = 0; i < RC; ++i) yv[i] = 0.f;
  for (int ch = lane; ch < nch; ch += 32) {
    float2 xs[COLS / 2];
    const float4* src = (const float4*)(hp + ch * COLS);
    const int sw = ch & 7;
#pragma unroll
    for (int i = 0; i < COLS / 4; ++i) {
      const float4 v = src[i ^ sw];
      xs[2 * i] = make_float2(v.x, v.y);
      xs[2 * i + 1] = make_float2(v.z, v.w);
    }
    const int g = BITS == 4 ? (ch >> 1) : ch;
    const float xsum = BITS == 4 ? hsum[ch] : hsum[2 * ch] + hsum[2 * ch + 1];
#pragma unroll
    for (int rr = 0; rr < RC; ++rr) {
      const uint4 w = *(const uint4*)(slot + rr * row_bytes + ch * 16);
      const float2 a = BITS == 4 ? dot32_q4(w, xs, make_float2(0.f, 0.f)) : dot64_q2(w, xs, make_float2(0.f, 0.f));
      yv[rr] += bf16f(ds[rr * gpr + g]) * hK * (a.x + a.y) + bf16f(db[rr * gpr + g]) * xsum;
    }
  }
  const float s = warp_reduce_rows<RC>(yv, lane);
#pragma unroll
  for (int rr = 0; rr < RC; ++rr)
    if (lane == lane_of_reduced_row<RC>(rr)) y_out[rr] = s;
}

template <int BITS>
static __device__ __forceinline__ void gateup_dispatch(int RB, const unsigned char* slot, int H, const float* xp,
                                                       const float* xs_sum, float xK, float* h_out, int lane) {
  if (RB == 1) gateup_item<1, BITS>(slot, H, xp, xs_sum, xK, h_out, lane);
  else if (RB == 2) gateup_item<2, BITS>(slot, H, xp, xs_sum, xK, h_out, lane);
  else if (RB == 4) gateup_item<4, BITS>(slot, H, xp, xs_sum, xK, h_out, lane);
  else gateup_item<8, BITS>(slot, H, xp, xs_sum, xK, h_out, lane);
}

template <int BITS>
static __device__ __forceinline__ void down_dispatch(int RC, const unsigned char* slot, int I, const float* hp,
                                                     const float* hsum, float hK, float* y_out, int lane) {
  if (RC == 4) down_item<4, BITS>(slot, I, hp, hsum, hK, y_out, lane);
  else down_item<8, BITS>(slot, I, hp, hsum, hK, y_out, lane);
}

// Item j of this CTA's list (gate/up items, then down items k-major).
struct ItemRef {
  bool gateup;
  int k;   // position in the top-K list
  int r0;  // first row (gate/up: row of I; down: row of H)
  int ob;  // down: index of the owned output block
};

static __device__ __forceinline__ ItemRef item_ref(int j, int nBc, int own, int cta, int G, const FusedGeometry& g) {
  ItemRef it;
  if (j < nBc) {
    const int gi = cta + G * j;
    it.gateup = true;
    it.k = gi / g.nIB;
    it.r0 = (gi - it.k * g.nIB) * g.RB;
    it.ob = 0;
  } else {
    const int jc = j - nBc;
    it.gateup = false;
    it.k = jc / own;
    it.ob = jc - it.k * own;
    it.r0 = (cta + G * it.ob) * g.RC;
  }
  return it;
}

// Issue the copies of one item into a slot (all lanes), then commit.
static __device__ __forceinline__ void issue_item(const ItemRef& it, unsigned char* slot, const FusedMisc* misc,
                                                  int H, int I, const FusedGeometry& g, int lane, uint64_t pol) {
  const qe_expert& ex = misc->ex[it.k];
  if (it.gateup) {
    const int bits = ex.gate.bits;
    const uint32_t wbytes = (uint32_t)(g.RB * H * bits / 8);
    const uint32_t sbytes = (uint32_t)(g.RB * (H / kGroup) * 2);
    const size_t wrow = (size_t)H * bits / 32;
    const size_t srow = (size_t)(H / kGroup);
    warp_copy_async(slot, ex.gate.wq + (size_t)it.r0 * wrow, wbytes, lane, pol);
    warp_copy_async(slot + g.RB * H / 2, ex.up.wq + (size_t)it.r0 * wrow, wbytes, lane, pol);
    unsigned char* sd = slot + g.RB * H;
    warp_copy_async(sd, ex.gate.scales + (size_t)it.r0 * srow, sbytes, lane, pol);
    warp_copy_async(sd + sbytes, ex.gate.biases + (size_t)it.r0 * srow, sbytes, lane, pol);
    warp_copy_async(sd + 2 * sbytes, ex.up.scales + (size_t)it.r0 * srow, sbytes, lane, pol);
    warp_copy_async(sd + 3 * sbytes, ex.up.biases + (size_t)it.r0 * srow, sbytes, lane, pol);
  } else {
    const qe_qmat& d = ex.down;
    const uint32_t wbytes = (uint32_t)(g.RC * I * d.bits / 8);
    const uint32_t sbytes = (uint32_t)(g.RC * (I / kGroup) * 2);
    warp_copy_async(slot, d.wq + (size_t)it.r0 * I * d.bits / 32, wbytes, lane, pol);
    warp_copy_async(slot + g.RC * I / 2, d.scales + (size_t)it.r0 * (I / kGroup), sbytes, lane, pol);
    warp_copy_async(slot + g.RC * I / 2 + sbytes, d.biases + (size_t)it.r0 * (I / kGroup), sbytes, lane, pol);
  }
  cp_async_commit();
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
  unsigned char* ring = smem + g.off_ring + (size_t)warp * g.nslot * g.slot;
  WsControl* ctl = p.ctl;

  if (tid == 0) {
    misc->abort = 0;
    misc->t_lastB = 0;
    misc->t_lastC = 0;
    QE_TRACE(kTrStart);
    if (p.trace) p.trace[(size_t)cta * 64 + 12] = clock64();
  }
  if (tid < kMaxK) {
    misc->claim[tid] = 0;
    misc->hflag[tid] = 0;
  }

  // ------------------------------------------------------------- routing
  // The router dot s_e = sum_c W[e,c] x_c gamma_c does not depend on the
  // RMSNorm scale, so it runs on the same loads as the sum of squares; the
  // logit is s_e * rinv (+ offset_e), all in fp64.  Warp w covers the column
  // slice [w*S, (w+1)*S), S = H/16, of each router row its CTA owns; the 16
  // slice sums are added in slice order.
  const int nrows = E > cta ? (E - cta + G - 1) / G : 0;
  {
    const int S = H / kWarps;
    double ss = 0.0;
    double acc[kRouterRows];
#pragma unroll
    for (int m = 0; m < kRouterRows; ++m) acc[m] = 0.0;
    for (int i = lane; i < S / 4; i += 32) {
      const int c = warp * S + 4 * i;
      float4 wv[kRouterRows];
#pragma unroll
      for (int m = 0; m < kRouterRows; ++m)
        if (m < nrows) wv[m] = __ldg((const float4*)(p.router_w + (size_t)(cta + G * m) * H + c));
      double xv[4];
      load_x4(p, c, xv);
      ss += xv[0] * xv[0] + xv[1] * xv[1] + xv[2] * xv[2] + xv[3] * xv[3];
      if (p.gamma) {
        const float4 gm = *(const float4*)(p.gamma + c);
        xv[0] *= (double)gm.x; xv[1] *= (double)gm.y; xv[2] *= (double)gm.z; xv[3] *= (double)gm.w;
      }
#pragma unroll
      for (int m = 0; m < kRouterRows; ++m) {
        if (m < nrows) {
          double a = acc[m];
          a = fma((double)wv[m].x, xv[0], a);
          a = fma((double)wv[m].y, xv[1], a);
          a = fma((double)wv[m].z, xv[2], a);
          a = fma((double)wv[m].w, xv[3], a);
          acc[m] = a;
        }
      }
    }
    ss = warp_sum_d(ss);
#pragma unroll
    for (int m = 0; m < kRouterRows; ++m) {
      if (m < nrows) {
        const double t = warp_sum_d(acc[m]);
        if (lane == 0) misc->rpart[m][warp] = t;
      }
    }
    if (lane == 0) misc->redd[warp] = ss;
  }
  __syncthreads();
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
  float xnv[kChunkMax];
  {
    float amax = 0.f;
#pragma unroll
    for (int q = 0; q < kChunkMax; ++q) {
      const int ch = warp + kWarps * q;
      xnv[q] = 0.f;
      if (ch < H / 32) {
        const int c = ch * 32 + lane;
        const double gm = p.gamma ? (double)p.gamma[c] : 1.0;
        xnv[q] = (float)((double)load_x(p, c) * rinv * gm);
        amax = fmaxf(amax, fabsf(xnv[q]));
      }
    }
    amax = warp_max(amax);
    if (lane == 0) misc->redf[warp] = amax;
  }
  __syncthreads();
  if (tid == 0) {
    QE_TRACE(kTrRouterDone);
    __threadfence();
    if (cta != p.skip_cta) atomicAdd(&ctl->route_ctr, 1u);
  }
  {
    float m = 0.f;
    for (int w = 0; w < kWarps; ++w) m = fmaxf(m, misc->redf[w]);
    const int Ex = xscale_exponent(m);
    if (tid == 0) misc->xK = acc_scale(Ex);
#pragma unroll
    for (int q = 0; q < kChunkMax; ++q) {
      const int ch = warp + kWarps * q;
      if (ch < H / 32) {
        const int c = ch * 32 + lane;
        const float sm = warp_sum(xnv[q]);
        if (lane == 0) xsum[ch] = sm;
        xp4[swz_q4(c)] = xprime_q4(xnv[q], c, Ex);
        xp2[swz_q2(c)] = xprime_q2(xnv[q], c, Ex);
      }
    }
  }
  if (tid == 0) {
    if (!wait_geq(&ctl->route_ctr, (unsigned)G, deadline, abort_flag)) {
      set_error(&ctl->err, QE_ERR_TIMEOUT);
      misc->abort = 1;
    }
    QE_TRACE(kTrRouteBarrier);
  }
  __syncthreads();

  // ---------------------------------------------------------------- top-K
  // Thread t ranks logits t and t+512.  Each warp finds its own top-K by K
  // rounds of warp_argmax_key (a sorted candidate list); warp 0 then merges
  // the 16 lists, one list per lane.
  if (!*abort_flag) {
    const unsigned iA = (unsigned)tid, iB = (unsigned)(tid + kFusedThreads);
    bool hasA = tid < E, hasB = tid + kFusedThreads < E;
    const unsigned long long kA = hasA ? dkey(__ldcg(&p.logit_part[iA])) : 0ull;
    const unsigned long long kB = hasB ? dkey(__ldcg(&p.logit_part[iB])) : 0ull;
    for (int k = 0; k < K; ++k) {
      const bool useA = hasA && (!hasB || kA >= kB);  // equal keys: A has the lower index
      const unsigned bi = (hasA || hasB) ? (useA ? iA : iB) : 0xffffffffu;
      const unsigned win = warp_argmax_key(useA ? kA : kB, bi);
      if (lane == 0) misc->cand_idx[warp][k] = win;
      if (bi != 0xffffffffu && bi == win) {
        if (useA) hasA = false;
        else hasB = false;
      }
    }
  }
  __syncthreads();
  if (warp == 0 && !*abort_flag) {
    int ptr = 0;
    for (int k = 0; k < K; ++k) {
      unsigned bi = 0xffffffffu;
      unsigned long long bk = 0;
      if (lane < kWarps && ptr < K) {
        bi = misc->cand_idx[lane][ptr];
        if (bi != 0xffffffffu) bk = dkey(__ldcg(&p.logit_part[bi]));
      }
      const unsigned win = warp_argmax_key(bk, bi);
      if (lane == 0) misc->idx[k] = (int)win;
      if (bi != 0xffffffffu && bi == win) ++ptr;
    }
    __syncwarp();
    // renormalised softmax over the K kept logits (sum in k order); lanes
    // k < K also fetch and check the K expert descriptors
    const double lmax = __ldcg(&p.logit_part[misc->idx[0]]);
    const double ev = lane < K ? exp(__ldcg(&p.logit_part[misc->idx[lane]]) - lmax) : 0.0;
    double s = 0.0;
    for (int k = 0; k < K; ++k) s += __shfl_sync(0xffffffffu, ev, k);
    if (lane < K) {
      misc->wk[lane] = (float)(ev / s);
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

  // ------------------------------------------------ expert phase (per warp)
  const int nBc = g.nB > cta ? (g.nB - cta + G - 1) / G : 0;
  const int own = g.nCB > cta ? (g.nCB - cta + G - 1) / G : 0;
  const int nItems = nBc + K * own;
  const int MR = g.max_own * g.RC;  // rows of one expert's slice of ycomb
  const int nmine = warp < nItems ? (nItems - warp + kWarps - 1) / kWarps : 0;
  if (!*abort_flag && nmine > 0) {
    const uint64_t pol = policy_evict_first();
    for (int q = 0; q < g.nslot && q < nmine; ++q)
      issue_item(item_ref(warp + kWarps * q, nBc, own, cta, G, g), ring + (size_t)q * g.slot, misc, H, I, g,
                 lane, pol);
    for (int q = 0; q < nmine; ++q) {
      const int j = warp + kWarps * q;
      const ItemRef it = item_ref(j, nBc, own, cta, G, g);
      unsigned char* sl = ring + (size_t)(q % g.nslot) * g.slot;
      // groups committed after this item's own: the items already issued ahead
      const int later = (q + g.nslot <= nmine ? g.nslot : nmine - q) - 1;
      if (later >= 1) cp_async_wait<1>(); else cp_async_wait<0>();
      __syncwarp();
      if (q == 0 && lane == 0) QE_TRACE(16 + warp);
      if (it.gateup) {
        float* hdst = p.hbuf + (size_t)it.k * I + it.r0;
        if (misc->ex[it.k].gate.bits == 4)
          gateup_dispatch<4>(g.RB, sl, H, xp4, xsum, misc->xK, hdst, lane);
        else
          gateup_dispatch<2>(g.RB, sl, H, xp2, xsum, misc->xK, hdst, lane);
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          red_release_add(&ctl->ready[it.k], 1u);
          if (p.trace) atomicMax(&misc->t_lastB, (unsigned long long)gtimer());
        }
      } else {
        const int k = it.k;
        const int dbits = misc->ex[k].down.bits;
        // stage h_k in shared memory (first warp to need it) or wait for it
        unsigned won = 0;
        if (lane == 0) won = atomicCAS(&misc->claim[k], 0u, 1u) == 0u;
        won = __shfl_sync(0xffffffffu, won, 0);
        int ok = 1;
        if (won) {
          if (lane == 0) ok = wait_geq(&ctl->ready[k], (unsigned)g.nIB, deadline, abort_flag);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (ok) {
            if (lane == 0 && k == 0) QE_TRACE(kTrHFirst);
            if (lane == 0 && k == K - 1) QE_TRACE(kTrHLast);
            float* hpk = hp + (size_t)k * I;
            float* hsk = hsum + (size_t)k * (I / 32);
            const float* hsrc = p.hbuf + (size_t)k * I;
            float am = 0.f;
            for (int c = lane; c < I; c += 32) am = fmaxf(am, fabsf(__ldcg(hsrc + c)));
            const int Eh = xscale_exponent(warp_max(am));
            for (int ch = 0; ch < I / 32; ++ch) {
              const int c = ch * 32 + lane;
              const float v = __ldcg(hsrc + c);
              const float sm = warp_sum(v);
              if (lane == 0) hsk[ch] = sm;
              if (dbits == 4) hpk[swz_q4(c)] = xprime_q4(v, c, Eh);
              else hpk[swz_q2(c)] = xprime_q2(v, c, Eh);
            }
            if (lane == 0) misc->hK[k] = acc_scale(Eh);
            __threadfence_block();
            __syncwarp();
            if (lane == 0) *(volatile int*)&misc->hflag[k] = 1;
          }
        } else {
          if (lane == 0) {
            unsigned spins = 0;
            while (*(volatile int*)&misc->hflag[k] == 0) {
              if (*abort_flag || ((++spins & 15u) == 0 && gtimer() > deadline)) { ok = 0; break; }
              __nanosleep(32);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          __threadfence_block();
        }
        if (!ok) {
          if (lane == 0) { set_error(&ctl->err, QE_ERR_TIMEOUT); *abort_flag = 1; }
          break;
        }
        float* ydst = ycomb + (size_t)k * MR + it.ob * g.RC;
        const float* hpk = hp + (size_t)k * I;
        const float* hsk = hsum + (size_t)k * (I / 32);
        if (dbits == 4)
          down_dispatch<4>(g.RC, sl, I, hpk, hsk, misc->hK[k], ydst, lane);
        else
          down_dispatch<2>(g.RC, sl, I, hpk, hsk, misc->hK[k], ydst, lane);
        if (lane == 0 && p.trace) atomicMax(&misc->t_lastC, (unsigned long long)gtimer());
      }
      if (q == 0 && lane == 0) QE_TRACE(32 + warp);
      __syncwarp();
      // refill this slot with the item nslot places ahead
      if (q + g.nslot < nmine)
        issue_item(item_ref(warp + kWarps * (q + g.nslot), nBc, own, cta, G, g), sl, misc, H, I, g, lane, pol);
      if (*abort_flag) break;
    }
    cp_async_wait<0>();  // nothing may still be landing when the CTA exits
  }
  __syncthreads();
  if (tid == 0) QE_TRACE(48);

  // ----------------------------------------------- combine of owned rows
  if (!*abort_flag) {
    for (int lr = tid; lr < own * g.RC; lr += kFusedThreads) {
      const int ob = lr / g.RC;
      const int r = (cta + G * ob) * g.RC + (lr - ob * g.RC);
      float acc = 0.f;
      for (int k = 0; k < K; ++k) acc += misc->wk[k] * ycomb[(size_t)k * MR + lr];
      if (p.add_residual) acc += load_x(p, r);
      p.out[r] = acc;
    }
  }
  __syncthreads();
  if (tid == 0) {
    QE_TRACE(49);
    __threadfence();
    const unsigned prev = atomicAdd(&ctl->exit_ctr, 1u);
    QE_TRACE(53);
    if (prev == (unsigned)G - 1) {
      ctl->route_ctr = 0;
      for (int k = 0; k < kMaxK; ++k) ctl->ready[k] = 0;
      __threadfence();
      ctl->exit_ctr = 0;
      __threadfence();
    }
    if (p.trace) {
      p.trace[(size_t)cta * 64 + kTrLastB] = misc->t_lastB;
      p.trace[(size_t)cta * 64 + kTrLastC] = misc->t_lastC;
    }
    QE_TRACE(kTrEnd);
    if (p.trace) p.trace[(size_t)cta * 64 + 13] = clock64();
  }
}

// ------------------------------------------------------------ host side

static int align_up(int v, int a) { return (v + a - 1) / a * a; }
static int gcd_int(int a, int b) { while (b) { int t = a % b; a = b; b = t; } return a; }

int fused_geometry(int H, int E, int K, int I, int sms, int smem_optin, FusedGeometry* out) {
  FusedGeometry g{};
  // rows per item: every copied segment must be a multiple of 16 bytes
  // (RB*H and RC*I multiples of 512)
  g.RB = 8 / gcd_int(H / kGroup, 8);
  g.RC = 8 / gcd_int(I / kGroup, 8);
  if (g.RC < 4) g.RC = 4;
  if (I % g.RB || H % g.RC) return QE_ERR_UNSUPPORTED;
  if (E > kRouterRows * sms) return QE_ERR_UNSUPPORTED;
  if (H > kChunkMax * 32 * kWarps) return QE_ERR_UNSUPPORTED;
  g.nIB = I / g.RB;
  g.nB = K * g.nIB;
  g.nCB = H / g.RC;
  g.grid = sms;
  g.max_own = (g.nCB + sms - 1) / sms;
  const int slotB = g.RB * H + 4 * g.RB * (H / kGroup) * 2;
  const int slotC = g.RC * I / 2 + 2 * g.RC * (I / kGroup) * 2;
  g.slot = align_up(slotB > slotC ? slotB : slotC, 128);
  int off = 0;
  g.off_xp4 = off; off = align_up(off + 4 * H, 128);
  g.off_xp2 = off; off = align_up(off + 4 * H, 128);
  g.off_xs = off; off = align_up(off + 4 * (H / 32), 128);
  g.off_hp = off; off = align_up(off + 4 * K * I, 128);
  g.off_hs = off; off = align_up(off + 4 * K * (I / 32), 128);
  g.off_ycomb = off; off = align_up(off + 4 * K * g.max_own * g.RC, 128);
  g.off_misc = off; off = align_up(off + (int)sizeof(FusedMisc), 1024);
  g.off_ring = off;
  const int budget = smem_optin - off;
  g.nslot = budget >= 2 * kWarps * g.slot ? 2 : (budget >= kWarps * g.slot ? 1 : 0);
  if (g.nslot == 0) return QE_ERR_UNSUPPORTED;
  g.smem_bytes = off + g.nslot * kWarps * g.slot;
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
