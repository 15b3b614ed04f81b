// qe_fused.cu -- the single-token layer step as ONE persistent kernel:
// RMSNorm -> router (fp64) -> top-K -> gate/up dequant-matvec + SwiGLU ->
// down dequant-matvec -> weighted combine (+ residual).
//
// One CTA per SM, launched cooperatively so all CTAs are resident.  Each CTA
// has 15 consumer warps and 1 producer warp.  After routing, the producer's
// elected lane streams this CTA's share of the selected experts' packed rows
// into two shared-memory rings with bulk copies (cp.async.bulk, completion on
// mbarriers): ring B holds gate/up row pairs, ring C holds down rows.  Ring C
// fills while gate/up is still being computed, so the down weights are on chip
// when h becomes ready.  Consumer warps process items as they land.
//
// Cross-CTA dependencies, each a bounded wait (QE_ERR_TIMEOUT on expiry):
//   1. router -> top-K: every CTA writes its half-row logits, then arrives on
//      a counter; each CTA then ranks all E logits itself.
//   2. gate/up -> down: expert k's down rows need all of h_k; every gate/up
//      item of expert k bumps ready[k] after storing its h values, and the
//      first warp of a CTA that needs h_k waits for ready[k] == items(k) and
//      stages h_k (in x' form) in shared memory for the others.
// The last CTA to finish resets the counters, so the workspace is ready for
// the next launch (also inside a CUDA graph).
#include <math.h>

#include "qe_device.cuh"

namespace qe {

constexpr int kConsumerWarps = 15;
constexpr int kFusedWarps = kConsumerWarps + 1;
constexpr int kFusedThreads = kFusedWarps * 32;

struct FusedMisc {
  int abort;
  int xexp;
  float xK;
  int pad;
  double rinv;
  int idx[kMaxK];
  float wk[kMaxK];
  qe_expert ex[kMaxK];
  float hK[kMaxK];
  unsigned claim[kMaxK];
  int issuedB, issuedC;
  float redf[32];
  double redd[32];
};

static __device__ __forceinline__ float load_x(const FusedParams& p, int c) {
  return p.x_bf16 ? bf16f(((const uint16_t*)p.x)[c]) : ((const float*)p.x)[c];
}

static __device__ __forceinline__ bool desc_ok(const qe_qmat& m, int bits) {
  return m.bits == bits && m.wq && m.scales && m.biases && ((uintptr_t)m.wq & 15) == 0 &&
         ((uintptr_t)m.scales & 15) == 0 && ((uintptr_t)m.biases & 15) == 0;
}

// ------------------------------------------------------------ gate/up item
// RB rows of gate and RB rows of up of one expert, staged in a ring slot as
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
#pragma unroll
    for (int i = 0; i < COLS / 4; ++i) {
      float4 v = src[i];
      xs[2 * i] = make_float2(v.x, v.y);
      xs[2 * i + 1] = make_float2(v.z, v.w);
    }
    const int g = BITS == 4 ? (ch >> 1) : ch;
    const float xsum = BITS == 4 ? xs_sum[ch] : xs_sum[2 * ch] + xs_sum[2 * ch + 1];
#pragma unroll
    for (int rr = 0; rr < RB; ++rr) {
      const uint4 wg = *(const uint4*)(gw + rr * row_bytes + ch * 16);
      const uint4 wu = *(const uint4*)(uw + rr * row_bytes + ch * 16);
      float2 ag = BITS == 4 ? dot32_q4(wg, xs, make_float2(0.f, 0.f)) : dot64_q2(wg, xs, make_float2(0.f, 0.f));
      float2 au = BITS == 4 ? dot32_q4(wu, xs, make_float2(0.f, 0.f)) : dot64_q2(wu, xs, make_float2(0.f, 0.f));
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
#pragma unroll
    for (int i = 0; i < COLS / 4; ++i) {
      float4 v = src[i];
      xs[2 * i] = make_float2(v.x, v.y);
      xs[2 * i + 1] = make_float2(v.z, v.w);
    }
    const int g = BITS == 4 ? (ch >> 1) : ch;
    const float xsum = BITS == 4 ? hsum[ch] : hsum[2 * ch] + hsum[2 * ch + 1];
#pragma unroll
    for (int rr = 0; rr < RC; ++rr) {
      const uint4 w = *(const uint4*)(slot + rr * row_bytes + ch * 16);
      float2 a = BITS == 4 ? dot32_q4(w, xs, make_float2(0.f, 0.f)) : dot64_q2(w, xs, make_float2(0.f, 0.f));
      yv[rr] += bf16f(ds[rr * gpr + g]) * hK * (a.x + a.y) + bf16f(db[rr * gpr + g]) * xsum;
    }
  }
  const float s = warp_reduce_rows<RC>(yv, lane);
#pragma unroll
  for (int rr = 0; rr < RC; ++rr)
    if (lane == lane_of_reduced_row<RC>(rr)) y_out[rr] = s;
}

template <int BITS>
static __device__ __forceinline__ void gateup_dispatch(int RB, const unsigned char* slot, int H,
                                                       const float* xp, const float* xs_sum, float xK,
                                                       float* h_out, int lane) {
  if (RB == 2) gateup_item<2, BITS>(slot, H, xp, xs_sum, xK, h_out, lane);
  else if (RB == 4) gateup_item<4, BITS>(slot, H, xp, xs_sum, xK, h_out, lane);
  else gateup_item<8, BITS>(slot, H, xp, xs_sum, xK, h_out, lane);
}

template <int BITS>
static __device__ __forceinline__ void down_dispatch(int RC, const unsigned char* slot, int I,
                                                     const float* hp, const float* hsum, float hK,
                                                     float* y_out, int lane) {
  if (RC == 4) down_item<4, BITS>(slot, I, hp, hsum, hK, y_out, lane);
  else down_item<8, BITS>(slot, I, hp, hsum, hK, y_out, lane);
}

// The producer publishes how many items of a ring it has issued.  A consumer
// waits for its item to be issued before it waits on the slot's full
// barrier: a parity wait only tells the current phase from the one before,
// so waiting on lap L of a slot whose lap L-1 has not even been issued would
// return at once.
static __device__ __forceinline__ void publish_issued(int* ctr, int v) {
  asm volatile("st.release.cta.shared::cta.s32 [%0], %1;" ::"r"(smem_u32(ctr)), "r"(v) : "memory");
}

static __device__ __forceinline__ bool wait_issued(int* ctr, int j, uint64_t deadline,
                                                   volatile int* abort_flag) {
  unsigned spins = 0;
  for (;;) {
    int v;
    asm volatile("ld.acquire.cta.shared::cta.s32 %0, [%1];" : "=r"(v) : "r"(smem_u32(ctr)) : "memory");
    if (v > j) return true;
    if (*abort_flag) return false;
    if ((++spins & 15u) == 0 && gtimer() > deadline) return false;
    __nanosleep(20);
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
  uint64_t* bars = (uint64_t*)(smem + g.off_bars);
  uint64_t* fullB = bars;
  uint64_t* emptyB = fullB + g.nslotB;
  uint64_t* fullC = emptyB + g.nslotB;
  uint64_t* emptyC = fullC + g.nslotC;
  uint64_t* hready = emptyC + g.nslotC;
  unsigned char* ringB = smem + g.off_ringB;
  unsigned char* ringC = smem + g.off_ringC;
  float* xp4 = (float*)(smem + g.off_xp4);
  float* xp2 = (float*)(smem + g.off_xp2);
  float* xsum = (float*)(smem + g.off_xs);
  float* hp = (float*)(smem + g.off_hp);      // [K][I], after routing
  float* hsum = (float*)(smem + g.off_hs);    // [K][I/32]
  double* xg = (double*)(smem + g.off_hp);    // [H] during routing (same region)
  double* lg = (double*)(smem + g.off_logit);
  float* ycomb = (float*)(smem + g.off_ycomb);
  WsControl* ctl = p.ctl;

  if (tid == 0) {
    misc->abort = 0;
    for (int i = 0; i < g.nslotB; ++i) { mbar_init(&fullB[i], 1); mbar_init(&emptyB[i], 1); }
    for (int i = 0; i < g.nslotC; ++i) { mbar_init(&fullC[i], 1); mbar_init(&emptyC[i], 1); }
    for (int k = 0; k < K; ++k) { mbar_init(&hready[k], 1); misc->claim[k] = 0; }
    misc->issuedB = 0;
    misc->issuedC = 0;
    fence_mbar_init();
  }

  // ---------------------------------------------- RMSNorm (pass 1: sum x^2)
  double ss = 0.0;
  for (int c = tid; c < H; c += kFusedThreads) {
    const double v = (double)load_x(p, c);
    ss += v * v;
  }
  ss = warp_sum_d(ss);
  if (lane == 0) misc->redd[warp] = ss;
  __syncthreads();
  if (tid == 0) {
    double t = 0.0;
    for (int w = 0; w < kFusedWarps; ++w) t += misc->redd[w];
    misc->rinv = 1.0 / sqrt(t / (double)H + (double)p.eps);
  }
  __syncthreads();
  const double rinv = misc->rinv;

  // --------------------------------------------------- pass 2: apply, x'
  float amax = 0.f;
  for (int c = tid; c < H; c += kFusedThreads) {
    const double xv = (double)load_x(p, c);
    const double gm = p.gamma ? (double)p.gamma[c] : 1.0;
    xg[c] = xv * gm;
    const float xn = (float)(xv * rinv * gm);
    xp4[c] = xn;
    amax = fmaxf(amax, fabsf(xn));
  }
  amax = warp_max(amax);
  if (lane == 0) misc->redf[warp] = amax;
  __syncthreads();
  if (tid == 0) {
    float m = 0.f;
    for (int w = 0; w < kFusedWarps; ++w) m = fmaxf(m, misc->redf[w]);
    misc->xexp = xscale_exponent(m);
    misc->xK = acc_scale(misc->xexp);
  }
  __syncthreads();
  {
    const int Ex = misc->xexp;
    for (int ch = warp; ch < H / 32; ch += kFusedWarps) {
      const int c = ch * 32 + lane;
      const float v = xp4[c];
      const float s = warp_sum(v);
      if (lane == 0) xsum[ch] = s;
      xp4[c] = xprime_q4(v, c, Ex);
      xp2[c] = xprime_q2(v, c, Ex);
    }
  }

  // ------------------------------------------------ router: half-row logits
  {
    const int half_len = H / 2;
    int m = 0;
    for (int hr = cta + G * warp; hr < 2 * E; hr = cta + G * (warp + kFusedWarps * (++m))) {
      const int e = hr >> 1, half = hr & 1;
      const float4* wrow = (const float4*)(p.router_w + (size_t)e * H + half * half_len);
      const double* xh = xg + half * half_len;
      double acc = 0.0;
#pragma unroll 4
      for (int i = lane; i < half_len / 4; i += 32) {
        const float4 wv = __ldg(wrow + i);
        const double* xx = xh + 4 * i;
        acc = fma((double)wv.x, xx[0], acc);
        acc = fma((double)wv.y, xx[1], acc);
        acc = fma((double)wv.z, xx[2], acc);
        acc = fma((double)wv.w, xx[3], acc);
      }
      acc = warp_sum_d(acc);
      if (lane == 0) p.logit_part[half * E + e] = acc;
    }
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    if (cta != p.skip_cta) atomicAdd(&ctl->route_ctr, 1u);
    if (!wait_geq(&ctl->route_ctr, (unsigned)G, deadline, abort_flag)) {
      set_error(&ctl->err, QE_ERR_TIMEOUT);
      misc->abort = 1;
    }
  }
  __syncthreads();

  // ---------------------------------------------------------------- top-K
  if (warp == 0 && !*abort_flag) {
    for (int e = lane; e < E; e += 32) {
      double v = (__ldcg(&p.logit_part[e]) + __ldcg(&p.logit_part[E + e])) * rinv;
      if (p.offset) v += (double)p.offset[e];
      lg[e] = v;
    }
    __syncwarp();
    unsigned taken = 0;
    for (int k = 0; k < K; ++k) {
      double bv = 0.0;
      int bi = 0x7fffffff;
      for (int i = 0, e = lane; e < E; ++i, e += 32) {
        if (taken & (1u << i)) continue;
        const double v = lg[e];
        if (bi == 0x7fffffff || v > bv) { bv = v; bi = e; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        const bool take = oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi));
        if (take) { bv = ov; bi = oi; }
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      if (lane == 0) misc->idx[k] = bi;
    }
    __syncwarp();
    if (lane == 0) {
      const double lmax = lg[misc->idx[0]];
      double ev[kMaxK];
      double s = 0.0;
      for (int k = 0; k < K; ++k) { ev[k] = exp(lg[misc->idx[k]] - lmax); s += ev[k]; }
      for (int k = 0; k < K; ++k) {
        misc->wk[k] = (float)(ev[k] / s);
        if (cta == 0 && p.topk_idx) p.topk_idx[k] = misc->idx[k];
        if (cta == 0 && p.topk_w) p.topk_w[k] = misc->wk[k];
      }
    }
  }
  __syncthreads();
  if (tid < K && !*abort_flag) {
    const qe_expert ex = p.experts[misc->idx[tid]];
    const int bits = ex.gate.bits;
    if (!(bits == 4 || bits == 2) || !desc_ok(ex.gate, bits) || !desc_ok(ex.up, bits) ||
        !desc_ok(ex.down, bits)) {
      set_error(&ctl->err, QE_ERR_INVALID_ARG);
      misc->abort = 1;
    }
    misc->ex[tid] = ex;
  }
  __syncthreads();

  // ------------------------------------------------ expert phase (B and C)
  const int RB = g.RB, RC = g.RC, nIB = g.nIB;
  const int nBc = g.nB > cta ? (g.nB - cta + G - 1) / G : 0;
  const int own = g.nCB > cta ? (g.nCB - cta + G - 1) / G : 0;
  const int nCc = K * own;
  const int MR = g.max_own * RC;  // rows of one expert's slice of ycomb

  if (warp == kConsumerWarps) {
    // --------------------------------------------------------- producer
    int issuedB = 0, issuedC = 0;
    if (lane == 0 && !*abort_flag) {
      const uint64_t pol = policy_evict_first();
      const int gpr_h = H / kGroup, gpr_i = I / kGroup;
      for (int jb = 0; jb < nBc; ++jb) {
        const int gi = cta + G * jb;
        const int k = gi / nIB, r0 = (gi - k * nIB) * RB;
        const int slot = jb % g.nslotB;
        if (jb >= g.nslotB && !mbar_wait(&emptyB[slot], ((jb / g.nslotB) - 1) & 1, deadline, abort_flag)) {
          set_error(&ctl->err, QE_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        const qe_expert& ex = misc->ex[k];
        const int bits = ex.gate.bits;
        const uint32_t wbytes = (uint32_t)(RB * H * bits / 8);
        const uint32_t sbytes = (uint32_t)(RB * gpr_h * 2);
        unsigned char* dst = ringB + (size_t)slot * g.slotB;
        const size_t wrow = (size_t)H * bits / 32;
        mbar_arrive_expect_tx(&fullB[slot], 2 * wbytes + 4 * sbytes);
        bulk_g2s(dst, ex.gate.wq + (size_t)r0 * wrow, wbytes, &fullB[slot], pol);
        bulk_g2s(dst + RB * H / 2, ex.up.wq + (size_t)r0 * wrow, wbytes, &fullB[slot], pol);
        unsigned char* sdst = dst + RB * H;
        bulk_g2s(sdst, ex.gate.scales + (size_t)r0 * gpr_h, sbytes, &fullB[slot], pol);
        bulk_g2s(sdst + sbytes, ex.gate.biases + (size_t)r0 * gpr_h, sbytes, &fullB[slot], pol);
        bulk_g2s(sdst + 2 * sbytes, ex.up.scales + (size_t)r0 * gpr_h, sbytes, &fullB[slot], pol);
        bulk_g2s(sdst + 3 * sbytes, ex.up.biases + (size_t)r0 * gpr_h, sbytes, &fullB[slot], pol);
        issuedB = jb + 1;
        publish_issued(&misc->issuedB, issuedB);
      }
      for (int jc = 0; jc < nCc && !*abort_flag; ++jc) {
        const int k = jc / own, ob = jc - k * own;
        const int r0 = (cta + G * ob) * RC;
        const int slot = jc % g.nslotC;
        if (jc >= g.nslotC && !mbar_wait(&emptyC[slot], ((jc / g.nslotC) - 1) & 1, deadline, abort_flag)) {
          set_error(&ctl->err, QE_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        const qe_qmat& d = misc->ex[k].down;
        const uint32_t wbytes = (uint32_t)(RC * I * d.bits / 8);
        const uint32_t sbytes = (uint32_t)(RC * gpr_i * 2);
        unsigned char* dst = ringC + (size_t)slot * g.slotC;
        mbar_arrive_expect_tx(&fullC[slot], wbytes + 2 * sbytes);
        bulk_g2s(dst, d.wq + (size_t)r0 * I * d.bits / 32, wbytes, &fullC[slot], pol);
        bulk_g2s(dst + RC * I / 2, d.scales + (size_t)r0 * gpr_i, sbytes, &fullC[slot], pol);
        bulk_g2s(dst + RC * I / 2 + sbytes, d.biases + (size_t)r0 * gpr_i, sbytes, &fullC[slot], pol);
        issuedC = jc + 1;
        publish_issued(&misc->issuedC, issuedC);
      }
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------- consumers
    for (int j = warp; j < nBc + nCc; j += kConsumerWarps) {
      if (*abort_flag) break;
      if (j < nBc) {
        const int gi = cta + G * j;
        const int k = gi / nIB, r0 = (gi - k * nIB) * RB;
        const int slot = j % g.nslotB;
        if (!wait_issued(&misc->issuedB, j, deadline, abort_flag) ||
            !mbar_wait(&fullB[slot], (j / g.nslotB) & 1, deadline, abort_flag)) {
          if (lane == 0) { set_error(&ctl->err, QE_ERR_TIMEOUT); *abort_flag = 1; }
          break;
        }
        const unsigned char* sl = ringB + (size_t)slot * g.slotB;
        float* hdst = p.hbuf + (size_t)k * I + r0;
        if (misc->ex[k].gate.bits == 4)
          gateup_dispatch<4>(RB, sl, H, xp4, xsum, misc->xK, hdst, lane);
        else
          gateup_dispatch<2>(RB, sl, H, xp2, xsum, misc->xK, hdst, lane);
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&emptyB[slot]);
          __threadfence();
          red_release_add(&ctl->ready[k], 1u);
        }
      } else {
        const int jc = j - nBc;
        const int k = jc / own, ob = jc - k * own;
        const int dbits = misc->ex[k].down.bits;
        // stage h_k in shared memory (first warp to need it), or wait for it
        unsigned won = 0;
        if (lane == 0) won = (atomicCAS(&misc->claim[k], 0u, 1u) == 0u);
        won = __shfl_sync(0xffffffffu, won, 0);
        if (won) {
          int ok = 1;
          if (lane == 0) ok = wait_geq(&ctl->ready[k], (unsigned)nIB, deadline, abort_flag);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) {
            if (lane == 0) { set_error(&ctl->err, QE_ERR_TIMEOUT); *abort_flag = 1; }
            break;
          }
          float* hpk = hp + (size_t)k * I;
          float* hsk = hsum + (size_t)k * (I / 32);
          const float* hsrc = p.hbuf + (size_t)k * I;
          float am = 0.f;
          for (int c = lane; c < I; c += 32) {
            const float v = __ldcg(hsrc + c);
            hpk[c] = v;
            am = fmaxf(am, fabsf(v));
          }
          const int Eh = xscale_exponent(warp_max(am));
          for (int ch = 0; ch < I / 32; ++ch) {
            const int c = ch * 32 + lane;
            const float v = hpk[c];
            const float s = warp_sum(v);
            if (lane == 0) hsk[ch] = s;
            hpk[c] = dbits == 4 ? xprime_q4(v, c, Eh) : xprime_q2(v, c, Eh);
          }
          if (lane == 0) misc->hK[k] = acc_scale(Eh);
          __syncwarp();
          if (lane == 0) mbar_arrive(&hready[k]);
        } else {
          int ok = 1;
          if (lane == 0) ok = mbar_wait(&hready[k], 0, deadline, abort_flag);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) {
            if (lane == 0) { set_error(&ctl->err, QE_ERR_TIMEOUT); *abort_flag = 1; }
            break;
          }
        }
        const int slot = jc % g.nslotC;
        if (!wait_issued(&misc->issuedC, jc, deadline, abort_flag) ||
            !mbar_wait(&fullC[slot], (jc / g.nslotC) & 1, deadline, abort_flag)) {
          if (lane == 0) { set_error(&ctl->err, QE_ERR_TIMEOUT); *abort_flag = 1; }
          break;
        }
        const unsigned char* sl = ringC + (size_t)slot * g.slotC;
        float* ydst = ycomb + (size_t)k * MR + ob * RC;
        const float* hpk = hp + (size_t)k * I;
        const float* hsk = hsum + (size_t)k * (I / 32);
        if (dbits == 4)
          down_dispatch<4>(RC, sl, I, hpk, hsk, misc->hK[k], ydst, lane);
        else
          down_dispatch<2>(RC, sl, I, hpk, hsk, misc->hK[k], ydst, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&emptyC[slot]);
      }
    }
    // ------------------------------------------- combine of owned rows
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
    if (!*abort_flag) {
      for (int lr = tid; lr < own * RC; lr += kConsumerWarps * 32) {
        const int ob = lr / RC;
        const int r = (cta + G * ob) * RC + (lr - ob * RC);
        float acc = 0.f;
        for (int k = 0; k < K; ++k) acc += misc->wk[k] * ycomb[(size_t)k * MR + lr];
        if (p.add_residual) acc += load_x(p, r);
        p.out[r] = acc;
      }
    }
  }

  // --------------------------------------------------------------- exit
  __syncthreads();
  // Every copy issued must have landed before the CTA exits.  Without an
  // abort the consumers already waited for all of them and these waits
  // return at once; after an abort some were never consumed.
  if (warp == kConsumerWarps && lane == 0) {
    const uint64_t dl = gtimer() + p.budget_ns;
    volatile int never = 0;
    const int iB = misc->issuedB, iC = misc->issuedC;
    for (int s = 0; s < g.nslotB && s < iB; ++s) {
      const int last = s + ((iB - 1 - s) / g.nslotB) * g.nslotB;
      mbar_wait(&fullB[s], (last / g.nslotB) & 1, dl, &never);
    }
    for (int s = 0; s < g.nslotC && s < iC; ++s) {
      const int last = s + ((iC - 1 - s) / g.nslotC) * g.nslotC;
      mbar_wait(&fullC[s], (last / g.nslotC) & 1, dl, &never);
    }
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(&ctl->exit_ctr, 1u);
    if (prev == (unsigned)G - 1) {
      ctl->route_ctr = 0;
      for (int k = 0; k < kMaxK; ++k) ctl->ready[k] = 0;
      __threadfence();
      ctl->exit_ctr = 0;
      __threadfence();
    }
  }
}

// ------------------------------------------------------------ host side

static int align_up(int v, int a) { return (v + a - 1) / a * a; }
static int gcd_int(int a, int b) { while (b) { int t = a % b; a = b; b = t; } return a; }

int fused_geometry(int H, int E, int K, int I, int sms, int smem_optin, FusedGeometry* out) {
  FusedGeometry g{};
  // rows per item: keep every bulk copy a multiple of 16 bytes
  g.RB = 8 / gcd_int(H / kGroup, 8);
  if (g.RB < 2) g.RB = 2;
  g.RC = 8 / gcd_int(I / kGroup, 8);
  if (g.RC < 4) g.RC = 4;
  if (I % g.RB || H % g.RC) return QE_ERR_UNSUPPORTED;
  g.nIB = I / g.RB;
  g.nB = K * g.nIB;
  g.nCB = H / g.RC;
  g.grid = sms;
  g.max_own = (g.nCB + sms - 1) / sms;
  g.slotB = align_up(g.RB * H + 4 * g.RB * (H / kGroup) * 2, 128);
  g.slotC = align_up(g.RC * I / 2 + 2 * g.RC * (I / kGroup) * 2, 128);
  const int maxBc = (g.nB + sms - 1) / sms;
  const int maxCc = K * g.max_own;
  // fixed regions
  int off = 0;
  g.off_xp4 = off; off = align_up(off + 4 * H, 128);
  g.off_xp2 = off; off = align_up(off + 4 * H, 128);
  g.off_xs = off; off = align_up(off + 4 * (H / 32), 128);
  g.off_hp = off;
  const int hp_bytes = align_up(4 * K * I, 128);
  const int xg_bytes = 8 * H;
  g.off_hs = off + hp_bytes;
  off = align_up(off + (hp_bytes + 4 * K * (I / 32) > xg_bytes ? hp_bytes + 4 * K * (I / 32) : xg_bytes), 128);
  g.off_logit = off; off = align_up(off + 8 * E, 128);
  g.off_ycomb = off; off = align_up(off + 4 * K * g.max_own * g.RC, 128);
  g.off_misc = off; off = align_up(off + (int)sizeof(FusedMisc), 128);
  const int fixed = off;
  const int bar_bytes_per_slot = 16;
  int budget = smem_optin - fixed - 16 * kMaxK - 256;
  if (budget < 2 * (g.slotB + bar_bytes_per_slot) + (g.slotC + bar_bytes_per_slot))
    return QE_ERR_UNSUPPORTED;
  int nC = maxCc;
  const int capC = (budget * 2 / 5) / (g.slotC + bar_bytes_per_slot);
  if (nC > capC) nC = capC;
  if (nC < 1) nC = 1;
  int nB = (budget - nC * (g.slotC + bar_bytes_per_slot)) / (g.slotB + bar_bytes_per_slot);
  if (nB > maxBc) nB = maxBc;
  if (nB < 2) nB = 2;
  g.nslotB = nB;
  g.nslotC = nC;
  g.off_ringB = align_up(off, 1024);
  off = g.off_ringB + nB * g.slotB;
  g.off_ringC = align_up(off, 128);
  off = g.off_ringC + nC * g.slotC;
  g.off_bars = align_up(off, 16);
  off = g.off_bars + 8 * (2 * nB + 2 * nC + kMaxK);
  g.smem_bytes = align_up(off, 128);
  if (g.smem_bytes > smem_optin) return QE_ERR_UNSUPPORTED;
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
