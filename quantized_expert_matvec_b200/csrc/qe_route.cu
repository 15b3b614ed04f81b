// qe_route.cu -- RMSNorm + router + top-K for T tokens (moe_route and the
// batched layer step).  Norm and router logits are evaluated in double
// precision so the expert choice is an fp64 decision.
#include <cooperative_groups.h>
#include <cuda_fp16.h>
#include <math.h>

#include "qe_device.cuh"

namespace qe {

namespace cg = cooperative_groups;

// One CTA per token: two-pass RMSNorm; x*gamma (fp64) for the router; xn
// (fp32) and, if requested, x' for the expert matvecs with its 32-column sums.
__global__ void __launch_bounds__(256) route_norm_kernel(const RouteParams p) {
  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H;
  __shared__ double red_d[8];
  __shared__ float red_f[8];
  __shared__ double s_rinv;
  __shared__ int s_exp;
  auto ldx = [&](int c) -> double {
    return p.x_bf16 ? (double)bf16f(((const uint16_t*)p.x)[(size_t)t * H + c])
                    : (double)((const float*)p.x)[(size_t)t * H + c];
  };
  double ss = 0.0;
  for (int c = tid; c < H; c += 256) { const double v = ldx(c); ss += v * v; }
  ss = warp_sum_d(ss);
  if (lane == 0) red_d[warp] = ss;
  __syncthreads();
  if (tid == 0) {
    double a = 0.0;
    for (int w = 0; w < 8; ++w) a += red_d[w];
    s_rinv = 1.0 / sqrt(a / (double)H + (double)p.eps);
    p.rinv[t] = s_rinv;
  }
  __syncthreads();
  const double rinv = s_rinv;
  float amax = 0.f;
  for (int c = tid; c < H; c += 256) {
    const double xv = ldx(c);
    const double gm = p.gamma ? (double)p.gamma[c] : 1.0;
    p.xg[(size_t)t * H + c] = xv * gm;
    const float xn = (float)(xv * rinv * gm);
    if (p.xn_out) p.xn_out[(size_t)t * H + c] = xn;
    if (p.xn_ws) p.xn_ws[(size_t)t * H + c] = xn;
    if (p.xh) p.xh[(size_t)t * H + c] = __half_as_ushort(__float2half_rn(xn));
    amax = fmaxf(amax, fabsf(xn));
  }
  if (!p.xp4) return;
  amax = warp_max(amax);
  if (lane == 0) red_f[warp] = amax;
  __syncthreads();
  if (tid == 0) {
    float m = 0.f;
    for (int w = 0; w < 8; ++w) m = fmaxf(m, red_f[w]);
    s_exp = xscale_exponent(m);
    p.xexp[t] = s_exp;
  }
  __syncthreads();
  const int Ex = s_exp;
  for (int ch = warp; ch < H / 32; ch += 8) {
    const int c = ch * 32 + lane;
    const float v = (float)(ldx(c) * rinv * (p.gamma ? (double)p.gamma[c] : 1.0));
    const float s = warp_sum(v);
    if (lane == 0) p.xsum[(size_t)t * (H / 32) + ch] = s;
    p.xp4[(size_t)t * H + xperm_q4(c)] = xprime_q4(v, c, Ex);
    p.xp2[(size_t)t * H + xperm_q2(c)] = xprime_q2(v, c, Ex);
  }
}

// Router logits for few tokens: one warp per expert row, all T (<= 4) tokens.
__global__ void __launch_bounds__(256) route_logits_gemv_kernel(const RouteParams p) {
  const int warp = (blockIdx.x * 256 + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int H = p.H, T = p.T;
  if (warp >= p.E) return;
  const int e = warp;
  const float4* wrow = (const float4*)(p.router_w + (size_t)e * H);
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
  for (int i = lane; i < H / 4; i += 32) {
    const float4 wv = __ldg(wrow + i);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      if (t >= T) break;
      const double* xx = p.xg + (size_t)t * H + 4 * i;
      double a = acc[t];
      a = fma((double)wv.x, xx[0], a);
      a = fma((double)wv.y, xx[1], a);
      a = fma((double)wv.z, xx[2], a);
      a = fma((double)wv.w, xx[3], a);
      acc[t] = a;
    }
  }
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    if (t >= T) break;
    const double s = warp_sum_d(acc[t]);
    if (lane == 0)
      p.logits[(size_t)t * p.E + e] = s * p.rinv[t] + (p.offset ? (double)p.offset[e] : 0.0);
  }
}

// Router logits for many tokens: fp64 tiled product.  A CTA takes a tile of
// 64 experts x 64 tokens and one eighth of the hidden columns; the eight
// CTAs of a thread-block cluster take the eight eighths of the same tile and
// add their partial tiles through distributed shared memory, in rank order,
// so the result does not depend on timing.  Each thread keeps 4 x 4 partial
// sums; columns come in 32-wide chunks, loaded into registers one chunk
// ahead and staged in shared memory (W converted to fp64), transposed to
// [k][expert] and [k][token] with the row index XOR-ed by rsw(k) (a multiple
// of 4): the transposing stores spread over the banks and the compute reads
// of four consecutive rows stay contiguous.
constexpr int kRT = 64;     // experts and tokens per tile
constexpr int kRK = 32;     // columns per chunk
constexpr int kRSplit = 8;  // CTAs per cluster (column eighths)
static __device__ __forceinline__ int rsw(int k) { return ((k >> 2) & 3) << 2; }
__global__ void __cluster_dims__(kRSplit, 1, 1) __launch_bounds__(256)
    route_logits_tiled_kernel(const RouteParams p) {
  __shared__ __align__(16) double sbuf[2 * kRK * kRT];  // sW [k][e], sX [k][t]; later the partial tile [t][e]
  double* sW = sbuf;
  double* sX = sbuf + kRK * kRT;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int H = p.H, E = p.E, T = p.T;
  const int tiles_e = (E + kRT - 1) / kRT;
  const int tile = blockIdx.x / kRSplit;
  const int e0 = (tile % tiles_e) * kRT, t0 = (tile / tiles_e) * kRT;
  const int nch = H / kRK;  // H is a multiple of 64
  const int ch0 = rank * nch / kRSplit, ch1 = (rank + 1) * nch / kRSplit;
  const int tid = threadIdx.x;
  const int te = (tid & 15) * 4, tt = (tid >> 4) * 4;
  double acc[4][4] = {};
  float4 wn[2];
  double2 xn[4];
  auto fetch = [&](int ch) {
    const int k0 = ch * kRK;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int u = tid + 256 * j, r = u >> 3, c4 = (u & 7) * 4;
      wn[j] = e0 + r < E ? __ldg((const float4*)(p.router_w + (size_t)(e0 + r) * H + k0 + c4))
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int u = tid + 256 * j, r = u >> 4, c2 = (u & 15) * 2;
      xn[j] = t0 + r < T ? *(const double2*)(p.xg + (size_t)(t0 + r) * H + k0 + c2) : make_double2(0.0, 0.0);
    }
  };
  if (ch0 < ch1) fetch(ch0);
  for (int ch = ch0; ch < ch1; ++ch) {
    __syncthreads();  // the previous chunk is consumed
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int u = tid + 256 * j, r = u >> 3, c4 = (u & 7) * 4;
      sW[(c4 + 0) * kRT + (r ^ rsw(c4 + 0))] = wn[j].x;
      sW[(c4 + 1) * kRT + (r ^ rsw(c4 + 1))] = wn[j].y;
      sW[(c4 + 2) * kRT + (r ^ rsw(c4 + 2))] = wn[j].z;
      sW[(c4 + 3) * kRT + (r ^ rsw(c4 + 3))] = wn[j].w;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int u = tid + 256 * j, r = u >> 4, c2 = (u & 15) * 2;
      sX[(c2 + 0) * kRT + (r ^ rsw(c2 + 0))] = xn[j].x;
      sX[(c2 + 1) * kRT + (r ^ rsw(c2 + 1))] = xn[j].y;
    }
    __syncthreads();
    if (ch + 1 < ch1) fetch(ch + 1);
#pragma unroll 4
    for (int k = 0; k < kRK; ++k) {
      const int we = te ^ rsw(k), xt = tt ^ rsw(k);
      const double2 wa = *(const double2*)(sW + k * kRT + we), wb = *(const double2*)(sW + k * kRT + we + 2);
      const double2 xa = *(const double2*)(sX + k * kRT + xt), xb = *(const double2*)(sX + k * kRT + xt + 2);
      const double w[4] = {wa.x, wa.y, wb.x, wb.y}, x[4] = {xa.x, xa.y, xb.x, xb.y};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fma(w[i], x[j], acc[i][j]);
    }
  }
  __syncthreads();
  double* part = sbuf;  // [t][e] partial tile of this CTA's columns
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) part[(tt + j) * kRT + te + i] = acc[i][j];
  cluster.sync();
  // rank r adds the partials of token rows [8r, 8r + 8)
  for (int u = tid; u < kRT * kRT / kRSplit; u += 256) {
    const int tl = rank * (kRT / kRSplit) + u / kRT, el = u % kRT;
    double sum = 0.0;
#pragma unroll
    for (int q = 0; q < kRSplit; ++q) sum += cluster.map_shared_rank(part, q)[tl * kRT + el];
    const int t = t0 + tl, e = e0 + el;
    if (t < T && e < E) p.logits[(size_t)t * E + e] = sum * p.rinv[t] + (p.offset ? (double)p.offset[e] : 0.0);
  }
  cluster.sync();  // no CTA leaves while another still reads its partial tile
}

// Top-K + renormalised softmax weights: one warp per token.
__global__ void __launch_bounds__(256) route_topk_kernel(const RouteParams p) {
  const int t = (blockIdx.x * 256 + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (t >= p.T) return;
  const int E = p.E, K = p.K;
  const double* lg = p.logits + (size_t)t * E;
  unsigned taken = 0;
  int idx[kMaxK];
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
      if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) { bv = ov; bi = oi; }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    idx[k] = bi;
  }
  if (lane == 0) {
    const double lmax = lg[idx[0]];
    double ev[kMaxK];
    double s = 0.0;
    for (int k = 0; k < K; ++k) { ev[k] = exp(lg[idx[k]] - lmax); s += ev[k]; }
    for (int k = 0; k < K; ++k) {
      p.idx[(size_t)t * K + k] = idx[k];
      p.w[(size_t)t * K + k] = (float)(ev[k] / s);
    }
  }
}

cudaError_t launch_route(const RouteParams& p, cudaStream_t s) {
  if (p.T <= 0) return cudaSuccess;
  route_norm_kernel<<<p.T, 256, 0, s>>>(p);
  if (p.T <= 4) {
    const int blocks = (p.E * 32 + 255) / 256;
    route_logits_gemv_kernel<<<blocks, 256, 0, s>>>(p);
  } else {
    const int tiles = ((p.E + kRT - 1) / kRT) * ((p.T + kRT - 1) / kRT);
    route_logits_tiled_kernel<<<tiles * kRSplit, 256, 0, s>>>(p);
  }
  route_topk_kernel<<<(p.T * 32 + 255) / 256, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace qe
