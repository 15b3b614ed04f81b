// qe_route.cu -- RMSNorm + router + top-K for T tokens (moe_route and the
// batched layer step).  Norm and router logits are evaluated in double
// precision so the expert choice is an fp64 decision.
#include <cuda_fp16.h>
#include <math.h>

#include "qe_device.cuh"

namespace qe {

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

// Router logits for many tokens: fp64 tiled product, 32 experts x 32
// tokens per CTA (enough CTAs to cover the SMs), 2x2 outputs per thread,
// 32-column steps through shared memory with float4 loads of W.
constexpr int kRT = 32, kRK = 32;
__global__ void __launch_bounds__(256) route_logits_tiled_kernel(const RouteParams p) {
  __shared__ __align__(16) double sW[kRK][kRT + 2];
  __shared__ __align__(16) double sX[kRK][kRT + 2];
  const int H = p.H, E = p.E, T = p.T;
  const int e0 = blockIdx.x * kRT, t0 = blockIdx.y * kRT;
  const int tid = threadIdx.x;
  const int te = (tid & 15) * 2, tt = (tid >> 4) * 2;
  double acc[2][2] = {};
  for (int c0 = 0; c0 < H; c0 += kRK) {
    // 32 rows x 32 columns of W (fp32 -> fp64) and of x*gamma (fp64)
    {
      const int r = tid >> 3, c4 = (tid & 7) * 4;
      const int e = e0 + r, t = t0 + r;
      if (e < E) {
        const float4 v = *(const float4*)(p.router_w + (size_t)e * H + c0 + c4);
        sW[c4][r] = v.x; sW[c4 + 1][r] = v.y; sW[c4 + 2][r] = v.z; sW[c4 + 3][r] = v.w;
      } else {
        sW[c4][r] = 0.0; sW[c4 + 1][r] = 0.0; sW[c4 + 2][r] = 0.0; sW[c4 + 3][r] = 0.0;
      }
      for (int u = 0; u < 4; ++u) sX[c4 + u][r] = t < T ? p.xg[(size_t)t * H + c0 + c4 + u] : 0.0;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < kRK; ++c) {
      const double w0 = sW[c][te], w1 = sW[c][te + 1];
      const double x0 = sX[c][tt], x1 = sX[c][tt + 1];
      acc[0][0] = fma(w0, x0, acc[0][0]);
      acc[0][1] = fma(w0, x1, acc[0][1]);
      acc[1][0] = fma(w1, x0, acc[1][0]);
      acc[1][1] = fma(w1, x1, acc[1][1]);
    }
    __syncthreads();
  }
  for (int a = 0; a < 2; ++a)
    for (int b = 0; b < 2; ++b) {
      const int e = e0 + te + a, t = t0 + tt + b;
      if (e < E && t < T)
        p.logits[(size_t)t * E + e] = acc[a][b] * p.rinv[t] + (p.offset ? (double)p.offset[e] : 0.0);
    }
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
    dim3 grid((p.E + kRT - 1) / kRT, (p.T + kRT - 1) / kRT);
    route_logits_tiled_kernel<<<grid, 256, 0, s>>>(p);
  }
  route_topk_kernel<<<(p.T * 32 + 255) / 256, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace qe
