// qe_ffn.cu -- expert FFN for T tokens x K selected experts as separate
// launches (moe_expert_ffn_q4/q2/mixed), and the weighted combine.
//
//   xprep : x' (pre-scaled activations) and 32-column sums per token
//   gateup: warp per (token, slot k, RB rows): g, u, h = silu(g) u
//   hprep : x' of h per (token, k), using the bits of the expert's down matrix
//   down  : warp per (token, k, RC rows): y
// Weights are read straight from HBM with 128-bit streaming loads.
#include <math.h>

#include "qe_device.cuh"

namespace qe {

constexpr int kFfnRB = 4;  // gate/up rows per warp item (of each matrix)
constexpr int kFfnRC = 4;  // down rows per warp item

static __device__ __forceinline__ bool ffn_desc_ok(const qe_expert& ex, int mode) {
  const int b = ex.gate.bits;
  if (!(b == 4 || b == 2)) return false;
  if (mode != 0 && b != mode) return false;
  const qe_qmat* m[3] = {&ex.gate, &ex.up, &ex.down};
  for (int i = 0; i < 3; ++i) {
    if (m[i]->bits != b || !m[i]->wq || !m[i]->scales || !m[i]->biases) return false;
    if (((uintptr_t)m[i]->wq & 15) || ((uintptr_t)m[i]->scales & 1) || ((uintptr_t)m[i]->biases & 1)) return false;
  }
  return true;
}

// Per-vector x' preparation: one CTA per vector of length n.
__global__ void __launch_bounds__(256) xprep_kernel(const float* __restrict__ src, int n, float* xp4,
                                                    float* xp2, float* xsum, int* xexp) {
  const int v = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* x = src + (size_t)v * n;
  __shared__ float red[8];
  __shared__ int s_e;
  float am = 0.f;
  for (int c = tid; c < n; c += 256) am = fmaxf(am, fabsf(x[c]));
  am = warp_max(am);
  if (lane == 0) red[warp] = am;
  __syncthreads();
  if (tid == 0) {
    float m = 0.f;
    for (int w = 0; w < 8; ++w) m = fmaxf(m, red[w]);
    s_e = xscale_exponent(m);
    xexp[v] = s_e;
  }
  __syncthreads();
  const int E = s_e;
  for (int ch = warp; ch < n / 32; ch += 8) {
    const int c = ch * 32 + lane;
    const float val = x[c];
    const float s = warp_sum(val);
    if (lane == 0) xsum[(size_t)v * (n / 32) + ch] = s;
    if (xp4) xp4[(size_t)v * n + xperm_q4(c)] = xprime_q4(val, c, E);
    if (xp2) xp2[(size_t)v * n + xperm_q2(c)] = xprime_q2(val, c, E);
  }
}

// x' of h: one CTA per (token, k); the down matrix's bits pick the form.
__global__ void __launch_bounds__(256) hprep_kernel(const FfnParams p) {
  const int a = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int I = p.I;
  const int e = p.idx[a];
  const int bits = p.experts[e].down.bits;
  const float* h = p.h + (size_t)a * I;
  const unsigned am_bits = p.hamax[a];
  const int E = xscale_exponent(__uint_as_float(am_bits));
  if (tid == 0) p.hexp[a] = E;
  for (int ch = warp; ch < I / 32; ch += 8) {
    const int c = ch * 32 + lane;
    const float v = h[c];
    const float s = warp_sum(v);
    if (lane == 0) p.hsum[(size_t)a * (I / 32) + ch] = s;
    if (bits == 4) p.hp[(size_t)a * I + xperm_q4(c)] = xprime_q4(v, c, E);
    else p.hp[(size_t)a * I + xperm_q2(c)] = xprime_q2(v, c, E);
  }
}

// NM matrices x R rows of each, one warp: returns the warp-reduced partials
// (row i of matrix m is reduced value m*R + i).
template <int NM, int R, int BITS>
static __device__ __forceinline__ float rows_dot_global(const qe_qmat* mats, int r0, int cols,
                                                        const float* __restrict__ xp,
                                                        const float* __restrict__ xs_sum, float xK,
                                                        int lane) {
  const int nch = cols / 32;  // 32-column chunks (4-bit: 4 words, 2-bit: 2 words)
  const int wpr = cols * BITS / 32;
  const int gpr = cols / kGroup;
  float yv[NM * R];
#pragma unroll
  for (int i = 0; i < NM * R; ++i) yv[i] = 0.f;
  for (int ch = lane; ch < nch; ch += 32) {
    float2 xs[16];
    const float4* src = (const float4*)(xp + ch * 32);  // global x' in pair order
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 v = __ldg(src + i);
      xs[2 * i] = make_float2(v.x, v.y);
      xs[2 * i + 1] = make_float2(v.z, v.w);
    }
    const int g = ch >> 1;
    const float xsum = xs_sum[ch];
#pragma unroll
    for (int m = 0; m < NM; ++m) {
#pragma unroll
      for (int rr = 0; rr < R; ++rr) {
        const size_t row = (size_t)(r0 + rr);
        float2 a;
        if (BITS == 4) a = dot32_q4(__ldcs((const ulonglong2*)(mats[m].wq + row * wpr) + ch), xs, make_float2(0.f, 0.f));
        else a = dot32_q2(__ldcs((const unsigned long long*)(mats[m].wq + row * wpr) + ch), xs, make_float2(0.f, 0.f));
        const float s = bf16f(__ldg(mats[m].scales + row * gpr + g));
        const float b = bf16f(__ldg(mats[m].biases + row * gpr + g));
        yv[m * R + rr] += s * xK * (a.x + a.y) + b * xsum;
      }
    }
  }
  return warp_reduce_rows<NM * R>(yv, lane);
}

__global__ void __launch_bounds__(256, 2) gateup_kernel(const FfnParams p) {
  const int lane = threadIdx.x & 31;
  const int item = (blockIdx.x * 256 + threadIdx.x) >> 5;
  const int nIB = p.I / kFfnRB;
  if (item >= p.T * p.K * nIB) return;
  const int a = item / nIB;  // assignment t*K + k
  const int r0 = (item - a * nIB) * kFfnRB;
  const int t = a / p.K;
  const int e = p.idx[a];
  const qe_expert ex = p.experts[e];
  if (!ffn_desc_ok(ex, p.mode)) {
    if (lane == 0 && r0 == 0) set_error(p.err, QE_ERR_INVALID_ARG);
    return;
  }
  const qe_qmat mats[2] = {ex.gate, ex.up};
  const int H = p.H;
  const float xK = acc_scale(p.xexp[t]);
  const float* xs_sum = p.xsum + (size_t)t * (H / 32);
  float s;
  if (ex.gate.bits == 4)
    s = rows_dot_global<2, kFfnRB, 4>(mats, r0, H, p.xp4 + (size_t)t * H, xs_sum, xK, lane);
  else
    s = rows_dot_global<2, kFfnRB, 2>(mats, r0, H, p.xp2 + (size_t)t * H, xs_sum, xK, lane);
  float am = 0.f;
#pragma unroll
  for (int rr = 0; rr < kFfnRB; ++rr) {
    const float gv = __shfl_sync(0xffffffffu, s, lane_of_reduced_row<2 * kFfnRB>(rr));
    const float uv = __shfl_sync(0xffffffffu, s, lane_of_reduced_row<2 * kFfnRB>(kFfnRB + rr));
    const float hv = gv / (1.0f + expf(-gv)) * uv;
    if (lane == rr) p.h[(size_t)a * p.I + r0 + rr] = hv;
    am = fmaxf(am, fabsf(hv));
  }
  if (lane == 0) atomicMax(p.hamax + a, __float_as_uint(am));
}

__global__ void __launch_bounds__(256, 2) down_kernel(const FfnParams p) {
  const int lane = threadIdx.x & 31;
  const int item = (blockIdx.x * 256 + threadIdx.x) >> 5;
  const int nOB = p.H / kFfnRC;
  if (item >= p.T * p.K * nOB) return;
  const int a = item / nOB;
  const int r0 = (item - a * nOB) * kFfnRC;
  const int e = p.idx[a];
  const qe_expert ex = p.experts[e];
  if (!ffn_desc_ok(ex, p.mode)) return;
  const int I = p.I;
  const float hK = acc_scale(p.hexp[a]);
  const float* hs = p.hsum + (size_t)a * (I / 32);
  float s;
  if (ex.down.bits == 4)
    s = rows_dot_global<1, kFfnRC, 4>(&ex.down, r0, I, p.hp + (size_t)a * I, hs, hK, lane);
  else
    s = rows_dot_global<1, kFfnRC, 2>(&ex.down, r0, I, p.hp + (size_t)a * I, hs, hK, lane);
#pragma unroll
  for (int rr = 0; rr < kFfnRC; ++rr)
    if (lane == lane_of_reduced_row<kFfnRC>(rr)) p.y[(size_t)a * p.H + r0 + rr] = s;
}

cudaError_t launch_ffn(const FfnParams& p, cudaStream_t s) {
  if (p.T <= 0) return cudaSuccess;
  const int A = p.T * p.K;
  if (!p.skip_xprep) xprep_kernel<<<p.T, 256, 0, s>>>(p.xn, p.H, p.xp4, p.xp2, p.xsum, p.xexp);
  cudaError_t e = cudaMemsetAsync(p.hamax, 0, sizeof(unsigned) * A, s);
  if (e != cudaSuccess) return e;
  const long items_gu = (long)A * (p.I / kFfnRB);
  gateup_kernel<<<(unsigned)((items_gu * 32 + 255) / 256), 256, 0, s>>>(p);
  hprep_kernel<<<A, 256, 0, s>>>(p);
  const long items_d = (long)A * (p.H / kFfnRC);
  down_kernel<<<(unsigned)((items_d * 32 + 255) / 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

// out[t,r] = sum_k w[t,k] y[t,k,r] (+ residual[t,r]); k ascending.
// residual is fp32, or bf16 bit patterns when res_bf16 is set.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y, const float* __restrict__ w,
                                                      const void* residual, int res_bf16, int T, int K, int H,
                                                      float* out) {
  const size_t n = (size_t)T * H;
  for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (size_t)gridDim.x * 256) {
    const size_t t = i / H, r = i - t * H;
    float acc = 0.f;
    for (int k = 0; k < K; ++k) acc += w[t * K + k] * y[(t * K + k) * H + r];
    if (residual) acc += res_bf16 ? bf16f(((const uint16_t*)residual)[i]) : ((const float*)residual)[i];
    out[i] = acc;
  }
}

cudaError_t launch_combine(const float* y, const float* w, const void* residual, int res_bf16, int T, int K,
                           int H, float* out, cudaStream_t s) {
  const size_t n = (size_t)T * H;
  if (n == 0) return cudaSuccess;
  size_t blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  combine_kernel<<<(unsigned)blocks, 256, 0, s>>>(y, w, residual, res_bf16, T, K, H, out);
  return cudaGetLastError();
}

}  // namespace qe
