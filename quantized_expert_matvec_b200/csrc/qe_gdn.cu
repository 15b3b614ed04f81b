// qe_gdn.cu -- GatedDeltaNet decode step: one token through the recurrent
// state of one linear-attention layer.
//
// lilting.ch, "Flash-MoE: running a 397B-parameter model on a 48 GB MacBook",
// section "GatedDeltaNet acceleration": 45 of the model's 60 layers update
// 64 heads x 128x128 state matrices per token, a recurrence written there as
// the BLAS calls scal, gemv and ger.  Read as the gated delta rule, per head:
//   S <- alpha S               (scal)
//   u <- S k                   (gemv: what the decayed state recalls at k)
//   S <- S + beta (v - u) k^T  (ger: write the correction at key k)
//   o <- S q                   (gemv: read out with the query)
// S is fp32 [heads][dv][dk], row i answering value component i.
//
// The step reads and writes the whole state once (8 MiB per layer at 64
// heads x 128 x 128) and does 5 flops per state element: it is bound by HBM
// bandwidth, so the kernel is plain coalesced float4 traffic with no tensor
// cores.  One warp owns RB consecutive rows of one head: each lane holds
// float4 column chunks of the RB rows (a 128-wide row is one 512-byte
// coalesced access), the RB recalls and the RB read-outs are each summed by
// one transposed warp reduction (a plain butterfly when RB = 1), and every row
// goes back to HBM right after its update.  The state is read once and written once with streaming
// (evict-first) accesses; k and q are read per warp from L2.
//
// Programmatic dependent launch: each CTA first prefetches its state rows into
// L2 (when the whole grid is resident) and lets the next kernel in the stream
// start, and only then waits for the
// previous kernel to finish before it reads anything.  The prefetch moves no
// data into registers, so it is correct even when the previous kernel wrote
// the same state (L2 is where the writes land); it only takes the DRAM
// latency of the state off the critical path.
#include <cuda_runtime.h>
#include <stdint.h>

#include "qe_device.cuh"
#include "qe_internal.h"

namespace qe {
namespace {

constexpr int kGdnWarps = 8;
constexpr int kGdnThreads = 32 * kGdnWarps;

struct GdnArgs {
  long long n_heads;
  int dk, dv;
  float* S;
  const float* q;
  const float* k;
  const float* v;
  const float* alpha;
  const float* beta;
  float* o;
  int prefetch;  // prefetch the state rows into L2 before the dependency wait
};

QE_DEV float dot4(const float4& a, const float4& b, float acc) {
  acc = fmaf(a.x, b.x, acc);
  acc = fmaf(a.y, b.y, acc);
  acc = fmaf(a.z, b.z, acc);
  return fmaf(a.w, b.w, acc);
}

// V: float4 chunks per lane and row (dk <= 128 V); RB: rows per warp.
template <int V, int RB>
__global__ void __launch_bounds__(kGdnThreads) qe_gdn_step_kernel(GdnArgs a) {
  const int lane = threadIdx.x & 31;
  const int nq = a.dk >> 2;                   // float4 per row
  const int wph = (a.dv + RB - 1) / RB;       // warps per head
  const long long gw = (long long)blockIdx.x * kGdnWarps + (threadIdx.x >> 5);
  const long long h = gw / wph;
  const bool live = h < a.n_heads;            // uniform over the warp
  const int r0 = (int)(gw - h * wph) * RB;
  float4* S4 = reinterpret_cast<float4*>(a.S);

  // prologue: pull this warp's state rows toward L2, then release the next
  // kernel and wait for the previous one
  if (live && a.prefetch) {
    const int lines = (a.dk + 31) >> 5;       // 128-byte lines per row
    for (int i = lane; i < RB * lines; i += 32) {
      const int r = i / lines;
      if (r0 + r < a.dv)
        prefetch_l2(a.S + ((size_t)h * a.dv + r0 + r) * a.dk + (size_t)(i - r * lines) * 32);
    }
  }
  grid_launch_dependents();
  grid_dependency_wait();
  if (!live) return;

  const float4* k4 = reinterpret_cast<const float4*>(a.k) + (size_t)h * nq;
  const float4* q4 = reinterpret_cast<const float4*>(a.q) + (size_t)h * nq;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 kk[V], qq[V];
#pragma unroll
  for (int c = 0; c < V; ++c) {
    const int j = lane + 32 * c;
    kk[c] = j < nq ? k4[j] : zero;
    qq[c] = j < nq ? q4[j] : zero;
  }
  float4 x[RB][V];
  float vi[RB];
#pragma unroll
  for (int r = 0; r < RB; ++r) {
    const bool ok = r0 + r < a.dv;
    const size_t row = (size_t)h * a.dv + r0 + r;
#pragma unroll
    for (int c = 0; c < V; ++c) {
      const int j = lane + 32 * c;
      x[r][c] = (ok && j < nq) ? __ldcs(S4 + row * nq + j) : zero;
    }
    vi[r] = ok ? a.v[row] : 0.f;
  }
  const float al = a.alpha[h], be = a.beta[h];

  // scal, then the recall gemv
  float part[RB];
#pragma unroll
  for (int r = 0; r < RB; ++r) {
    part[r] = 0.f;
#pragma unroll
    for (int c = 0; c < V; ++c) {
      x[r][c].x *= al;
      x[r][c].y *= al;
      x[r][c].z *= al;
      x[r][c].w *= al;
      part[r] = dot4(x[r][c], kk[c], part[r]);
    }
  }
  const float u_mine = warp_reduce_rows<RB>(part, lane);
  // ger: row r += beta (v_r - u_r) k, then the read-out gemv
#pragma unroll
  for (int r = 0; r < RB; ++r) {
    const float u = __shfl_sync(0xffffffffu, u_mine, lane_of_reduced_row<RB>(r));
    const float cr = be * (vi[r] - u);
    part[r] = 0.f;
#pragma unroll
    for (int c = 0; c < V; ++c) {
      x[r][c].x = fmaf(cr, kk[c].x, x[r][c].x);
      x[r][c].y = fmaf(cr, kk[c].y, x[r][c].y);
      x[r][c].z = fmaf(cr, kk[c].z, x[r][c].z);
      x[r][c].w = fmaf(cr, kk[c].w, x[r][c].w);
      part[r] = dot4(x[r][c], qq[c], part[r]);
    }
    const bool ok = r0 + r < a.dv;
    const size_t row = (size_t)h * a.dv + r0 + r;
#pragma unroll
    for (int c = 0; c < V; ++c) {
      const int j = lane + 32 * c;
      if (ok && j < nq) __stcs(S4 + row * nq + j, x[r][c]);
    }
  }
  const float o_mine = warp_reduce_rows<RB>(part, lane);
  const int my_row = reduced_row_of_lane<RB>(lane);
  if (lane == lane_of_reduced_row<RB>(my_row) && r0 + my_row < a.dv) a.o[(size_t)h * a.dv + r0 + my_row] = o_mine;
}

template <int V, int RB>
cudaError_t launch_gdn_t(const GdnArgs& a, cudaStream_t s) {
  const long long warps = a.n_heads * ((a.dv + RB - 1) / RB);
  const long long blocks = (warps + kGdnWarps - 1) / kGdnWarps;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(kGdnThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, qe_gdn_step_kernel<V, RB>, a);
}

template <int RB>
cudaError_t launch_gdn_rb(const GdnArgs& a, cudaStream_t s) {
  const int V = (a.dk / 4 + 31) / 32;
  switch (V) {
    case 1: return launch_gdn_t<1, RB>(a, s);
    case 2: return launch_gdn_t<2, RB>(a, s);
    case 3: return launch_gdn_t<3, RB>(a, s);
    default: return launch_gdn_t<4, RB>(a, s);
  }
}

}  // namespace

cudaError_t launch_gdn_step(long long n_heads, int dk, int dv, float* S, const float* q, const float* k,
                            const float* v, const float* alpha, const float* beta, float* o, int sms,
                            cudaStream_t s) {
  GdnArgs a{n_heads, dk, dv, S, q, k, v, alpha, beta, o, 0};
  // A grid that fits on the GPU at once (64 warps per SM) gets one row per
  // warp: the step is then a chain of latencies (dependency wait, L2, two
  // reductions), and the shortest chain wins.  Larger grids run in waves and
  // take four rows per warp, which keeps more bytes in flight per warp.  The
  // L2 prefetch pays only when the whole grid is resident and can start it
  // while the previous kernel drains; in later waves it only doubles requests.
  // (Measured at 45 layers x 64 heads x 128 x 128 and at 8 times the heads.)
  const long long rows = n_heads * (long long)dv;
  const long long resident_warps = (long long)sms * 64;
  if (rows <= resident_warps) {
    a.prefetch = 1;
    return launch_gdn_rb<1>(a, s);
  }
  a.prefetch = (rows + 3) / 4 <= resident_warps;
  return launch_gdn_rb<4>(a, s);
}

}  // namespace qe

using namespace qe;

extern "C" QE_API int gdn_decode_step(int n_heads, int dk, int dv, float* state, const float* q, const float* k,
                                      const float* v, const float* alpha, const float* beta, float* out,
                                      qe_stream_t stream) {
  if (n_heads < 0 || dv < 1 || dk < 4 || dk > 512 || (dk & 3))
    return fail(QE_ERR_INVALID_ARG, "gdn_decode_step: need n_heads >= 0, dv >= 1, 4 <= dk <= 512, dk %% 4 == 0 "
                                    "(got %d, %d, %d)", n_heads, dv, dk);
  if (n_heads == 0) return QE_OK;
  if (!state || !q || !k || !v || !alpha || !beta || !out) return fail(QE_ERR_INVALID_ARG, "gdn_decode_step: NULL pointer");
  if (((uintptr_t)state | (uintptr_t)q | (uintptr_t)k) & 15)
    return fail(QE_ERR_INVALID_ARG, "gdn_decode_step: state, q and k must be 16-byte aligned");
  if (((uintptr_t)v | (uintptr_t)alpha | (uintptr_t)beta | (uintptr_t)out) & 3)
    return fail(QE_ERR_INVALID_ARG, "gdn_decode_step: v, alpha, beta and out must be 4-byte aligned");
  // out must not overlap any input (other warps still read q, k, v, alpha, beta
  // and the state while a warp writes its outputs)
  const uintptr_t o0 = (uintptr_t)out, o1 = o0 + sizeof(float) * (size_t)n_heads * dv;
  auto overlaps = [&](const void* p, size_t bytes) {
    const uintptr_t p0 = (uintptr_t)p, p1 = p0 + bytes;
    return p0 < o1 && o0 < p1;
  };
  const size_t nh = (size_t)n_heads;
  if (overlaps(state, 4 * nh * dv * dk) || overlaps(q, 4 * nh * dk) || overlaps(k, 4 * nh * dk) ||
      overlaps(v, 4 * nh * dv) || overlaps(alpha, 4 * nh) || overlaps(beta, 4 * nh))
    return fail(QE_ERR_INVALID_ARG, "gdn_decode_step: out overlaps an input");
  static int sms_of[64];  // SM count per device, read once
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
    if (!sms_of[dev]) cudaDeviceGetAttribute(&sms_of[dev], cudaDevAttrMultiProcessorCount, dev);
    if (sms_of[dev] > 0) sms = sms_of[dev];
  }
  const cudaError_t e = launch_gdn_step(n_heads, dk, dv, state, q, k, v, alpha, beta, out, sms, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "gdn_decode_step launch");
  return QE_OK;
}
