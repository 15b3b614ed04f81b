// qe_grouped.cu -- batched layer step (T tokens per step): the (token, k)
// assignments are grouped by expert so each selected expert's weights are
// streamed from HBM once per step and reused by all of its tokens.
//
//   group kernel : counting sort of the T*K assignments by expert (stable:
//                  ascending assignment id inside an expert)
//   expert kernel: persistent CTAs take whole experts from a shared counter;
//                  per expert: stage the x' of its tokens in shared memory,
//                  gate/up rows (a warp takes blocks of kRowBlk rows and
//                  runs every token over them; after the first token the
//                  block's packed words come from L1),
//                  h = silu(g) u in shared memory, then down rows ->
//                  y[assignment][H]
//   combine      : out[t] = sum_k w[t,k] y[t*K+k] (+ x[t])
// Up to kTokTile tokens of an expert are processed per pass over its weights.
#include <math.h>

#include "qe_device.cuh"

namespace qe {

constexpr int kGWarps = 16;
constexpr int kGThreads = kGWarps * 32;
constexpr int kTokTile = 8;  // tokens staged per pass over an expert's weights
constexpr int kRowBlk = 4;   // rows per warp block

// Round a count of 4-byte elements up to a multiple of 4 (16 bytes).
static __host__ __device__ __forceinline__ int al4(int n) { return (n + 3) & ~3; }

// -------------------------------------------------------------- grouping
__global__ void __launch_bounds__(1024) group_kernel(const int32_t* __restrict__ idx, int A, int E, int* count,
                                                     int* start, int* list, int* order, int* n_active,
                                                     int* err) {
  extern __shared__ int sh[];
  int* cnt = sh;          // [E]
  int* cur = sh + E;      // [E]
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int a = tid; a < A; a += blockDim.x) {
    const int e = idx[a];
    if (e < 0 || e >= E) { set_error(err, QE_ERR_INVALID_ARG); continue; }
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  if (tid == 0) {
    int s = 0, na = 0;
    for (int e = 0; e < E; ++e) {
      start[e] = s;
      cur[e] = s;
      count[e] = cnt[e];
      s += cnt[e];
      if (cnt[e] > 0) order[na++] = e;
    }
    start[E] = s;
    *n_active = na;
  }
  __syncthreads();
  for (int a = tid; a < A; a += blockDim.x) {
    const int e = idx[a];
    if (e < 0 || e >= E) continue;
    list[atomicAdd(&cur[e], 1)] = a;
  }
  __syncthreads();
  // restore ascending assignment order inside each expert (lists are short)
  for (int e = tid; e < E; e += blockDim.x) {
    int* l = list + start[e];
    const int n = cnt[e];
    for (int i = 1; i < n; ++i) {
      const int v = l[i];
      int j = i - 1;
      while (j >= 0 && l[j] > v) { l[j + 1] = l[j]; --j; }
      l[j + 1] = v;
    }
  }
  __syncthreads();
  // larger groups first so the persistent CTAs end together: a stable
  // counting sort of the active experts by descending token count
  if (tid == 0) {
    int na = 0, maxc = 0;
    for (int e = 0; e < E; ++e) maxc = cnt[e] > maxc ? cnt[e] : maxc;
    for (int c = maxc; c >= 1; --c)
      for (int e = 0; e < E; ++e)
        if (cnt[e] == c) order[na++] = e;
  }
}

struct ExpertParams {
  int H, I, K, T;
  const qe_expert* experts;
  const float* xp4;   // [T][H] x' (linear layout, global)
  const float* xp2;
  const float* xsum;  // [T][H/32]
  const int* xexp;    // [T]
  const int* start;
  const int* list;
  const int* order;
  const int* n_active;
  int* work;          // shared work counter (reset by the caller)
  float* y;           // [T*K][H]
  int* err;
  int tile;           // tokens per pass over an expert's weights
};

// Stage the x' (4- or 2-bit form, swizzled) and 32-column sums of `nt`
// tokens into shared memory.
static __device__ void stage_tokens(const ExpertParams& p, int bits, const int* toks, int nt, float* xs_sm,
                                    float* sum_sm, float* xk_sm) {
  const int H = p.H;
  const float* src = bits == 4 ? p.xp4 : p.xp2;
  for (int i = threadIdx.x; i < nt * H; i += kGThreads) {
    const int t = i / H, c = i - t * H;
    const float v = src[(size_t)toks[t] * H + c];
    xs_sm[t * H + (bits == 4 ? swz_q4(c) : swz_q2(c))] = v;
  }
  for (int i = threadIdx.x; i < nt * (H / 32); i += kGThreads) {
    const int t = i / (H / 32), c = i - t * (H / 32);
    sum_sm[i] = p.xsum[(size_t)toks[t] * (H / 32) + c];
  }
  if (threadIdx.x < nt) xk_sm[threadIdx.x] = acc_scale(p.xexp[toks[threadIdx.x]]);
}

// kRowBlk rows (r0 .. r0+nv-1) of a packed matrix with `cols` columns
// against one token's x' (shared memory): acc[i] collects this lane's partial
// sum of row r0+i.  The block's packed rows are small (kRowBlk * cols/2
// bytes), so the tokens after the first read them from L1.
template <int BITS>
static __device__ __forceinline__ void block_rows(const qe_qmat& m, int r0, int nv, int cols, const float* xs_t,
                                                  const float* sum_t, float xk, float (&acc)[kRowBlk], int lane) {
  const int gpr = cols / kGroup;
  const size_t rowb = (size_t)cols * BITS / 8;
  const unsigned char* base = (const unsigned char*)m.wq + (size_t)r0 * rowb;
  for (int lc = lane; lc < cols / 32; lc += 32) {
    uint4 w[kRowBlk];
    uint32_t sb[kRowBlk];
    const int g = lc >> 1;
#pragma unroll
    for (int i = 0; i < kRowBlk; ++i) {
      if (i < nv) {
        const unsigned char* rp = base + (size_t)i * rowb;
        if (BITS == 4) {
          w[i] = __ldg((const uint4*)rp + lc);
        } else {
          const uint2 v = __ldg((const uint2*)rp + lc);
          w[i] = make_uint4(v.x, v.y, 0u, 0u);
        }
        const size_t gi = (size_t)(r0 + i) * gpr + g;
        sb[i] = (uint32_t)__ldg(m.scales + gi) | ((uint32_t)__ldg(m.biases + gi) << 16);
      }
    }
    float2 xs[16];
    if (BITS == 4) load_xs32_q4(xs_t, lc, xs);
    else load_xs32_q2(xs_t, lc, xs);
    const float xsum = sum_t[lc];
#pragma unroll
    for (int i = 0; i < kRowBlk; ++i) {
      if (i < nv) {
        const float2 a = BITS == 4 ? dot32_q4(w[i], xs, make_float2(0.f, 0.f))
                                   : dot32_q2(make_uint2(w[i].x, w[i].y), xs, make_float2(0.f, 0.f));
        acc[i] += bf16f(sb[i] & 0xFFFFu) * xk * (a.x + a.y) + bf16f(sb[i] >> 16) * xsum;
      }
    }
  }
}

__global__ void __launch_bounds__(kGThreads, 1) grouped_expert_kernel(const ExpertParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int H = p.H, I = p.I, tile = p.tile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // every region starts on a 16-byte boundary (float4 reads of x' and h')
  float* xs_sm = (float*)smem;                            // [tile][H]
  float* xsum_sm = xs_sm + al4(tile * H);                 // [tile][H/32]
  float* xk_sm = xsum_sm + al4(tile * (H / 32));          // [tile]
  float* h_sm = xk_sm + al4(tile);                        // [tile][I] raw h
  float* hp_sm = h_sm + al4(tile * I);                    // [tile][I] x' of h
  float* hsum_sm = hp_sm + al4(tile * I);                 // [tile][I/32]
  float* hk_sm = hsum_sm + al4(tile * (I / 32));          // [tile]
  int* toks = (int*)(hk_sm + al4(tile));                  // [tile]
  int* asg = toks + al4(tile);                            // [tile]
  unsigned* hmax = (unsigned*)(asg + al4(tile));          // [tile]
  __shared__ int s_item;
  __shared__ qe_expert s_ex;
  const int na = *p.n_active;
  for (;;) {
    if (threadIdx.x == 0) s_item = atomicAdd(p.work, 1);
    __syncthreads();
    const int item = s_item;
    __syncthreads();
    if (item >= na) break;
    const int e = p.order[item];
    // the descriptor lives in shared memory, not in 24 registers
    if (threadIdx.x == 0) s_ex = p.experts[e];
    __syncthreads();
    const qe_expert& ex = s_ex;
    const int bits = ex.gate.bits;
    if (!(bits == 4 || bits == 2) || ex.up.bits != bits || ex.down.bits != bits || !ex.gate.wq || !ex.up.wq ||
        !ex.down.wq || ((uintptr_t)ex.gate.wq & 15) || ((uintptr_t)ex.up.wq & 15) || ((uintptr_t)ex.down.wq & 15)) {
      if (threadIdx.x == 0) set_error(p.err, QE_ERR_INVALID_ARG);
      continue;
    }
    const int n = p.start[e + 1] - p.start[e];
    for (int t0 = 0; t0 < n; t0 += tile) {
      const int nt = n - t0 < tile ? n - t0 : tile;
      if (threadIdx.x < nt) {
        const int a = p.list[p.start[e] + t0 + threadIdx.x];
        asg[threadIdx.x] = a;
        toks[threadIdx.x] = a / p.K;
        hmax[threadIdx.x] = 0u;
      }
      __syncthreads();
      stage_tokens(p, bits, toks, nt, xs_sm, xsum_sm, xk_sm);
      __syncthreads();
      // -------------------------------- gate/up: kRowBlk-row blocks per warp
      for (int r0 = warp * kRowBlk; r0 < I; r0 += kGWarps * kRowBlk) {
        const int nv = I - r0 < kRowBlk ? I - r0 : kRowBlk;
        for (int t = 0; t < nt; ++t) {
          float ga[kRowBlk], ua[kRowBlk];
#pragma unroll
          for (int i = 0; i < kRowBlk; ++i) { ga[i] = 0.f; ua[i] = 0.f; }
          const float* xst = xs_sm + t * H;
          const float* sst = xsum_sm + t * (H / 32);
          if (bits == 4) {
            block_rows<4>(ex.gate, r0, nv, H, xst, sst, xk_sm[t], ga, lane);
            block_rows<4>(ex.up, r0, nv, H, xst, sst, xk_sm[t], ua, lane);
          } else {
            block_rows<2>(ex.gate, r0, nv, H, xst, sst, xk_sm[t], ga, lane);
            block_rows<2>(ex.up, r0, nv, H, xst, sst, xk_sm[t], ua, lane);
          }
          const float gv = warp_reduce_rows<kRowBlk>(ga, lane);
          const float uv = warp_reduce_rows<kRowBlk>(ua, lane);
          const int i = reduced_row_of_lane<kRowBlk>(lane);
          if (lane == lane_of_reduced_row<kRowBlk>(i) && i < nv) {
            const float hv = gv / (1.0f + expf(-gv)) * uv;
            h_sm[t * I + r0 + i] = hv;
            atomicMax(&hmax[t], __float_as_uint(fabsf(hv)));
          }
        }
      }
      __syncthreads();
      // -------------------------------------------------- x' of h, per token
      for (int i = threadIdx.x; i < nt * I; i += kGThreads) {
        const int t = i / I, c = i - t * I;
        const int Eh = xscale_exponent(__uint_as_float(hmax[t]));
        hp_sm[t * I + (bits == 4 ? swz_q4(c) : swz_q2(c))] =
            bits == 4 ? xprime_q4(h_sm[i], c, Eh) : xprime_q2(h_sm[i], c, Eh);
      }
      for (int i = warp; i < nt * (I / 32); i += kGWarps) {
        const int t = i / (I / 32), ch = i - t * (I / 32);
        const float sm = warp_sum(h_sm[t * I + ch * 32 + lane]);
        if (lane == 0) hsum_sm[i] = sm;
      }
      if (threadIdx.x < nt) hk_sm[threadIdx.x] = acc_scale(xscale_exponent(__uint_as_float(hmax[threadIdx.x])));
      __syncthreads();
      // ----------------------------------- down: kRowBlk-row blocks per warp
      for (int r0 = warp * kRowBlk; r0 < H; r0 += kGWarps * kRowBlk) {
        const int nv = H - r0 < kRowBlk ? H - r0 : kRowBlk;
        for (int t = 0; t < nt; ++t) {
          float ya[kRowBlk];
#pragma unroll
          for (int i = 0; i < kRowBlk; ++i) ya[i] = 0.f;
          if (bits == 4) block_rows<4>(ex.down, r0, nv, I, hp_sm + t * I, hsum_sm + t * (I / 32), hk_sm[t], ya, lane);
          else block_rows<2>(ex.down, r0, nv, I, hp_sm + t * I, hsum_sm + t * (I / 32), hk_sm[t], ya, lane);
          const float yv = warp_reduce_rows<kRowBlk>(ya, lane);
          const int i = reduced_row_of_lane<kRowBlk>(lane);
          if (lane == lane_of_reduced_row<kRowBlk>(i) && i < nv) p.y[(size_t)asg[t] * H + r0 + i] = yv;
        }
      }
      __syncthreads();
    }
  }
}

// Shared memory of the expert kernel for a token tile of `tile`.
size_t grouped_smem_bytes(int H, int I, int tile) {
  const size_t f = (size_t)al4(tile * H) + al4(tile * (H / 32)) + al4(tile) + 2 * (size_t)al4(tile * I) +
                   al4(tile * (I / 32)) + al4(tile);
  return 4 * (f + 3 * (size_t)al4(tile)) + 64;
}

// Largest token tile (<= kTokTile) whose buffers fit in shared memory.
int grouped_tile(int H, int I, int smem_optin) {
  for (int t = kTokTile; t >= 1; --t)
    if (grouped_smem_bytes(H, I, t) <= (size_t)smem_optin) return t;
  return 0;
}

cudaError_t launch_grouped(const GroupedParams& gp, cudaStream_t s) {
  const int A = gp.T * gp.K;
  if (A == 0) return cudaSuccess;
  int* n_active = gp.grp_count + gp.E;  // the workspace reserves E+2 ints
  int* work = n_active + 1;
  const size_t gsm = sizeof(int) * 2 * (size_t)gp.E;
  group_kernel<<<1, 1024, gsm, s>>>(gp.idx, A, gp.E, gp.grp_count, gp.grp_start, gp.grp_list, gp.grp_order,
                                    n_active, gp.err);
  cudaError_t e = cudaMemsetAsync(work, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  cudaFuncAttributes fa{};
  e = cudaFuncGetAttributes(&fa, grouped_expert_kernel);
  if (e != cudaSuccess) return e;
  optin -= (int)fa.sharedSizeBytes;  // static shared memory counts against the limit
  ExpertParams p{};
  p.H = gp.H; p.I = gp.I; p.K = gp.K; p.T = gp.T;
  p.tile = grouped_tile(gp.H, gp.I, optin);
  if (p.tile == 0) return cudaErrorInvalidConfiguration;
  p.experts = gp.experts;
  p.xp4 = gp.xp4; p.xp2 = gp.xp2; p.xsum = gp.xsum; p.xexp = gp.xexp;
  p.start = gp.grp_start; p.list = gp.grp_list; p.order = gp.grp_order; p.n_active = n_active; p.work = work;
  p.y = gp.y; p.err = gp.err;
  static int attr_done = 0;
  if (!attr_done) {
    e = cudaFuncSetAttribute(grouped_expert_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e != cudaSuccess) return e;
    attr_done = 1;
  }
  grouped_expert_kernel<<<sms, kGThreads, grouped_smem_bytes(gp.H, gp.I, p.tile), s>>>(p);
  return cudaGetLastError();
}

}  // namespace qe
