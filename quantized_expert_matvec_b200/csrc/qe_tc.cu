// qe_tc.cu -- tensor-core gate/up of the batched layer step, for the experts
// that receive at least kTcMinTokens tokens in one step.  There the tokens of
// one expert form a real dense contraction: G = W_gate X^T and U = W_up X^T
// with X the [n, H] block of the tokens' normalised activations.
//
// One persistent CTA per SM (256 threads) takes items (expert, 128 rows of
// gate and up).  Per 64-column block of H (one quantisation group):
//   - all threads copy the packed gate/up words of the 128 rows and the fp16
//     activation rows of the tokens into a 4-stage shared-memory ring
//     (cp.async, 16 bytes per thread and copy);
//   - all threads dequantise the packed words (w = q*scale + bias, fp32, then
//     rounded to fp16) into 128-byte-swizzled K-major tiles;
//   - one thread issues tcgen05.mma (kind::f16, M = 128, N = tokens rounded up
//     to 16, K = 16, fp32 accumulators in tensor memory: gate in columns
//     [0, N), up in [N, 2N)) and commits to an mbarrier; the stage is reused
//     once that commit has arrived.
// The epilogue reads the accumulators (tcgen05.ld), forms h = silu(g) * u and
// writes h and the running max |h| of each (token, k) assignment for the
// CUDA-core down kernel.  Every wait is bounded; a wait that gives up records
// QE_ERR_TIMEOUT, lets the copies and MMAs in flight finish, frees the tensor
// memory and returns.
#include <cuda_fp16.h>
#include <math.h>
#include <string.h>

#include "qe_device.cuh"

namespace qe {

constexpr int kTcThreads = 256;
constexpr int kTcM = 128;         // rows per item (MMA M)
constexpr int kTcKB = 64;         // K block: one group, one 128-byte row of fp16
constexpr int kTcN = 128;         // tokens per pass (MMA N <= kTcN)
constexpr int kTcRing = 4;        // ring stages of packed words + activation tile
constexpr int kTcTmemCols = 256;  // gate [0, N) and up [N, 2N)
constexpr int kTcMinTokens = 16;

// Shared memory: ring stage = activation tile (kTcN rows x 128 B) then the
// packed gate and up words (128 rows x 32 B each at most); then two fp16
// A-tile pairs (gate, up: 128 rows x 128 B each).  Every tile is 1024-byte
// aligned, as the 128-byte swizzle expects.
constexpr int kTcBTile = kTcN * 128;                   // 16 KB
constexpr int kTcPk = kTcM * 32;                       // 4 KB (4-bit), 2 KB used at 2-bit
constexpr int kTcStage = kTcBTile + 2 * kTcPk;         // 24 KB
constexpr int kTcATile = kTcM * 128;                   // 16 KB
constexpr int kTcSmem = kTcRing * kTcStage + 2 * 2 * kTcATile + 1024;  // + alignment slack

struct TcParams {
  int H, I, K;
  const qe_expert* experts;
  const uint16_t* xh;  // [T][H] fp16 bits of xn
  const int* count;
  const int* start;
  const int* list;
  const int* order;
  int* ctl;            // [3] experts with >= kTcMinTokens tokens (they lead `order`), [4] work counter
  float* h;            // [T*K][I]
  unsigned* hamax;     // [T*K]
  int* err;
  unsigned long long budget_ns;
};

// Offset of 16-byte chunk c (0..7) of row r in a 128-byte-swizzled K-major tile.
static __device__ __forceinline__ uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), leading byte offset 16 (unused by
// this layout), descriptor version 1.
static __device__ __forceinline__ uint64_t tc_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
         (2ull << 61);
}

// Instruction descriptor: fp16 A and B, fp32 D, both K-major, M = 128, N.
static __device__ __forceinline__ uint32_t tc_idesc(int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(kTcM >> 4) << 24);
}

static __device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

static __device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

static __device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
static __device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
static __device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

static __device__ __forceinline__ void tc_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
static __device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 16-byte copy with zero fill: src_bytes 0 writes zeros.
static __device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}

static __device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  return (uint32_t)__half_as_ushort(__float2half_rn(a)) | ((uint32_t)__half_as_ushort(__float2half_rn(b)) << 16);
}

// Dequantise one thread's half row (32 columns) of one matrix into the fp16
// tile: r = row, hf = half, pk = packed words of the row for this K block.
template <int BITS>
static __device__ __forceinline__ void tc_dequant(const unsigned char* pk_row, int r, int hf, float s, float b,
                                                  unsigned char* tile) {
  if (BITS == 4) {
    const uint4 w = *(const uint4*)(pk_row + hf * 16);  // 4 words: columns 32hf + 8j + i
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t v = ws[j];
      uint4 o;
      o.x = pack_h2(fmaf((float)(v & 15u), s, b), fmaf((float)((v >> 4) & 15u), s, b));
      o.y = pack_h2(fmaf((float)((v >> 8) & 15u), s, b), fmaf((float)((v >> 12) & 15u), s, b));
      o.z = pack_h2(fmaf((float)((v >> 16) & 15u), s, b), fmaf((float)((v >> 20) & 15u), s, b));
      o.w = pack_h2(fmaf((float)((v >> 24) & 15u), s, b), fmaf((float)(v >> 28), s, b));
      *(uint4*)(tile + sw128(r, hf * 4 + j)) = o;
    }
  } else {
    const uint2 w = *(const uint2*)(pk_row + hf * 8);  // 2 words: columns 32hf + 16j + i
    const uint32_t ws[2] = {w.x, w.y};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t v = ws[j];
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const uint32_t u = v >> (16 * m);
        uint4 o;
        o.x = pack_h2(fmaf((float)(u & 3u), s, b), fmaf((float)((u >> 2) & 3u), s, b));
        o.y = pack_h2(fmaf((float)((u >> 4) & 3u), s, b), fmaf((float)((u >> 6) & 3u), s, b));
        o.z = pack_h2(fmaf((float)((u >> 8) & 3u), s, b), fmaf((float)((u >> 10) & 3u), s, b));
        o.w = pack_h2(fmaf((float)((u >> 12) & 3u), s, b), fmaf((float)((u >> 14) & 3u), s, b));
        *(uint4*)(tile + sw128(r, hf * 4 + 2 * j + m)) = o;
      }
    }
  }
}

template <int BITS>
static __device__ void tc_item(const TcParams& p, const qe_expert& ex, int r0, const int* asg, const int* toks, int nt,
                               unsigned char* sm, uint32_t tmem, uint64_t* mma_done, uint32_t (&ncommit)[2],
                               uint64_t deadline, volatile int* abort_flag) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H, I = p.I;
  const int N = (nt + 15) & ~15;
  const int nkb = H / kTcKB;
  const int gpr = H / kGroup;
  const size_t rowb = (size_t)H * BITS / 8;
  constexpr int PB = kTcKB * BITS / 8;  // packed bytes of one row in one K block
  const uint32_t idesc = tc_idesc(N);
  unsigned char* ring = sm;
  unsigned char* atile = sm + kTcRing * kTcStage;
  const int r = tid >> 1, hf = tid & 1;  // this thread's dequant row and half
  const uint64_t pol = policy_evict_first();  // each weight row is read by one CTA once

  auto issue = [&](int kb) {
    unsigned char* st = ring + (kb % kTcRing) * kTcStage;
    // activation rows: token t, 16-byte chunk c of the K block
    for (int u = tid; u < N * 8; u += kTcThreads) {
      const int t = u >> 3, c = u & 7;
      const bool live = t < nt;
      const uint16_t* src = p.xh + (live ? (size_t)toks[t] * H + kb * kTcKB + c * 8 : 0);
      cp_async16_zfill(st + sw128(t, c), src, live ? 16u : 0u);
    }
    // packed words: PB bytes per row and matrix, in 16-byte pieces
    constexpr int PPR = PB / 16;  // pieces per row
    for (int u = tid; u < 2 * kTcM * PPR; u += kTcThreads) {
      const int m = u / (kTcM * PPR), rem = u - m * (kTcM * PPR);
      const int rr = rem / PPR, pc = rem - rr * PPR;
      const unsigned char* src =
          (const unsigned char*)(m ? ex.up.wq : ex.gate.wq) + (size_t)(r0 + rr) * rowb + (size_t)kb * PB + pc * 16;
      cp_async16(st + kTcBTile + m * kTcPk + rr * PB + pc * 16, src, pol);
    }
    cp_async_commit();
  };

  // per-row scale and bias of the next K block, loaded a block ahead
  auto load_sb = [&](int kb, float (&sb)[4]) {
    const size_t gi = (size_t)(r0 + r) * gpr + kb;
    sb[0] = bf16f(__ldg(ex.gate.scales + gi));
    sb[1] = bf16f(__ldg(ex.gate.biases + gi));
    sb[2] = bf16f(__ldg(ex.up.scales + gi));
    sb[3] = bf16f(__ldg(ex.up.biases + gi));
  };

  // the item's scale/bias rows (128 rows x gpr entries, 4 arrays) into L2
  for (int u = tid; u < 4 * kTcM; u += kTcThreads) {
    const int a = u / kTcM, rr = u - a * kTcM;
    const uint16_t* base = a == 0 ? ex.gate.scales : a == 1 ? ex.gate.biases : a == 2 ? ex.up.scales : ex.up.biases;
    for (int o = 0; o < gpr * 2; o += 128) prefetch_l2((const unsigned char*)(base + (size_t)(r0 + rr) * gpr) + o);
  }

  const int pre = nkb < kTcRing - 1 ? nkb : kTcRing - 1;
  for (int kb = 0; kb < pre; ++kb) issue(kb);
  float sb[4], sbn[4];
  load_sb(0, sb);
  bool ok = true;
  for (int kb = 0; kb < nkb && ok; ++kb) {
    const int issued = kb + 3 < nkb ? kb + 3 : nkb;  // blocks whose copies are committed
    const int later = issued - kb - 1;
    if (later >= 2) cp_async_wait<2>();
    else if (later == 1) cp_async_wait<1>();
    else cp_async_wait<0>();
    if (kb + 1 < nkb) load_sb(kb + 1, sbn);
    __syncthreads();
    // dequantise block kb into A tile pair kb & 1 (free: its MMAs, block kb-2,
    // completed before block kb-1's copies were issued)
    const unsigned char* st = ring + (kb % kTcRing) * kTcStage;
    unsigned char* ag = atile + (kb & 1) * 2 * kTcATile;
    tc_dequant<BITS>(st + kTcBTile + r * PB, r, hf, sb[0], sb[1], ag);
    tc_dequant<BITS>(st + kTcBTile + kTcPk + r * PB, r, hf, sb[2], sb[3], ag + kTcATile);
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sa = smem_u32(ag), sbt = smem_u32(st);
#pragma unroll
      for (int k = 0; k < kTcKB / 16; ++k) {
        const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
        tc_mma(tmem, tc_desc(sa + k * 32), tc_desc(sbt + k * 32), idesc, acc);
        tc_mma(tmem + (uint32_t)N, tc_desc(sa + kTcATile + k * 32), tc_desc(sbt + k * 32), idesc, acc);
      }
      tc_commit(&mma_done[kb & 1]);
    }
    ++ncommit[kb & 1];
    // block kb-1's MMAs done: its ring stage and A tile pair may be reused
    if (kb >= 1) {
      const int b = (kb - 1) & 1;
      bool w = mbar_wait(&mma_done[b], (ncommit[b] - 1) & 1, deadline, abort_flag);
      ok = __syncthreads_and(w) != 0;  // one decision for the whole CTA
    }
    if (ok && kb + 3 < nkb) issue(kb + 3);
#pragma unroll
    for (int i = 0; i < 4; ++i) sb[i] = sbn[i];
  }
  // the last block's MMAs (and with them every earlier one)
  const int bl = (nkb - 1) & 1;
  if (ok) ok = __syncthreads_and(mbar_wait(&mma_done[bl], (ncommit[bl] - 1) & 1, deadline, abort_flag)) != 0;
  cp_async_wait<0>();
  if (!ok) {
    if (tid == 0) set_error(p.err, QE_ERR_TIMEOUT);
    *abort_flag = 1;
    // let the MMAs already issued finish before tensor memory is freed
    // (a second bounded wait that ignores the abort flag)
    volatile int no_abort = 0;
    const uint64_t dl2 = gtimer() + p.budget_ns;
    for (int b = 0; b < 2; ++b)
      if (ncommit[b] > 0) mbar_wait(&mma_done[b], (ncommit[b] - 1) & 1, dl2, &no_abort);
    __syncthreads();
    return;
  }
  tc_fence_after();
  // epilogue: warp w reads rows 32*(w & 3) .. +31 (its tensor-memory lane
  // quadrant) and the tokens of half w >> 2, 8 columns at a time
  const int q = warp & 3, half = warp >> 2;
  const int row = r0 + 32 * q + lane;
  const int tb = half * (N / 2), te = tb + N / 2;
  for (int c0 = tb; c0 < te; c0 += 8) {
    float g[8], u[8];
    tc_ld8(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, g);
    tc_ld8(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(N + c0), u);
    tc_wait_ld();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int t = c0 + j;
      if (t < nt) {
        const float hv = g[j] / (1.0f + expf(-g[j])) * u[j];
        const int a = asg[t];
        p.h[(size_t)a * I + row] = hv;
        const float m = warp_max(fabsf(hv));
        if (lane == 0) atomicMax(&p.hamax[a], __float_as_uint(m));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
}

__global__ void __launch_bounds__(kTcThreads, 1) grouped_tc_gateup_kernel(const TcParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t mma_done[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_item, s_abort;
  __shared__ qe_expert s_ex;
  __shared__ int asg[kTcN], toks[kTcN];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int n_tc = p.ctl[3];
  const int ipe = p.I / kTcM;
  const int n_items = n_tc * ipe;
  if (n_items == 0) return;  // no expert has enough tokens: nothing allocated yet
  const uint64_t deadline = gtimer() + p.budget_ns;
  volatile int* abort_flag = &s_abort;
  if (tid == 0) {
    mbar_init(&mma_done[0], 1);
    mbar_init(&mma_done[1], 1);
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  uint32_t ncommit[2] = {0u, 0u};
  for (;;) {
    if (tid == 0) s_item = atomicAdd(&p.ctl[4], 1);
    __syncthreads();
    const int item = s_item;
    if (item >= n_items || *abort_flag) break;
    const int e = p.order[item / ipe];
    const int r0 = (item % ipe) * kTcM;
    if (tid == 0) s_ex = p.experts[e];
    __syncthreads();
    const int bits = s_ex.gate.bits;
    const bool ok = (bits == 4 || bits == 2) && s_ex.up.bits == bits && s_ex.gate.wq && s_ex.up.wq &&
                    s_ex.gate.scales && s_ex.gate.biases && s_ex.up.scales && s_ex.up.biases &&
                    ((uintptr_t)s_ex.gate.wq & 15) == 0 && ((uintptr_t)s_ex.up.wq & 15) == 0;
    if (!ok) {
      if (tid == 0) set_error(p.err, QE_ERR_INVALID_ARG);
      __syncthreads();
      continue;
    }
    const int n = p.count[e], s0 = p.start[e];
    for (int t0 = 0; t0 < n && !*abort_flag; t0 += kTcN) {
      const int nt = min(kTcN, n - t0);
      if (tid < nt) {
        const int a = p.list[s0 + t0 + tid];
        asg[tid] = a;
        toks[tid] = a / p.K;
      }
      __syncthreads();
      if (bits == 4) tc_item<4>(p, s_ex, r0, asg, toks, nt, sm, tmem, mma_done, ncommit, deadline, abort_flag);
      else tc_item<2>(p, s_ex, r0, asg, toks, nt, sm, tmem, mma_done, ncommit, deadline, abort_flag);
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols) : "memory");
  }
}

bool tc_eligible(int H, int I) { return I % kTcM == 0 && H % kTcKB == 0; }

cudaError_t launch_tc_gateup(const GroupedParams& gp, int* ctl, unsigned long long budget_ns, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static int attr_dev = -1;
  cudaError_t e;
  if (attr_dev != dev) {
    if ((e = cudaFuncSetAttribute(grouped_tc_gateup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem)) !=
        cudaSuccess)
      return e;
    attr_dev = dev;
  }
  TcParams p{};
  p.H = gp.H; p.I = gp.I; p.K = gp.K;
  p.experts = gp.experts; p.xh = gp.xh;
  p.count = gp.grp_count; p.start = gp.grp_start; p.list = gp.grp_list; p.order = gp.grp_order;
  p.ctl = ctl; p.h = gp.h; p.hamax = gp.hamax; p.err = gp.err; p.budget_ns = budget_ns;
  grouped_tc_gateup_kernel<<<sms, kTcThreads, kTcSmem, s>>>(p);
  return cudaGetLastError();
}

int tc_min_tokens() { return kTcMinTokens; }

}  // namespace qe
