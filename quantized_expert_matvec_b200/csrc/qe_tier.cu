// qe_tier.cu -- two-tier expert residency: hot experts resident in HBM, cold
// experts in page-locked host memory behind an HBM cache of expert slots with
// least-recently-used replacement.
//
// Follows the tiering of the Flash-MoE pages (lilting.ch "Flash-MoE: running
// a 397B-parameter model on a 48 GB MacBook", sections "Core technique: SSD
// expert streaming" and "Trust the OS": experts streamed from storage on
// demand into a page cache; nzkcom.pages.dev "flash-moe-romance-vs-utility",
// adopted optimisations: frequently used experts kept at 4 bits, the rest
// at 2 bits).  On B200 the storage tier is pinned host memory over PCIe and
// the cache is a pool of HBM slots managed here instead of by an OS.
//
// The cache's bookkeeping lives on the device, so that a layer whose experts
// are all cached never waits for the host:
//   - a slot map (cold expert -> slot or -1), per-slot last-use stamps and
//     per-slot claim marks (the last call that claimed the slot), all in
//     device memory;
//   - tier_resolve_kernel (one CTA) replays the replacement policy in stream
//     order: the call's distinct cold experts are found, hits claim their
//     slots (stamped most recent), then each miss takes the unclaimed slot
//     with the oldest stamp and queues a copy task; every cold expert's
//     descriptor is written into the layer's table;
//   - tier_fill_kernel copies the queued experts from host memory, which is
//     mapped into the device's address space, into their slots.
// A tiered layer step is therefore a fixed sequence of kernel launches
// (routing, resolve, fill, experts; for one token the routing and the resolve
// are one kernel, tier_route_kernel) and can be captured in a CUDA graph.
#include <mutex>
#include <vector>

#include "qe_device.cuh"
#include "qe_internal.h"

namespace qe {

struct TierState {                // device
  unsigned call;                  // calls resolved so far; claim marks compare to it
  int status;                     // first error found on the device (QE_OK if none)
  unsigned long long clock;       // last stamp given to a slot
  unsigned long long hits, misses, h2d_bytes;
  int n_tasks;                    // copies queued by the last resolve
  unsigned route_done;            // CTAs of the running routing launch that are done (0 between launches)
};

struct TierDev {                  // device pointers and constants, passed by value
  TierState* st;
  int32_t* key_slot;              // [L*E] slot of a cold expert, -1 if not cached
  const unsigned long long* cold_src;  // [L*E] device-visible address of a cold expert, 0 if hot
  int32_t* slot_key;              // [S] expert held by a slot, -1 if none
  uint32_t* slot_call;            // [S] call that last claimed the slot
  unsigned long long* slot_stamp; // [S] last use; unique, larger is more recent
  unsigned long long* task_src;   // [max selections] source of a queued copy
  int32_t* task_slot;             // [max selections] its slot
  unsigned char* cache;           // S * slot_bytes
  unsigned long long slot_bytes, expert_bytes;
  int n_slots, E;
  qe_expert tmpl;                 // descriptor of an expert stored at cache + 0
};

constexpr int kResolveThreads = 1024;
constexpr int kFillThreads = 512;
constexpr int kMaxTierSel = 4096;  // selections one call may resolve (max_tokens * top_k)

__device__ __forceinline__ qe_expert slot_descriptor(const TierDev& d, int slot) {
  qe_expert x = d.tmpl;
  const size_t off = (size_t)slot * d.slot_bytes;
  x.gate.wq = (const uint32_t*)((const char*)x.gate.wq + off);
  x.gate.scales = (const uint16_t*)((const char*)x.gate.scales + off);
  x.gate.biases = (const uint16_t*)((const char*)x.gate.biases + off);
  x.up.wq = (const uint32_t*)((const char*)x.up.wq + off);
  x.up.scales = (const uint16_t*)((const char*)x.up.scales + off);
  x.up.biases = (const uint16_t*)((const char*)x.up.biases + off);
  x.down.wq = (const uint32_t*)((const char*)x.down.wq + off);
  x.down.scales = (const uint16_t*)((const char*)x.down.scales + off);
  x.down.biases = (const uint16_t*)((const char*)x.down.biases + off);
  return x;
}

// One CTA.  The call's selections are loaded in parallel into shared memory
// (expert key, cold or not, slot at the start of the call) and deduplicated
// there; thread 0 then replays the replacement policy over the distinct cold
// experts in call order, reading shared memory only; the whole CTA searches
// for each miss's victim; finally every first occurrence writes its
// descriptor.  Every __syncthreads below is reached by all threads: the
// branches around them test shared values written before the preceding
// barrier.  n <= kMaxTierSel.
// (A __device__ function so that the single-token routing kernel's last CTA
// can run it too; called by all kResolveThreads threads of one CTA.)
__device__ __forceinline__ void tier_resolve_body(const TierDev& d, int layer, const int32_t* idx, int n,
                                                 qe_expert* table) {
  __shared__ int s_key[kMaxTierSel];    // expert key of selection i
  __shared__ int s_slot[kMaxTierSel];   // its slot: -1 not cached; -2 hot or duplicate; -3 index out of range
  __shared__ unsigned s_call;
  __shared__ unsigned long long s_clock;
  __shared__ int s_bad, s_kind, s_cur;
  __shared__ unsigned long long s_best[kResolveThreads / 32];
  __shared__ int s_besti[kResolveThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  TierState* st = d.st;
  __syncthreads();  // the caller's shared memory may still be in use
  // every load of the hit path in one round trip: the state's call counter
  // and clock, and each selection's slot (idx may be shared memory)
  if (tid == 0) {
    s_call = st->call + 1u;  // 0 after 2^32 calls
    s_clock = st->clock;
  }
  for (int i = tid; i < n; i += blockDim.x) {
    const int e = idx[i];
    if (e < 0 || e >= d.E) {
      s_key[i] = -1;
      s_slot[i] = -3;
      continue;
    }
    const int key = layer * d.E + e;
    s_key[i] = key;
    const unsigned long long src = d.cold_src[key];
    const int sl = d.key_slot[key];  // loaded with src, not after it
    s_slot[i] = src ? sl : -2;
  }
  __syncthreads();
  if (s_call == 0) {  // wrapped: forget every claim mark
    for (int s = tid; s < d.n_slots; s += blockDim.x) d.slot_call[s] = 0u;
    __syncthreads();
    if (tid == 0) s_call = 1u;
  }
  // later occurrences of an expert are dropped (marked hot) so that each
  // distinct cold expert is handled once, at its first occurrence
  int dup[kMaxTierSel / kResolveThreads];
#pragma unroll
  for (int r = 0; r < kMaxTierSel / kResolveThreads; ++r) {
    const int i = tid + r * kResolveThreads;
    dup[r] = 0;
    if (i < n && s_slot[i] >= -1)
      for (int j = 0; j < i; ++j)
        if (s_key[j] == s_key[i]) {
          dup[r] = 1;
          break;
        }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kMaxTierSel / kResolveThreads; ++r)
    if (dup[r]) s_slot[tid + r * kResolveThreads] = -2;
  __syncthreads();
  const unsigned call = s_call;
  unsigned long long clock = 0, hits = 0, misses = 0, bytes = 0;
  int n_tasks = 0;
  if (tid == 0) {
    st->call = call;
    st->n_tasks = 0;
    clock = s_clock;
    int n_cold = 0, bad = QE_OK;
    // hits claim their slots (most recent in call order) before any miss
    // chooses a victim, so that no miss of this call evicts them
    for (int i = 0; i < n; ++i) {
      if (s_slot[i] == -3) bad = QE_ERR_INVALID_ARG;
      if (s_slot[i] < -1) continue;
      ++n_cold;
      const int sl = s_slot[i];
      if (sl >= 0) {
        d.slot_call[sl] = call;
        d.slot_stamp[sl] = ++clock;
        ++hits;
      }
    }
    if (bad == QE_OK && n_cold > d.n_slots) bad = QE_ERR_OOM;
    if (bad != QE_OK) atomicCAS(&st->status, QE_OK, bad);
    s_bad = bad;
    s_cur = -1;
  }
  __syncthreads();
  if (s_bad != QE_OK) return;  // resolve nothing (the host refuses such calls before launching)
  // misses in call order: each takes the least recently used unclaimed slot
  for (;;) {
    if (tid == 0) {
      int i = s_cur + 1;
      while (i < n && s_slot[i] != -1) ++i;  // the next miss (cached slots are >= 0)
      s_cur = i;
      s_kind = i < n;
    }
    __syncthreads();
    if (!s_kind) break;
    unsigned long long best = ~0ull;
    int bi = -1;
    for (int s = tid; s < d.n_slots; s += blockDim.x) {
      const unsigned long long stamp = d.slot_stamp[s];
      if (d.slot_call[s] != call && stamp < best) {
        best = stamp;
        bi = s;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob < best) {
        best = ob;
        bi = oi;
      }
    }
    if (lane == 0) {
      s_best[warp] = best;
      s_besti[warp] = bi;
    }
    __syncthreads();
    if (tid == 0) {
      for (int w = 1; w < kResolveThreads / 32; ++w)
        if (s_best[w] < best) {
          best = s_best[w];
          bi = s_besti[w];
        }
      const int i = s_cur;
      if (bi < 0) {  // every slot claimed: cannot happen once n_cold <= n_slots
        atomicCAS(&st->status, QE_OK, QE_ERR_OOM);
        s_slot[i] = -2;
      } else {
        const int key = s_key[i];
        const int old = d.slot_key[bi];
        if (old >= 0) d.key_slot[old] = -1;
        d.slot_key[bi] = key;
        d.key_slot[key] = bi;
        d.slot_call[bi] = call;
        d.slot_stamp[bi] = ++clock;
        d.task_src[n_tasks] = d.cold_src[key];
        d.task_slot[n_tasks] = bi;
        ++n_tasks;
        ++misses;
        bytes += d.expert_bytes;
        s_slot[i] = bi;
      }
    }
    __syncthreads();
  }
  // descriptors of every distinct cold expert of the call
  for (int i = tid; i < n; i += blockDim.x)
    if (s_slot[i] >= 0) table[idx[i]] = slot_descriptor(d, s_slot[i]);
  if (tid == 0) {  // stores and reductions only: nothing left to wait for
    st->clock = clock;
    if (hits) atomicAdd(&st->hits, hits);
    if (misses) atomicAdd(&st->misses, misses);
    if (bytes) atomicAdd(&st->h2d_bytes, bytes);
    st->n_tasks = n_tasks;
  }
}

__global__ void __launch_bounds__(kResolveThreads) tier_resolve_kernel(TierDev d, int layer, const int32_t* idx,
                                                                        int n, qe_expert* table) {
  grid_dependency_wait();
  grid_launch_dependents();
  tier_resolve_body(d, layer, idx, n, table);
}

// Copy the queued experts from host memory (device-visible addresses) into
// their slots, 16 bytes per access, four accesses in flight per thread.
__global__ void __launch_bounds__(kFillThreads) tier_fill_kernel(TierDev d) {
  grid_dependency_wait();
  grid_launch_dependents();
  const int n = d.st->n_tasks;
  const unsigned long long per = d.expert_bytes / 16;  // expert bytes are a multiple of 256
  const unsigned long long total = (unsigned long long)n * per;
  const unsigned long long stride = (unsigned long long)gridDim.x * blockDim.x;
  for (unsigned long long j0 = (unsigned long long)blockIdx.x * blockDim.x + threadIdx.x; j0 < total;
       j0 += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const unsigned long long j = j0 + u * stride;
      if (j < total) {
        const unsigned long long t = j / per, o = j - t * per;
        v[u] = reinterpret_cast<const uint4*>(d.task_src[t])[o];
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const unsigned long long j = j0 + u * stride;
      if (j < total) {
        const unsigned long long t = j / per, o = j - t * per;
        reinterpret_cast<uint4*>(d.cache + (size_t)d.task_slot[t] * d.slot_bytes)[o] = v[u];
      }
    }
  }
}


// Routing of one token for the tiered step, with the resolve folded in:
// RMSNorm scale, router logits (fp64), top-K with renormalised softmax
// weights, then tier_resolve_body on the chosen experts.  Each CTA takes
// kRouteRows router rows, kRouteSplit warps per row, each warp one
// 1/kRouteSplit of the columns; every CTA also sums x^2 itself (x is small
// and in L2), so no CTA waits for another.  The last CTA to finish its
// logits (an acquire-release arrival counter in the tier's state, reset by
// that CTA for the next launch) takes the top-K and the resolve; the others
// just exit.  The last CTA's top-K runs over the whole block, one logit per
// thread.  Two routing launches on one tier must not overlap (all calls on a
// tier are ordered on the device).  The logit and weight formulas are
// moe_route's:
// l_e = (sum_c W[e,c] * x_c * gamma_c) / sqrt(mean(x^2) + eps) + offset_e,
// sums in fp64, ties to the lower index.
constexpr int kRouteSplit = 8;
constexpr int kRouteRows = kResolveThreads / 32 / kRouteSplit;  // 4
constexpr int kRouteUnroll = 4;

struct TierRoute {
  const void* x;
  int x_bf16;
  const float* gamma;
  const float* router_w;
  const float* offset;
  int H, E, K;
  float eps;
  double* logits;  // [E], workspace
  int32_t* idx;    // [K]
  float* w;        // [K]
};

// x[c..c+3] as floats (c % 4 == 0; fp32 rows are 16-byte aligned here, bf16
// rows 8-byte aligned)
__device__ __forceinline__ float4 load_x4(const TierRoute& r, int c) {
  if (!r.x_bf16) return *reinterpret_cast<const float4*>((const float*)r.x + c);
  const uint2 u = *reinterpret_cast<const uint2*>((const uint16_t*)r.x + c);
  return make_float4(bf16f(u.x & 0xffffu), bf16f(u.x >> 16), bf16f(u.y & 0xffffu), bf16f(u.y >> 16));
}

__global__ void __launch_bounds__(kResolveThreads) tier_route_kernel(TierRoute r, TierDev d, int layer,
                                                                      qe_expert* table) {
  __shared__ double s_part[kRouteRows][kRouteSplit];
  __shared__ double s_ss[kResolveThreads / 32];
  __shared__ double s_wv[kResolveThreads / 32];
  __shared__ int s_wi[kResolveThreads / 32];
  __shared__ double s_selv[kMaxK];
  __shared__ int s_sel[kMaxK];
  __shared__ int s_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  grid_dependency_wait();  // x comes from the previous kernel
  grid_launch_dependents();
  auto ldx = [&](int c) -> double {
    return r.x_bf16 ? (double)bf16f(((const uint16_t*)r.x)[c]) : (double)((const float*)r.x)[c];
  };
  // sum of squares: all of a thread's loads first (H <= 8192: at most 8)
  double xs[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int c = tid + u * kResolveThreads;
    xs[u] = c < r.H ? ldx(c) : 0.0;
  }
  double ss = 0.0;
#pragma unroll
  for (int u = 0; u < 8; ++u) ss += xs[u] * xs[u];
  ss = warp_sum_d(ss);
  if (lane == 0) s_ss[warp] = ss;
  // this warp's part of one router row: all of a lane's loads are issued
  // before its FMAs (4 float4 of W and 4 of x at a time)
  const int row = warp / kRouteSplit, part = warp % kRouteSplit;
  const int e = blockIdx.x * kRouteRows + row;
  double acc = 0.0;
  if (e < r.E) {
    const int q4 = r.H / 4 / kRouteSplit;  // float4 per part (H % 64 == 0, so whole); <= 256
    const float4* wrow = reinterpret_cast<const float4*>(r.router_w + (size_t)e * r.H) + part * q4;
    const int c0 = part * q4 * 4;
    for (int i0 = lane; i0 < q4; i0 += 32 * kRouteUnroll) {
      float4 wv[kRouteUnroll], xv[kRouteUnroll];
#pragma unroll
      for (int u = 0; u < kRouteUnroll; ++u) {
        const int i = i0 + 32 * u;
        if (i < q4) {
          wv[u] = __ldg(wrow + i);
          xv[u] = load_x4(r, c0 + 4 * i);
        }
      }
#pragma unroll
      for (int u = 0; u < kRouteUnroll; ++u) {
        const int i = i0 + 32 * u;
        if (i < q4) {
          const int c = c0 + 4 * i;
          double g0 = 1.0, g1 = 1.0, g2 = 1.0, g3 = 1.0;
          if (r.gamma) {
            const float4 gv = *reinterpret_cast<const float4*>(r.gamma + c);
            g0 = gv.x, g1 = gv.y, g2 = gv.z, g3 = gv.w;
          }
          acc = fma((double)wv[u].x, (double)xv[u].x * g0, acc);
          acc = fma((double)wv[u].y, (double)xv[u].y * g1, acc);
          acc = fma((double)wv[u].z, (double)xv[u].z * g2, acc);
          acc = fma((double)wv[u].w, (double)xv[u].w * g3, acc);
        }
      }
    }
  }
  acc = warp_sum_d(acc);
  if (lane == 0) s_part[row][part] = acc;
  __syncthreads();
  if (tid == 0) {
    // this CTA's logits, then its arrival: the acquire-release add orders the
    // stores before it for whichever CTA arrives last
    double q = 0.0;
    for (int w = 0; w < kResolveThreads / 32; ++w) q += s_ss[w];
    const double rinv = 1.0 / sqrt(q / (double)r.H + (double)r.eps);
    for (int rr = 0; rr < kRouteRows; ++rr) {
      const int ee = blockIdx.x * kRouteRows + rr;
      if (ee < r.E) {
        double a = 0.0;
        for (int p = 0; p < kRouteSplit; ++p) a += s_part[rr][p];
        r.logits[ee] = a * rinv + (r.offset ? (double)r.offset[ee] : 0.0);
      }
    }
    unsigned prev;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(&d.st->route_done) : "memory");
    s_last = prev == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;  // uniform: the whole CTA leaves
  // top-K over the block: one logit per thread (E <= kResolveThreads), K
  // rounds of a warp arg-max and an arg-max over the warps' winners; ties go
  // to the lower index
  const double lv = tid < r.E ? __ldcg(r.logits + tid) : 0.0;
  bool alive = tid < r.E;
  for (int k = 0; k < r.K; ++k) {
    double bv = lv;
    int bi = alive ? tid : 0x7fffffff;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == 0) {
      s_wv[warp] = bv;
      s_wi[warp] = bi;
    }
    __syncthreads();
    if (warp == 0) {
      bv = s_wv[lane];
      bi = s_wi[lane];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) {
          bv = ov;
          bi = oi;
        }
      }
      if (lane == 0) {
        s_sel[k] = bi;
        s_selv[k] = bv;
      }
    }
    __syncthreads();
    if (tid == s_sel[k]) alive = false;
  }
  if (warp == 0) {
    // renormalised softmax weights: lane k takes expert k's exponential,
    // lane 0 sums them in k order
    const int K = r.K;
    const double ev = lane < K ? exp(s_selv[lane] - s_selv[0]) : 0.0;
    double sum = 0.0;
    for (int k = 0; k < K; ++k) sum += __shfl_sync(0xffffffffu, ev, k);
    if (lane < K) {
      r.idx[lane] = s_sel[lane];
      r.w[lane] = (float)(ev / sum);
    }
    if (lane == 0) d.st->route_done = 0u;  // ready for the next launch
  }
  __syncthreads();
  tier_resolve_body(d, layer, s_sel, r.K, table);
}

}  // namespace qe

struct qe_tier {
  qe_cfg cfg;
  int L = 0, E = 0, bits = 2, dev = 0, max_tokens = 0, sms = 148;
  size_t expert_bytes = 0;
  int n_slots = 0;
  std::vector<unsigned char> is_cold;  // [L*E], host copy for argument checks
  std::vector<unsigned> mark;          // [L*E], host scratch for counting distinct experts
  unsigned mark_gen = 0;
  unsigned char* cache = nullptr;      // device, n_slots * expert_bytes
  void* state_mem = nullptr;           // device: TierState and the arrays of TierDev
  int32_t* idx_dev = nullptr;          // device staging of host indices [max selections]
  qe::TierDev d{};
  std::mutex mu;
};

namespace qe {

static size_t al256(size_t b) { return (b + 255) & ~(size_t)255; }

static int check_device(const qe_tier* t) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != t->dev) return fail(QE_ERR_INVALID_ARG, "tier belongs to device %d, current device is %d", t->dev, dev);
  return QE_OK;
}

static void tier_free(qe_tier* t) {
  if (!t) return;
  if (t->cache || t->state_mem) cudaDeviceSynchronize();  // kernels queued on the tier may still run
  if (t->cache) cudaFree(t->cache);
  if (t->state_mem) cudaFree(t->state_mem);
  delete t;
}

// Launch with programmatic stream serialisation: the kernel may start while
// the previous one drains; each of these kernels waits for it
// (griddepcontrol.wait) before touching memory.
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, int block, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Resolve + fill for `n` device indices of layer `layer` on stream s.
static int launch_resolve(qe_tier* t, int layer, const int32_t* idx_dev, int n, qe_expert* dev_table,
                          cudaStream_t s) {
  cudaError_t e = launch_pdl(tier_resolve_kernel, 1, kResolveThreads, s, t->d, layer, idx_dev, n, dev_table);
  if (e != cudaSuccess) return cuda_fail(e, "tier resolve launch");
  e = launch_pdl(tier_fill_kernel, t->sms, kFillThreads, s, t->d);
  if (e != cudaSuccess) return cuda_fail(e, "tier fill launch");
  return QE_OK;
}

}  // namespace qe

using namespace qe;

extern "C" {

int qe_tier_create(const qe_tier_desc* d, qe_tier** out) {
  if (!out) return fail(QE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!d) return fail(QE_ERR_INVALID_ARG, "desc is NULL");
  int rc = check_cfg(&d->cfg);
  if (rc) return rc;
  if (d->n_layers <= 0) return fail(QE_ERR_INVALID_ARG, "n_layers must be positive");
  if (!(d->cold_bits == 2 || d->cold_bits == 4)) return fail(QE_ERR_INVALID_ARG, "cold_bits must be 2 or 4");
  if (!d->cold_host) return fail(QE_ERR_INVALID_ARG, "cold_host is NULL");
  if (d->max_tokens <= 0 || (long long)d->max_tokens * d->cfg.top_k > kMaxTierSel)
    return fail(QE_ERR_INVALID_ARG, "max_tokens * top_k must be in [1, %d]", kMaxTierSel);
  const size_t eb = qe_expert_bytes(&d->cfg, d->cold_bits);
  const size_t nkeys = (size_t)d->n_layers * d->cfg.n_experts;
  if (nkeys > (size_t)0x7fffffff) return fail(QE_ERR_INVALID_ARG, "too many experts");
  const size_t n_slots = d->cache_bytes / eb;
  if (n_slots < 1) return fail(QE_ERR_INVALID_ARG, "cache_bytes %zu holds no %zu-byte expert", d->cache_bytes, eb);
  if (n_slots > (size_t)0x7fffffff) return fail(QE_ERR_INVALID_ARG, "cache too large");
  for (size_t k = 0; k < nkeys; ++k)
    if (((uintptr_t)d->cold_host[k] & 15) != 0)
      return fail(QE_ERR_INVALID_ARG, "cold expert %zu is not 16-byte aligned", k);
  qe_tier* t = new qe_tier();
  t->cfg = d->cfg;
  t->L = d->n_layers;
  t->E = d->cfg.n_experts;
  t->bits = d->cold_bits;
  t->max_tokens = d->max_tokens;
  t->expert_bytes = eb;  // segments are 256-byte multiples already
  t->n_slots = (int)n_slots;
  t->is_cold.assign(nkeys, 0);
  t->mark.assign(nkeys, 0u);
  // the device reads cold experts through their device-visible addresses
  std::vector<unsigned long long> src(nkeys, 0ull);
  cudaError_t e = cudaGetDevice(&t->dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&t->sms, cudaDevAttrMultiProcessorCount, t->dev);
  for (size_t k = 0; k < nkeys && e == cudaSuccess; ++k) {
    if (!d->cold_host[k]) continue;
    cudaPointerAttributes pa{};
    e = cudaPointerGetAttributes(&pa, d->cold_host[k]);
    if (e != cudaSuccess || pa.type != cudaMemoryTypeHost || !pa.devicePointer) {
      cudaGetLastError();
      delete t;
      return fail(QE_ERR_INVALID_ARG,
                  "cold expert %zu is not page-locked host memory mapped for the device (allocate it with "
                  "cudaHostAlloc, or register it with cudaHostRegisterMapped)", k);
    }
    src[k] = (unsigned long long)(uintptr_t)pa.devicePointer;
    t->is_cold[k] = 1;
  }
  if (e != cudaSuccess) {
    const int r = cuda_fail(e, "qe_tier_create");
    delete t;
    return r;
  }
  const size_t nsel = (size_t)d->max_tokens * d->cfg.top_k;
  // one device block: state, then the arrays, each 256-byte aligned
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off = al256(off + bytes); return o; };
  const size_t o_st = take(sizeof(TierState)), o_ks = take(4 * nkeys),
               o_src = take(8 * nkeys), o_sk = take(4 * n_slots), o_sc = take(4 * n_slots),
               o_stamp = take(8 * n_slots), o_tsrc = take(8 * nsel), o_tslot = take(4 * nsel),
               o_idx = take(4 * nsel);
  e = cudaMalloc(&t->cache, n_slots * eb);
  if (e != cudaSuccess) {
    cudaGetLastError();
    t->cache = nullptr;
    tier_free(t);
    return fail(QE_ERR_OOM, "tier: cudaMalloc of the %zu-byte expert cache failed", n_slots * eb);
  }
  e = cudaMalloc(&t->state_mem, off);
  if (e != cudaSuccess) {
    cudaGetLastError();
    t->state_mem = nullptr;
    tier_free(t);
    return fail(QE_ERR_OOM, "tier: cudaMalloc of %zu bytes of cache state failed", off);
  }
  char* b = (char*)t->state_mem;
  TierDev& dv = t->d;
  dv.st = (TierState*)(b + o_st);
  dv.key_slot = (int32_t*)(b + o_ks);
  dv.cold_src = (const unsigned long long*)(b + o_src);
  dv.slot_key = (int32_t*)(b + o_sk);
  dv.slot_call = (uint32_t*)(b + o_sc);
  dv.slot_stamp = (unsigned long long*)(b + o_stamp);
  dv.task_src = (unsigned long long*)(b + o_tsrc);
  dv.task_slot = (int32_t*)(b + o_tslot);
  dv.cache = t->cache;
  dv.slot_bytes = eb;
  dv.expert_bytes = eb;
  dv.n_slots = (int)n_slots;
  dv.E = t->E;
  dv.tmpl = pool_descriptor(&t->cfg, t->cache, t->bits);
  t->idx_dev = (int32_t*)(b + o_idx);
  // initial state: nothing cached; slot s stamped n_slots - s, so that the
  // highest slot is the least recently used (free slots are taken from the top)
  TierState st0{};
  st0.clock = n_slots;
  std::vector<int32_t> minus1(nkeys > n_slots ? nkeys : n_slots, -1);
  std::vector<unsigned long long> stamps(n_slots);
  for (size_t s = 0; s < n_slots; ++s) stamps[s] = n_slots - s;
  e = cudaMemcpy(dv.st, &st0, sizeof(st0), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(dv.key_slot, minus1.data(), 4 * nkeys, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy((void*)dv.cold_src, src.data(), 8 * nkeys, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(dv.slot_key, minus1.data(), 4 * n_slots, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemset(dv.slot_call, 0, 4 * n_slots);
  if (e == cudaSuccess) e = cudaMemcpy(dv.slot_stamp, stamps.data(), 8 * n_slots, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    const int r = cuda_fail(e, "qe_tier_create: initial state");
    tier_free(t);
    return r;
  }
  *out = t;
  return QE_OK;
}

int qe_tier_resolve(qe_tier* t, int layer, const int32_t* host_idx, int n, qe_expert* dev_table,
                    qe_stream_t stream) {
  if (!t) return fail(QE_ERR_INVALID_ARG, "tier is NULL");
  if (layer < 0 || layer >= t->L) return fail(QE_ERR_INVALID_ARG, "layer %d out of range [0, %d)", layer, t->L);
  if (n < 0 || n > t->max_tokens * t->cfg.top_k)
    return fail(QE_ERR_INVALID_ARG, "n = %d outside [0, max_tokens * top_k]", n);
  if (n == 0) return QE_OK;
  int rc;
  if (!host_idx) return fail(QE_ERR_INVALID_ARG, "host_idx is NULL");
  if ((rc = check_ptr(dev_table, "dev_table", false, 8))) return rc;
  if ((rc = check_device(t))) return rc;
  std::lock_guard<std::mutex> lock(t->mu);
  // checked on the host first, so that a refused call changes nothing
  if (++t->mark_gen == 0) {
    std::fill(t->mark.begin(), t->mark.end(), 0u);
    t->mark_gen = 1;
  }
  int n_cold = 0;
  for (int i = 0; i < n; ++i) {
    if (host_idx[i] < 0 || host_idx[i] >= t->E)
      return fail(QE_ERR_INVALID_ARG, "expert index %d out of range [0, %d)", host_idx[i], t->E);
    const size_t key = (size_t)layer * t->E + host_idx[i];
    if (t->is_cold[key] && t->mark[key] != t->mark_gen) {
      t->mark[key] = t->mark_gen;
      ++n_cold;
    }
  }
  if (n_cold > t->n_slots)
    return fail(QE_ERR_OOM, "one call needs %d cold experts but the cache holds %d slots", n_cold, t->n_slots);
  const cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(t->idx_dev, host_idx, sizeof(int32_t) * n, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "qe_tier_resolve: index upload");
  return launch_resolve(t, layer, t->idx_dev, n, dev_table, s);
}

int qe_tier_layer_step(qe_tier* t, int layer, const qe_layer* lw, const void* x, int x_dtype, int T, float* out,
                       int add_residual, int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                       qe_stream_t stream) {
  if (!t) return fail(QE_ERR_INVALID_ARG, "tier is NULL");
  const qe_cfg* c = &t->cfg;
  if (layer < 0 || layer >= t->L) return fail(QE_ERR_INVALID_ARG, "layer %d out of range [0, %d)", layer, t->L);
  if (T < 0 || T > t->max_tokens) return fail(QE_ERR_INVALID_ARG, "T = %d outside [0, max_tokens]", T);
  if (T == 0) return QE_OK;
  if (!lw) return fail(QE_ERR_INVALID_ARG, "layer is NULL");
  if (!(x_dtype == QE_F32 || x_dtype == QE_BF16)) return fail(QE_ERR_INVALID_ARG, "x_dtype must be QE_F32 or QE_BF16");
  int rc;
  if ((rc = check_ptr(x, "x", false, x_dtype == QE_BF16 ? 2 : 4)) || (rc = check_ptr(out, "out")) ||
      (rc = check_ptr(lw->router_w, "router_w", false, 16)) || (rc = check_ptr(lw->experts, "experts", false, 8)) ||
      (rc = check_ptr(lw->gamma, "gamma", true)) || (rc = check_ptr(lw->logit_offset, "logit_offset", true)) ||
      (rc = check_ptr(topk_idx, "topk_idx", true)) || (rc = check_ptr(topk_w, "topk_w", true)) ||
      (rc = check_ws(c, T, ws, ws_bytes)))
    return rc;
  if ((const void*)out == x) return fail(QE_ERR_INVALID_ARG, "out must not alias x");
  // the routing is not known on the host: a call may need up to T * top_k
  // cold experts at once, and the cache must be able to hold them all
  if (T * c->top_k > t->n_slots)
    return fail(QE_ERR_OOM, "T * top_k = %d may exceed the cache's %d slots", T * c->top_k, t->n_slots);
  if ((rc = check_device(t))) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  const WsLayout L = ws_layout(c->hidden, c->n_experts, c->top_k, c->inter, T);
  int32_t* idx = topk_idx ? topk_idx : (int32_t*)((char*)ws + L.idx);
  float* w = topk_w ? topk_w : (float*)((char*)ws + L.w);
  qe_expert* table = const_cast<qe_expert*>(lw->experts);
  if (T == 1 && fused_fits(c, x, x_dtype, lw->gamma)) {
    // one token: routing and resolve in one kernel, the fill, then the
    // single-token kernel with this routing (it does not route again, so it
    // reads exactly the experts resolved here)
    TierRoute r{x, x_dtype == QE_BF16, lw->gamma, lw->router_w, lw->logit_offset, c->hidden, c->n_experts,
                c->top_k, c->eps, (double*)((char*)ws + L.logits), idx, w};
    cudaError_t e;
    {
      std::lock_guard<std::mutex> lock(t->mu);
      e = launch_pdl(tier_route_kernel, (c->n_experts + kRouteRows - 1) / kRouteRows, kResolveThreads, s, r, t->d,
                     layer, table);
      if (e == cudaSuccess) e = launch_pdl(tier_fill_kernel, t->sms, kFillThreads, s, t->d);
    }
    if (e != cudaSuccess) return cuda_fail(e, "tier routing launch");
    return fused_step(c, lw, x, x_dtype, out, add_residual, nullptr, nullptr, ws, idx, w, s);
  }
  // several tokens (or a token the single-token kernel does not take): the
  // route kernels, resolve + fill, then the batched experts and combine
  rc = route_impl(c, x, x_dtype, lw->gamma, lw->router_w, lw->logit_offset, T, nullptr, idx, w, ws, ws_bytes,
                  true, s);
  if (rc) return rc;
  {
    std::lock_guard<std::mutex> lock(t->mu);
    rc = launch_resolve(t, layer, idx, T * c->top_k, table, s);
  }
  if (rc) return rc;
  return experts_and_combine(c, lw->experts, idx, w, x, x_dtype, T, out, add_residual, ws, s);
}

int qe_tier_stats(const qe_tier* t, uint64_t* hits, uint64_t* misses, uint64_t* h2d_bytes) {
  if (!t) return fail(QE_ERR_INVALID_ARG, "tier is NULL");
  int rc = check_device(t);
  if (rc) return rc;
  // the counters are updated by kernels on the caller's streams: wait for them
  cudaError_t e = cudaDeviceSynchronize();
  TierState st{};
  if (e == cudaSuccess) e = cudaMemcpy(&st, t->d.st, sizeof(st), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "qe_tier_stats");
  if (hits) *hits = st.hits;
  if (misses) *misses = st.misses;
  if (h2d_bytes) *h2d_bytes = st.h2d_bytes;
  if (st.status != QE_OK) return fail(st.status, "tier: a resolve on the device failed (status %d)", st.status);
  return QE_OK;
}

int qe_tier_slots(const qe_tier* t) { return t ? t->n_slots : 0; }

void qe_tier_destroy(qe_tier* t) { tier_free(t); }

}  // extern "C"
