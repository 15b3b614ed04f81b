// qe_tier.cu -- two-tier expert residency: hot experts resident in HBM, cold
// experts in pinned host memory behind an HBM cache of expert slots with LRU
// replacement, misses copied host->device on a side stream.
//
// Follows the tiering of the Flash-MoE pages (lilting.ch "Flash-MoE: running
// a 397B-parameter model on a 48 GB MacBook", sections "Core technique: SSD
// expert streaming" and "Trust the OS": experts streamed from storage on
// demand into a page cache; nzkcom.pages.dev "flash-moe-romance-vs-utility",
// adopted optimisations: frequently used experts kept at 4 bits, the rest
// at 2 bits).  On B200 the storage tier is pinned host memory over PCIe and
// the cache is a pool of HBM slots managed here instead of by an OS.
#include <list>
#include <mutex>
#include <vector>

#include "qe_internal.h"

struct qe_tier {
  qe_cfg cfg;
  int L = 0, E = 0, bits = 2, dev = 0, max_tokens = 0;
  size_t slot_bytes = 0, expert_bytes = 0;
  int n_slots = 0;
  std::vector<const void*> cold_host;  // [L*E], NULL for a hot expert
  unsigned char* cache = nullptr;      // device, n_slots * slot_bytes
  // LRU over slots: head = most recently used.  Free slots sit at the tail.
  std::vector<int> slot_key, key_slot, prev, next;
  std::vector<unsigned> slot_call;  // slot claimed by call number slot_call[s]
  std::vector<unsigned> key_call;   // key seen in call number key_call[k]
  int head = -1, tail = -1;
  unsigned call = 0;
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t ev_main = nullptr, ev_copy = nullptr, ev_idx = nullptr, ev_stage = nullptr;
  int32_t* idx_host = nullptr;      // pinned [max_tokens * K]
  qe_expert* stage_host = nullptr;  // pinned [max_tokens * K] descriptors
  int32_t* pos_host = nullptr;      // pinned [max_tokens * K] table positions
  qe_expert* stage_dev = nullptr;   // device copies of the two arrays above
  int32_t* pos_dev = nullptr;
  unsigned long long hits = 0, misses = 0, h2d_bytes = 0;
  std::mutex mu;
};

namespace qe {

// Scatter n descriptors into a device table: table[pos[j]] = desc[j].
__global__ void tier_scatter_kernel(const qe_expert* desc, const int32_t* pos, int n, qe_expert* table) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j < n) table[pos[j]] = desc[j];
}

static void lru_unlink(qe_tier* t, int s) {
  if (t->prev[s] >= 0) t->next[t->prev[s]] = t->next[s];
  else t->head = t->next[s];
  if (t->next[s] >= 0) t->prev[t->next[s]] = t->prev[s];
  else t->tail = t->prev[s];
  t->prev[s] = t->next[s] = -1;
}

static void lru_push_front(qe_tier* t, int s) {
  t->prev[s] = -1;
  t->next[s] = t->head;
  if (t->head >= 0) t->prev[t->head] = s;
  t->head = s;
  if (t->tail < 0) t->tail = s;
}

static int check_device(const qe_tier* t) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != t->dev) return fail(QE_ERR_INVALID_ARG, "tier belongs to device %d, current device is %d", t->dev, dev);
  return QE_OK;
}

static void tier_free(qe_tier* t) {
  if (!t) return;
  if (t->copy_stream) cudaStreamSynchronize(t->copy_stream);
  if (t->ev_stage) cudaEventSynchronize(t->ev_stage);
  if (t->cache) cudaFree(t->cache);
  if (t->stage_dev) cudaFree(t->stage_dev);
  if (t->pos_dev) cudaFree(t->pos_dev);
  if (t->idx_host) cudaFreeHost(t->idx_host);
  if (t->stage_host) cudaFreeHost(t->stage_host);
  if (t->pos_host) cudaFreeHost(t->pos_host);
  for (cudaEvent_t ev : {t->ev_main, t->ev_copy, t->ev_idx, t->ev_stage})
    if (ev) cudaEventDestroy(ev);
  if (t->copy_stream) cudaStreamDestroy(t->copy_stream);
  delete t;
}

// Resolve the experts of one call (caller holds t->mu).
static int resolve_locked(qe_tier* t, int layer, const int32_t* idx, int n, qe_expert* dev_table, cudaStream_t s) {
  const int E = t->E;
  ++t->call;
  if (t->call == 0) {  // wrapped: forget old claims
    std::fill(t->slot_call.begin(), t->slot_call.end(), 0u);
    std::fill(t->key_call.begin(), t->key_call.end(), 0u);
    t->call = 1;
  }
  for (int i = 0; i < n; ++i)
    if (idx[i] < 0 || idx[i] >= E) return fail(QE_ERR_INVALID_ARG, "expert index %d out of range [0, %d)", idx[i], E);
  // pass 1: hits claim their slots, so that no miss of this call evicts them
  int n_cold = 0;
  for (int i = 0; i < n; ++i) {
    const int key = layer * E + idx[i];
    if (!t->cold_host[key] || t->key_call[key] == t->call) continue;
    t->key_call[key] = t->call;
    ++n_cold;
    const int sl = t->key_slot[key];
    if (sl >= 0) {
      t->slot_call[sl] = t->call;
      lru_unlink(t, sl);
      lru_push_front(t, sl);
    }
  }
  if (n_cold > t->n_slots)
    return fail(QE_ERR_OOM, "one call needs %d cold experts but the cache holds %d slots", n_cold, t->n_slots);
  // pass 2: misses take the least recently used unclaimed slot
  int nd = 0, n_miss = 0;
  for (int i = 0; i < n; ++i) {
    const int key = layer * E + idx[i];
    if (!t->cold_host[key] || t->key_call[key] != t->call) continue;
    t->key_call[key] = t->call - 1;  // emit each distinct expert once (call - 1 != call)
    int sl = t->key_slot[key];
    if (sl >= 0) {
      ++t->hits;
    } else {
      sl = t->tail;
      while (sl >= 0 && t->slot_call[sl] == t->call) sl = t->prev[sl];
      if (sl < 0) return fail(QE_ERR_OOM, "no free cache slot");
      if (t->slot_key[sl] >= 0) t->key_slot[t->slot_key[sl]] = -1;
      t->slot_key[sl] = key;
      t->key_slot[key] = sl;
      t->slot_call[sl] = t->call;
      lru_unlink(t, sl);
      lru_push_front(t, sl);
      if (n_miss == 0) {
        // the copy may overwrite a slot that work already queued on `s` reads
        cudaError_t e = cudaEventRecord(t->ev_main, s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(t->copy_stream, t->ev_main, 0);
        if (e != cudaSuccess) return cuda_fail(e, "tier: order the copy stream after the compute stream");
      }
      cudaError_t e = cudaMemcpyAsync(t->cache + (size_t)sl * t->slot_bytes, t->cold_host[key], t->expert_bytes,
                                      cudaMemcpyHostToDevice, t->copy_stream);
      if (e != cudaSuccess) return cuda_fail(e, "tier: expert copy");
      ++t->misses;
      t->h2d_bytes += t->expert_bytes;
      ++n_miss;
    }
    if (nd == 0) {
      // the staging arrays of the previous call must have been consumed
      cudaError_t e = cudaEventSynchronize(t->ev_stage);
      if (e != cudaSuccess) return cuda_fail(e, "tier: staging wait");
    }
    t->stage_host[nd] = pool_descriptor(&t->cfg, t->cache + (size_t)sl * t->slot_bytes, t->bits);
    t->pos_host[nd] = idx[i];
    ++nd;
  }
  if (n_miss > 0) {
    cudaError_t e = cudaEventRecord(t->ev_copy, t->copy_stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, t->ev_copy, 0);
    if (e != cudaSuccess) return cuda_fail(e, "tier: order the compute stream after the copies");
  }
  if (nd > 0) {
    cudaError_t e = cudaMemcpyAsync(t->stage_dev, t->stage_host, sizeof(qe_expert) * nd, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(t->pos_dev, t->pos_host, sizeof(int32_t) * nd, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "tier: descriptor upload");
    tier_scatter_kernel<<<(nd + 127) / 128, 128, 0, s>>>(t->stage_dev, t->pos_dev, nd, dev_table);
    e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaEventRecord(t->ev_stage, s);
    if (e != cudaSuccess) return cuda_fail(e, "tier: descriptor scatter");
  }
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
  if (d->max_tokens <= 0) return fail(QE_ERR_INVALID_ARG, "max_tokens must be positive");
  const size_t eb = qe_expert_bytes(&d->cfg, d->cold_bits);
  const size_t nkeys = (size_t)d->n_layers * d->cfg.n_experts;
  if (nkeys > (size_t)0x7fffffff) return fail(QE_ERR_INVALID_ARG, "too many experts");
  const size_t n_slots = d->cache_bytes / eb;
  if (n_slots < 1) return fail(QE_ERR_INVALID_ARG, "cache_bytes %zu holds no %zu-byte expert", d->cache_bytes, eb);
  if (n_slots > (size_t)0x7fffffff) return fail(QE_ERR_INVALID_ARG, "cache too large");
  qe_tier* t = new qe_tier();
  t->cfg = d->cfg;
  t->L = d->n_layers;
  t->E = d->cfg.n_experts;
  t->bits = d->cold_bits;
  t->max_tokens = d->max_tokens;
  t->expert_bytes = eb;
  t->slot_bytes = eb;  // segments are 256-byte multiples already
  t->n_slots = (int)n_slots;
  t->cold_host.assign(d->cold_host, d->cold_host + nkeys);
  t->key_slot.assign(nkeys, -1);
  t->key_call.assign(nkeys, 0u);
  t->slot_key.assign(n_slots, -1);
  t->slot_call.assign(n_slots, 0u);
  t->prev.assign(n_slots, -1);
  t->next.assign(n_slots, -1);
  for (int s = (int)n_slots - 1; s >= 0; --s) lru_push_front(t, s);
  cudaError_t e = cudaGetDevice(&t->dev);
  const size_t nst = (size_t)d->max_tokens * d->cfg.top_k;
  if (e == cudaSuccess) {
    e = cudaMalloc(&t->cache, n_slots * t->slot_bytes);
    if (e != cudaSuccess) {
      cudaGetLastError();
      tier_free(t);
      return fail(QE_ERR_OOM, "tier: cudaMalloc of the %zu-byte expert cache failed", n_slots * eb);
    }
  }
  if (e == cudaSuccess) e = cudaMalloc(&t->stage_dev, sizeof(qe_expert) * nst);
  if (e == cudaSuccess) e = cudaMalloc(&t->pos_dev, sizeof(int32_t) * nst);
  if (e == cudaSuccess) e = cudaHostAlloc(&t->idx_host, sizeof(int32_t) * nst, cudaHostAllocDefault);
  if (e == cudaSuccess) e = cudaHostAlloc(&t->stage_host, sizeof(qe_expert) * nst, cudaHostAllocDefault);
  if (e == cudaSuccess) e = cudaHostAlloc(&t->pos_host, sizeof(int32_t) * nst, cudaHostAllocDefault);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&t->copy_stream, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&t->ev_main, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&t->ev_copy, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&t->ev_idx, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&t->ev_stage, cudaEventDisableTiming);
  if (e != cudaSuccess) {
    const int r = cuda_fail(e, "qe_tier_create");
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
  return resolve_locked(t, layer, host_idx, n, dev_table, (cudaStream_t)stream);
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
  if ((rc = check_device(t))) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  const WsLayout L = ws_layout(c->hidden, c->n_experts, c->top_k, c->inter, T);
  int32_t* idx = topk_idx ? topk_idx : (int32_t*)((char*)ws + L.idx);
  float* w = topk_w ? topk_w : (float*)((char*)ws + L.w);
  rc = route_impl(c, x, x_dtype, lw->gamma, lw->router_w, lw->logit_offset, T, nullptr, idx, w, ws, ws_bytes,
                  !(T == 1 && fused_fits(c, x, x_dtype, lw->gamma)), s);
  if (rc) return rc;
  std::lock_guard<std::mutex> lock(t->mu);
  const int n = T * c->top_k;
  // the one host synchronisation of the tiered step: the routing decides
  // which cold experts must be copied in
  cudaError_t e = cudaMemcpyAsync(t->idx_host, idx, sizeof(int32_t) * n, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaEventRecord(t->ev_idx, s);
  if (e == cudaSuccess) e = cudaEventSynchronize(t->ev_idx);
  if (e != cudaSuccess) return cuda_fail(e, "qe_tier_layer_step: read routing");
  rc = resolve_locked(t, layer, t->idx_host, n, const_cast<qe_expert*>(lw->experts), s);
  if (rc) return rc;
  // one token: the fused kernel with this routing (it does not route again,
  // so it reads exactly the experts resolved above)
  if (T == 1 && fused_fits(c, x, x_dtype, lw->gamma))
    return fused_step(c, lw, x, x_dtype, out, add_residual, nullptr, nullptr, ws, idx, w, s);
  return experts_and_combine(c, lw->experts, idx, w, x, x_dtype, T, out, add_residual, ws, s);
}

int qe_tier_stats(const qe_tier* t, uint64_t* hits, uint64_t* misses, uint64_t* h2d_bytes) {
  if (!t) return fail(QE_ERR_INVALID_ARG, "tier is NULL");
  qe_tier* m = const_cast<qe_tier*>(t);
  std::lock_guard<std::mutex> lock(m->mu);
  if (hits) *hits = t->hits;
  if (misses) *misses = t->misses;
  if (h2d_bytes) *h2d_bytes = t->h2d_bytes;
  return QE_OK;
}

int qe_tier_slots(const qe_tier* t) { return t ? t->n_slots : 0; }

void qe_tier_destroy(qe_tier* t) { tier_free(t); }

}  // extern "C"
