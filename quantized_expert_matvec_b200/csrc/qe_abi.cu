// qe_abi.cu -- the extern "C" entry points of include/qexpert.h: argument
// validation, error strings, workspace layout and kernel dispatch.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "qe_internal.h"

namespace qe {

static thread_local char g_err[512] = "";
static unsigned long long g_budget_ns = 200ull * 1000 * 1000;
static int g_skip_cta = -1;
static unsigned long long* g_trace = nullptr;

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(QE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

static size_t al(size_t v) { return (v + 255) & ~(size_t)255; }

qe_expert pool_descriptor(const qe_cfg* c, void* base, int bits) {
  const size_t H = c->hidden, I = c->inter;
  const size_t wq = al(I * H * bits / 8), sb = al(I * H / kGroup * 2);
  char* b = (char*)base;
  qe_expert x{};
  x.gate = {(const uint32_t*)b, (const uint16_t*)(b + 3 * wq), (const uint16_t*)(b + 3 * wq + sb), bits, 0};
  x.up = {(const uint32_t*)(b + wq), (const uint16_t*)(b + 3 * wq + 2 * sb), (const uint16_t*)(b + 3 * wq + 3 * sb),
          bits, 0};
  x.down = {(const uint32_t*)(b + 2 * wq), (const uint16_t*)(b + 3 * wq + 4 * sb),
            (const uint16_t*)(b + 3 * wq + 5 * sb), bits, 0};
  return x;
}

WsLayout ws_layout(int H, int E, int K, int I, int T) {
  WsLayout L{};
  const size_t t = T > 0 ? (size_t)T : 1;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = al(off + bytes); return o; };
  L.control = take(sizeof(WsControl));
  // the single-token kernel's records first: their place depends on the
  // shape only, not on T, so no batched call on the same workspace writes there
  L.f_logit = take(128 * (size_t)kMaxGrid);
  L.f_h = take(8 * (size_t)K * I);
  L.f_done = take(8 * (size_t)kMaxGrid * kDoneStride);
  const size_t nlog = (size_t)E * (t > 2 ? t : 2);
  L.logits = take(8 * nlog);
  L.rinv = take(8 * t);
  L.xg = take(8 * t * H);
  L.xn = take(4 * t * H);
  L.xp4 = take(4 * t * H);
  L.xp2 = take(4 * t * H);
  L.xsum = take(4 * t * (H / 32));
  L.xexp = take(4 * t);
  L.h = take(4 * t * K * I);
  L.hp = take(4 * t * K * I);
  L.hsum = take(4 * t * K * (I / 32));
  L.hexp = take(4 * t * K);
  L.hamax = take(4 * t * K);
  L.y = take(4 * t * K * H);
  L.idx = take(4 * t * K);
  L.w = take(4 * t * K);
  L.grp_count = take(4 * ((size_t)E + 8));
  L.grp_start = take(4 * ((size_t)E + 1));
  L.grp_list = take(4 * t * K);
  L.grp_order = take(4 * (size_t)E);
  L.xh = take(2 * t * H);
  L.xin = take(4 * t * H);
  L.xout = take(4 * t * H);
  L.total = off;
  return L;
}

int check_cfg(const qe_cfg* c) {
  if (!c) return fail(QE_ERR_INVALID_ARG, "cfg is NULL");
  if (c->group != kGroup) return fail(QE_ERR_INVALID_ARG, "group must be 64 (got %d)", c->group);
  if (c->hidden <= 0 || c->hidden % kGroup || c->hidden > kMaxDim)
    return fail(QE_ERR_INVALID_ARG, "hidden must be a positive multiple of 64 <= %d (got %d)", kMaxDim, c->hidden);
  if (c->inter <= 0 || c->inter % kGroup || c->inter > kMaxDim)
    return fail(QE_ERR_INVALID_ARG, "inter must be a positive multiple of 64 <= %d (got %d)", kMaxDim, c->inter);
  if (c->n_experts <= 0 || c->n_experts > kMaxE)
    return fail(QE_ERR_INVALID_ARG, "n_experts must be in [1, %d] (got %d)", kMaxE, c->n_experts);
  if (c->top_k <= 0 || c->top_k > kMaxK || c->top_k > c->n_experts)
    return fail(QE_ERR_INVALID_ARG, "top_k must be in [1, min(16, n_experts)] (got %d)", c->top_k);
  if (!(c->eps >= 0.0f)) return fail(QE_ERR_INVALID_ARG, "eps must be >= 0");
  return QE_OK;
}

// Pointers must be aligned to `align` bytes: their element size, or 16 where
// the kernels read them with 128-bit loads (router rows).
int check_ptr(const void* p, const char* name, bool may_be_null, unsigned align) {
  if (!p) return may_be_null ? QE_OK : fail(QE_ERR_INVALID_ARG, "%s is NULL", name);
  if (((uintptr_t)p & (align - 1)) != 0) return fail(QE_ERR_INVALID_ARG, "%s is not %u-byte aligned", name, align);
  return QE_OK;
}

int check_ws(const qe_cfg* c, int T, void* ws, size_t bytes) {
  if (!ws) return fail(QE_ERR_INVALID_ARG, "workspace is NULL");
  if (((uintptr_t)ws & 255) != 0) return fail(QE_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const size_t need = ws_layout(c->hidden, c->n_experts, c->top_k, c->inter, T).total;
  if (bytes < need) return fail(QE_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", bytes, need);
  return QE_OK;
}

template <typename P>
static P* at(void* base, size_t off) { return (P*)((char*)base + off); }

DevInfo dev_info() {
  static std::mutex mu;
  static DevInfo cache[64];
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  DevInfo& d = cache[dev & 63];
  if (d.sms == 0) {
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&d.optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  }
  return d;
}

int route_impl(const qe_cfg* c, const void* x, int x_dtype, const float* gamma, const float* router_w,
                      const float* offset, int T, float* xn, int32_t* idx, float* w, void* ws, size_t ws_bytes,
                      bool want_xprime, cudaStream_t s) {
  const WsLayout L = ws_layout(c->hidden, c->n_experts, c->top_k, c->inter, T);
  RouteParams p{};
  p.H = c->hidden; p.E = c->n_experts; p.K = c->top_k; p.T = T; p.eps = c->eps;
  p.x = x; p.x_bf16 = x_dtype == QE_BF16; p.gamma = gamma; p.router_w = router_w; p.offset = offset;
  p.xn_out = xn; p.idx = idx; p.w = w;
  p.rinv = at<double>(ws, L.rinv); p.xg = at<double>(ws, L.xg); p.logits = at<double>(ws, L.logits);
  p.xn_ws = at<float>(ws, L.xn);
  if (want_xprime) {
    p.xp4 = at<float>(ws, L.xp4); p.xp2 = at<float>(ws, L.xp2); p.xsum = at<float>(ws, L.xsum);
    p.xexp = at<int>(ws, L.xexp);
    p.xh = at<uint16_t>(ws, L.xh);
  }
  p.err = &at<WsControl>(ws, L.control)->err;
  cudaError_t e = launch_route(p, s);
  if (e != cudaSuccess) return cuda_fail(e, "moe_route launch");
  return QE_OK;
}

static int ffn_impl(const qe_cfg* c, const qe_expert* experts, const float* xn, const int32_t* idx, int T, float* y,
                    void* ws, size_t ws_bytes, int mode, bool skip_xprep, cudaStream_t s) {
  const WsLayout L = ws_layout(c->hidden, c->n_experts, c->top_k, c->inter, T);
  FfnParams p{};
  p.H = c->hidden; p.K = c->top_k; p.I = c->inter; p.T = T; p.mode = mode;
  p.experts = experts; p.idx = idx; p.xn = xn;
  p.xp4 = at<float>(ws, L.xp4); p.xp2 = at<float>(ws, L.xp2); p.xsum = at<float>(ws, L.xsum);
  p.xexp = at<int>(ws, L.xexp);
  p.h = at<float>(ws, L.h); p.hp = at<float>(ws, L.hp); p.hsum = at<float>(ws, L.hsum);
  p.hexp = at<int>(ws, L.hexp); p.hamax = at<unsigned>(ws, L.hamax);
  p.y = y; p.err = &at<WsControl>(ws, L.control)->err; p.skip_xprep = skip_xprep;
  cudaError_t e = launch_ffn(p, s);
  if (e != cudaSuccess) return cuda_fail(e, "moe_expert_ffn launch");
  return QE_OK;
}

// The single-token kernel reads x (and gamma) four elements at a time: it
// takes a token whose x is 16-byte aligned (8 for bf16) and whose gamma, if
// any, is 16-byte aligned; other tokens take the multi-kernel path.
bool fused_aligned(const void* x, int x_dtype, const float* gamma) {
  if (((uintptr_t)x & (x_dtype == QE_BF16 ? 7u : 15u)) != 0) return false;
  return gamma == nullptr || ((uintptr_t)gamma & 15u) == 0;
}

bool fused_fits(const qe_cfg* c, const void* x, int x_dtype, const float* gamma) {
  if (!fused_aligned(x, x_dtype, gamma)) return false;
  const DevInfo d = dev_info();
  FusedGeometry g;
  return fused_geometry(c->hidden, c->n_experts, c->top_k, c->inter, d.sms, d.optin, &g) == QE_OK;
}

int fused_step(const qe_cfg* c, const qe_layer* layer, const void* x, int x_dtype, float* out, int add_residual,
               int32_t* topk_idx, float* topk_w, void* ws, const int32_t* given_idx, const float* given_w,
               cudaStream_t s) {
  const WsLayout L = ws_layout(c->hidden, c->n_experts, c->top_k, c->inter, 1);
  FusedParams p{};
  const DevInfo d = dev_info();
  if (fused_geometry(c->hidden, c->n_experts, c->top_k, c->inter, d.sms, d.optin, &p.g) != QE_OK)
    return fail(QE_ERR_UNSUPPORTED, "shape not supported by the single-token kernel");
  p.H = c->hidden; p.E = c->n_experts; p.K = c->top_k; p.I = c->inter; p.eps = c->eps;
  p.x = x; p.x_bf16 = x_dtype == QE_BF16; p.add_residual = add_residual != 0;
  p.gamma = layer->gamma; p.router_w = layer->router_w; p.offset = layer->logit_offset;
  p.experts = layer->experts; p.out = out; p.topk_idx = topk_idx; p.topk_w = topk_w;
  p.ctl = at<WsControl>(ws, L.control);
  p.rec_logit = at<unsigned long long>(ws, L.f_logit);
  p.rec_h = at<unsigned long long>(ws, L.f_h);
  p.rec_done = at<unsigned long long>(ws, L.f_done);
  p.given_idx = given_idx;
  p.given_w = given_w;
  p.budget_ns = g_budget_ns;
  p.skip_cta = g_skip_cta;
  p.trace = g_trace;
  cudaError_t e = launch_fused_layer(p, s);
  if (e != cudaSuccess) return cuda_fail(e, "fused layer launch");
  return QE_OK;
}

}  // namespace qe

using namespace qe;

extern "C" {

const char* qe_last_error(void) { return g_err; }

const char* qe_version(void) { return "qexpert 0.1 (sm_100a)"; }

size_t qe_expert_bytes(const qe_cfg* c, int bits) {
  if (check_cfg(c) != QE_OK || !(bits == 4 || bits == 2)) return 0;
  const size_t H = c->hidden, I = c->inter;
  const size_t wq = al(I * H * bits / 8), sb = al(I * H / kGroup * 2);
  return 3 * wq + 6 * sb;
}

int qe_pool_table(const qe_cfg* c, void* base, int bits, int n, qe_expert* out, size_t* seg) {
  int rc = check_cfg(c);
  if (rc) return rc;
  if (!(bits == 4 || bits == 2)) return fail(QE_ERR_INVALID_ARG, "bits must be 4 or 2 (got %d)", bits);
  if (n < 0 || (n > 0 && (!base || !out))) return fail(QE_ERR_INVALID_ARG, "bad pool arguments");
  if (((uintptr_t)base & 255) != 0) return fail(QE_ERR_INVALID_ARG, "pool base must be 256-byte aligned");
  const size_t H = c->hidden, I = c->inter;
  const size_t wq = al(I * H * bits / 8), sb = al(I * H / kGroup * 2);
  const size_t offs[9] = {0, wq, 2 * wq, 3 * wq, 3 * wq + sb, 3 * wq + 2 * sb, 3 * wq + 3 * sb,
                          3 * wq + 4 * sb, 3 * wq + 5 * sb};
  if (seg) memcpy(seg, offs, sizeof(offs));
  const size_t stride = 3 * wq + 6 * sb;
  for (int e = 0; e < n; ++e) out[e] = pool_descriptor(c, (char*)base + (size_t)e * stride, bits);
  return QE_OK;
}

size_t qe_workspace_bytes(const qe_cfg* c, int T) {
  if (check_cfg(c) != QE_OK || T < 0) return 0;
  return ws_layout(c->hidden, c->n_experts, c->top_k, c->inter, T).total;
}

int qe_workspace_init(void* ws, size_t bytes, qe_stream_t stream) {
  if (!ws || bytes < sizeof(WsControl)) return fail(QE_ERR_INVALID_ARG, "bad workspace");
  cudaError_t e = cudaMemsetAsync(ws, 0, bytes, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "qe_workspace_init");
  return QE_OK;
}

int qe_workspace_status(void* ws, qe_stream_t stream) {
  if (!ws) return fail(QE_ERR_INVALID_ARG, "workspace is NULL");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "qe_workspace_status sync");
  int err = 0;
  e = cudaMemcpy(&err, &((WsControl*)ws)->err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "qe_workspace_status read");
  if (err != 0) {
    const int zero = 0;
    cudaMemcpy(&((WsControl*)ws)->err, &zero, sizeof(int), cudaMemcpyHostToDevice);
    return fail(err, err == QE_ERR_TIMEOUT ? "a bounded device wait gave up (QE_ERR_TIMEOUT)"
                                           : "the device rejected an expert descriptor");
  }
  return QE_OK;
}

void qe_set_wait_budget_ns(uint64_t ns) { g_budget_ns = ns ? ns : 1; }

void qe_test_skip_arrival(int cta) { g_skip_cta = cta; }

void qe_trace_fused(void* dev_buf) { g_trace = (unsigned long long*)dev_buf; }

int moe_route(const qe_cfg* c, const void* x, int x_dtype, const float* gamma, const float* router_w,
              const float* logit_offset, int T, float* xn, int32_t* topk_idx, float* topk_w, void* ws,
              size_t ws_bytes, qe_stream_t stream) {
  int rc = check_cfg(c);
  if (rc) return rc;
  if (T < 0) return fail(QE_ERR_INVALID_ARG, "T must be >= 0");
  if (T == 0) return QE_OK;
  if (!(x_dtype == QE_F32 || x_dtype == QE_BF16)) return fail(QE_ERR_INVALID_ARG, "x_dtype must be QE_F32 or QE_BF16");
  if ((rc = check_ptr(x, "x", false, x_dtype == QE_BF16 ? 2 : 4)) || (rc = check_ptr(router_w, "router_w", false, 16)) || (rc = check_ptr(gamma, "gamma", true)) ||
      (rc = check_ptr(logit_offset, "logit_offset", true)) || (rc = check_ptr(xn, "xn", true)) ||
      (rc = check_ptr(topk_idx, "topk_idx")) || (rc = check_ptr(topk_w, "topk_w")) ||
      (rc = check_ws(c, T, ws, ws_bytes)))
    return rc;
  return route_impl(c, x, x_dtype, gamma, router_w, logit_offset, T, xn, topk_idx, topk_w, ws, ws_bytes, false,
                    (cudaStream_t)stream);
}

static int ffn_entry(const qe_cfg* c, const qe_expert* experts, const float* xn, const int32_t* idx, int T, float* y,
                     void* ws, size_t ws_bytes, int mode, cudaStream_t s) {
  int rc = check_cfg(c);
  if (rc) return rc;
  if (T < 0) return fail(QE_ERR_INVALID_ARG, "T must be >= 0");
  if (T == 0) return QE_OK;
  if ((rc = check_ptr(experts, "experts", false, 8)) || (rc = check_ptr(xn, "xn")) || (rc = check_ptr(idx, "topk_idx")) ||
      (rc = check_ptr(y, "y")) || (rc = check_ws(c, T, ws, ws_bytes)))
    return rc;
  return ffn_impl(c, experts, xn, idx, T, y, ws, ws_bytes, mode, false, s);
}

int moe_expert_ffn_q4(const qe_cfg* c, const qe_expert* experts, const float* xn, const int32_t* idx, int T, float* y,
                      void* ws, size_t ws_bytes, qe_stream_t stream) {
  return ffn_entry(c, experts, xn, idx, T, y, ws, ws_bytes, 4, (cudaStream_t)stream);
}

int moe_expert_ffn_q2(const qe_cfg* c, const qe_expert* experts, const float* xn, const int32_t* idx, int T, float* y,
                      void* ws, size_t ws_bytes, qe_stream_t stream) {
  return ffn_entry(c, experts, xn, idx, T, y, ws, ws_bytes, 2, (cudaStream_t)stream);
}

int moe_expert_ffn_mixed(const qe_cfg* c, const qe_expert* experts, const float* xn, const int32_t* idx, int T,
                         float* y, void* ws, size_t ws_bytes, qe_stream_t stream) {
  return ffn_entry(c, experts, xn, idx, T, y, ws, ws_bytes, 0, (cudaStream_t)stream);
}

int moe_combine(const float* y, const float* w, const float* residual, int T, int K, int H, float* out,
                qe_stream_t stream) {
  if (T < 0 || K <= 0 || K > kMaxK || H <= 0) return fail(QE_ERR_INVALID_ARG, "bad combine shape");
  if (T == 0) return QE_OK;
  int rc;
  if ((rc = check_ptr(y, "y")) || (rc = check_ptr(w, "w")) || (rc = check_ptr(residual, "residual", true)) ||
      (rc = check_ptr(out, "out")))
    return rc;
  cudaError_t e = launch_combine(y, w, residual, 0, T, K, H, out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "moe_combine launch");
  return QE_OK;
}

int moe_layer_step(const qe_cfg* c, const qe_layer* layer, const void* x, int x_dtype, int T, float* out,
                   int add_residual, int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                   qe_stream_t stream) {
  int rc = check_cfg(c);
  if (rc) return rc;
  if (!layer) return fail(QE_ERR_INVALID_ARG, "layer is NULL");
  if (T < 0) return fail(QE_ERR_INVALID_ARG, "T must be >= 0");
  if (T == 0) return QE_OK;
  if (!(x_dtype == QE_F32 || x_dtype == QE_BF16)) return fail(QE_ERR_INVALID_ARG, "x_dtype must be QE_F32 or QE_BF16");
  if ((rc = check_ptr(x, "x", false, x_dtype == QE_BF16 ? 2 : 4)) || (rc = check_ptr(out, "out")) || (rc = check_ptr(layer->router_w, "router_w", false, 16)) ||
      (rc = check_ptr(layer->experts, "experts", false, 8)) || (rc = check_ptr(layer->gamma, "gamma", true)) ||
      (rc = check_ptr(layer->logit_offset, "logit_offset", true)) || (rc = check_ptr(topk_idx, "topk_idx", true)) ||
      (rc = check_ptr(topk_w, "topk_w", true)) || (rc = check_ws(c, T, ws, ws_bytes)))
    return rc;
  if ((const void*)out == x) return fail(QE_ERR_INVALID_ARG, "out must not alias x");
  cudaStream_t s = (cudaStream_t)stream;
  const WsLayout L = ws_layout(c->hidden, c->n_experts, c->top_k, c->inter, T);
  if (T == 1 && fused_fits(c, x, x_dtype, layer->gamma)) return fused_step(c, layer, x, x_dtype, out, add_residual, topk_idx, topk_w, ws,
                                                   nullptr, nullptr, s);
  // batched (or a single token whose shape does not fit the fused kernel):
  // route all tokens, then the expert FFNs, then the combine
  int32_t* idx = topk_idx ? topk_idx : at<int32_t>(ws, L.idx);
  float* w = topk_w ? topk_w : at<float>(ws, L.w);
  rc = route_impl(c, x, x_dtype, layer->gamma, layer->router_w, layer->logit_offset, T, nullptr, idx, w, ws, ws_bytes,
                  true, s);
  if (rc) return rc;
  return experts_and_combine(c, layer->experts, idx, w, x, x_dtype, T, out, add_residual, ws, s);
}

}  // extern "C"

namespace qe {

// Expert FFNs of routed tokens (x' already prepared by route_impl with
// want_xprime), then the weighted combine: the batched half of the layer step.
int experts_and_combine(const qe_cfg* c, const qe_expert* experts, const int32_t* idx, const float* w, const void* x,
                        int x_dtype, int T, float* out, int add_residual, void* ws, cudaStream_t s) {
  const WsLayout L = ws_layout(c->hidden, c->n_experts, c->top_k, c->inter, T);
  {
    GroupedParams gp{};
    gp.H = c->hidden; gp.E = c->n_experts; gp.K = c->top_k; gp.I = c->inter; gp.T = T;
    gp.experts = experts; gp.idx = idx; gp.w = w;
    gp.xp4 = at<float>(ws, L.xp4); gp.xp2 = at<float>(ws, L.xp2); gp.xsum = at<float>(ws, L.xsum);
    gp.xexp = at<int>(ws, L.xexp);
    gp.h = at<float>(ws, L.h); gp.hamax = at<unsigned>(ws, L.hamax);
    gp.xh = at<uint16_t>(ws, L.xh);
    gp.budget_ns = g_budget_ns;
    gp.y = at<float>(ws, L.y);
    gp.grp_count = at<int>(ws, L.grp_count); gp.grp_start = at<int>(ws, L.grp_start);
    gp.grp_list = at<int>(ws, L.grp_list); gp.grp_order = at<int>(ws, L.grp_order);
    gp.err = &at<WsControl>(ws, L.control)->err;
    cudaError_t ge = launch_grouped(gp, s);
    if (ge != cudaSuccess) return cuda_fail(ge, "moe_layer_step grouped experts");
  }
  cudaError_t e = launch_combine(at<float>(ws, L.y), w, add_residual ? x : nullptr, x_dtype == QE_BF16, T,
                                 c->top_k, c->hidden, out, s);
  if (e != cudaSuccess) return cuda_fail(e, "moe_layer_step combine");
  return QE_OK;
}

}  // namespace qe

extern "C" int moe_layer_step_host(const qe_cfg* c, const qe_layer* layer, const void* x_host, int x_dtype, int T,
                                   float* out_host, int add_residual, void* ws, size_t ws_bytes, qe_stream_t stream) {
  int rc = check_cfg(c);
  if (rc) return rc;
  if (T < 0) return fail(QE_ERR_INVALID_ARG, "T must be >= 0");
  if (T == 0) return QE_OK;
  if (!(x_dtype == QE_F32 || x_dtype == QE_BF16)) return fail(QE_ERR_INVALID_ARG, "x_dtype must be QE_F32 or QE_BF16");
  if (!x_host || !out_host) return fail(QE_ERR_INVALID_ARG, "x_host and out_host must not be NULL");
  if ((rc = check_ws(c, T, ws, ws_bytes))) return rc;
  const WsLayout L = ws_layout(c->hidden, c->n_experts, c->top_k, c->inter, T);
  cudaStream_t s = (cudaStream_t)stream;
  const size_t xb = (size_t)T * c->hidden * (x_dtype == QE_BF16 ? 2 : 4);
  const size_t ob = (size_t)T * c->hidden * 4;
  void* xd = at<unsigned char>(ws, L.xin);
  float* od = at<float>(ws, L.xout);
  cudaError_t e = cudaMemcpyAsync(xd, x_host, xb, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "moe_layer_step_host: copy x in");
  rc = moe_layer_step(c, layer, xd, x_dtype, T, od, add_residual, nullptr, nullptr, ws, ws_bytes, stream);
  if (rc) return rc;
  e = cudaMemcpyAsync(out_host, od, ob, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "moe_layer_step_host: copy out");
  return QE_OK;
}

// ---------------------------------------------------------------------------
// Single-token layer step whose scratch lives in the library itself.
//
// The fused single-token kernel needs device scratch besides its inputs and
// outputs: the control block (error word, launch epoch), the tagged router
// logits, the tagged SwiGLU activations and one "read the epoch" record per
// CTA.
// moe_layer_step takes them from a caller-allocated workspace; the entry
// point below takes them from a fixed array that every GPU loading this
// library holds until the process exits.
namespace qe {

constexpr size_t kStaticMaxKI = 16384;                                   // top_k * inter: 16 x 1024
constexpr size_t kStaticLogitsOff = sizeof(WsControl);                   // 256
constexpr size_t kStaticHOff = kStaticLogitsOff + 128 * (size_t)kMaxGrid;  // + 32 KiB of logit records
constexpr size_t kStaticDoneOff = kStaticHOff + 8 * kStaticMaxKI;          // + 128 KiB of h records
constexpr size_t kStaticBytes = kStaticDoneOff + 8 * (size_t)kMaxGrid * kDoneStride;  // + 8 KiB: 172,288 bytes

static __device__ __align__(256) unsigned char g_static_scratch[kStaticBytes];

// Device address of g_static_scratch on the current device.  In host code the
// name g_static_scratch only stands for the symbol, so the address is asked
// of the runtime once per device (with that device current) and cached.
static int static_scratch(unsigned char** out) {
  static std::mutex mu;
  static unsigned char* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "moe_layer_step_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(QE_ERR_UNSUPPORTED, "moe_layer_step_noalloc: device %d >= 64", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "moe_layer_step_noalloc: cudaGetSymbolAddress");
    if (!p || ((uintptr_t)p & 255) != 0)
      return fail(QE_ERR_CUDA, "moe_layer_step_noalloc: scratch address %p is not 256-byte aligned", p);
    addr[dev] = (unsigned char*)p;
  }
  *out = addr[dev];
  return QE_OK;
}

}  // namespace qe

extern "C" int moe_layer_step_noalloc(const qe_cfg* c, const qe_layer* layer, const void* x, int x_dtype,
                                      float* out, int add_residual, int32_t* topk_idx, float* topk_w,
                                      int32_t* dev_status, qe_stream_t stream) {
  int rc = check_cfg(c);
  if (rc) return rc;
  if (!layer) return fail(QE_ERR_INVALID_ARG, "layer is NULL");
  if (!(x_dtype == QE_F32 || x_dtype == QE_BF16)) return fail(QE_ERR_INVALID_ARG, "x_dtype must be QE_F32 or QE_BF16");
  if ((size_t)c->top_k * (size_t)c->inter > kStaticMaxKI)
    return fail(QE_ERR_INVALID_ARG,
                "moe_layer_step_noalloc: top_k * inter = %d exceeds the built-in scratch limit of %zu "
                "(use moe_layer_step with a workspace)",
                c->top_k * c->inter, kStaticMaxKI);
  if ((rc = check_ptr(x, "x", false, x_dtype == QE_BF16 ? 2 : 4)) || (rc = check_ptr(out, "out")) ||
      (rc = check_ptr(layer->router_w, "router_w", false, 16)) || (rc = check_ptr(layer->experts, "experts", false, 8)) ||
      (rc = check_ptr(layer->gamma, "gamma", true)) || (rc = check_ptr(layer->logit_offset, "logit_offset", true)) ||
      (rc = check_ptr(topk_idx, "topk_idx", true)) || (rc = check_ptr(topk_w, "topk_w", true)) ||
      (rc = check_ptr(dev_status, "dev_status", true)))
    return rc;
  if ((const void*)out == x) return fail(QE_ERR_INVALID_ARG, "out must not alias x");
  if (!fused_aligned(x, x_dtype, layer->gamma))
    return fail(QE_ERR_INVALID_ARG,
                "moe_layer_step_noalloc: x must be 16-byte aligned (8 for bf16) and gamma 16-byte aligned");
  FusedParams p{};
  const DevInfo d = dev_info();
  if (fused_geometry(c->hidden, c->n_experts, c->top_k, c->inter, d.sms, d.optin, &p.g) != QE_OK)
    return fail(QE_ERR_UNSUPPORTED,
                "moe_layer_step_noalloc: shape not supported by the single-token kernel (hidden %d must be <= "
                "4096, inter %d <= 1024, n_experts %d <= 8 x SMs, and the experts' share of one SM must fit "
                "in its shared memory)",
                c->hidden, c->inter, c->n_experts);
  unsigned char* scratch = nullptr;
  if ((rc = static_scratch(&scratch))) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  WsControl* ctl = (WsControl*)scratch;
  // the previous call's error word is cleared; its launch epoch stays, so
  // this call's records carry a tag no earlier call wrote
  cudaError_t e = cudaMemsetAsync(&ctl->err, 0, sizeof(ctl->err), s);
  if (e != cudaSuccess) return cuda_fail(e, "moe_layer_step_noalloc: clear the error word");
  p.H = c->hidden; p.E = c->n_experts; p.K = c->top_k; p.I = c->inter; p.eps = c->eps;
  p.x = x; p.x_bf16 = x_dtype == QE_BF16; p.add_residual = add_residual != 0;
  p.gamma = layer->gamma; p.router_w = layer->router_w; p.offset = layer->logit_offset;
  p.experts = layer->experts; p.out = out; p.topk_idx = topk_idx; p.topk_w = topk_w;
  p.ctl = ctl;
  p.rec_logit = (unsigned long long*)(scratch + kStaticLogitsOff);
  p.rec_h = (unsigned long long*)(scratch + kStaticHOff);
  p.rec_done = (unsigned long long*)(scratch + kStaticDoneOff);
  p.budget_ns = g_budget_ns;
  p.skip_cta = g_skip_cta;
  p.trace = g_trace;
  e = launch_fused_layer(p, s);
  if (e != cudaSuccess) return cuda_fail(e, "moe_layer_step_noalloc launch");
  if (dev_status) {
    e = cudaMemcpyAsync(dev_status, &ctl->err, sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "moe_layer_step_noalloc: copy status");
  }
  return QE_OK;
}
