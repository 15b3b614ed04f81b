// qe_internal.h -- host/device shared declarations of the CUDA library
// (kernel parameter blocks, workspace layout, launch wrappers).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/qexpert.h"

namespace qe {

constexpr int kMaxK = 16;
constexpr int kMaxE = 1024;
constexpr int kMaxDim = 8192;
constexpr int kGroup = 64;

// Control words at the start of every workspace.
struct WsControl {
  int err;                       // first device-side error (QE_ERR_*), 0 if none
  // launch epoch of the single-token kernel: every launch reads it, tags the
  // records it publishes with epoch + 1 (top bit set) and, at the end, CTA 0
  // advances it
  unsigned epoch;
  unsigned pad[62];
};
static_assert(sizeof(WsControl) == 256, "control block");

// Offsets (bytes) of the workspace regions for T tokens.
struct WsLayout {
  size_t control;   // WsControl
  size_t logits;    // double [max(2E, T*E)]
  size_t rinv;      // double [T]
  size_t xg;        // double [T*H]   x*gamma for the router
  size_t xn;        // float  [T*H]   normalised activations
  size_t xp4;       // float  [T*H]   x' for 4-bit matrices
  size_t xp2;       // float  [T*H]   x' for 2-bit matrices
  size_t xsum;      // float  [T*H/32] 32-column sums of xn
  size_t xexp;      // int    [T]     vector exponent E of xn
  size_t h;         // float  [T*K*I] SwiGLU outputs
  size_t hp;        // float  [T*K*I] x' of h (bits of the expert's down matrix)
  size_t hsum;      // float  [T*K*I/32]
  size_t hexp;      // int    [T*K]
  size_t hamax;     // unsigned [T*K] |h| max as float bits
  size_t y;         // float  [T*K*H] expert outputs
  size_t idx;       // int32  [T*K]
  size_t w;         // float  [T*K]
  size_t grp_count; // int    [E+8]  assignments per expert, then the grouping control words
  size_t grp_start; // int    [E+1]
  size_t grp_list;  // int    [T*K]  assignment ids (t*K+k) sorted by expert
  size_t grp_order; // int    [E]    active experts, most tokens first
  size_t xh;        // fp16   [T*H]  xn for the tensor-core gate/up
  size_t xin;       // float  [T*H]  device copy of a host x (moe_layer_step_host)
  size_t xout;      // float  [T*H]  device result before its copy to the host
  size_t f_logit;   // u64 [kMaxGrid*16] single-token kernel: tagged router logits, one 128-byte line per CTA
  size_t f_h;       // u64 [K*I]       single-token kernel: tagged SwiGLU outputs
  size_t f_done;    // u64 [kMaxGrid * kDoneStride] single-token kernel: per-CTA "read the epoch" records
  size_t total;
};

WsLayout ws_layout(int H, int E, int K, int I, int T);

// Geometry of the fused single-token kernel (host-computed, passed by value).
// Each CTA keeps its whole share of the selected experts resident in shared
// memory: per expert a gate/up slot (np_max row pairs + four scale/bias
// segments) and a down slot (no_max output rows + two segments).
constexpr int kMaxGrid = 256;
// one done record per 32-byte sector: every CTA polls all of them, and
// records packed into a few lines would put all that polling on a few L2
// slices
constexpr int kDoneStride = 4;
struct FusedGeometry {
  int grid;
  int nq, nrg;       // column quarters of a gate/up row; row groups (nq * nrg <= 16 warps)
  int np_max;        // most gate/up row pairs of one expert in one CTA: ceil(I / grid)
  int no_max;        // most output rows one CTA owns: ceil(H / grid)
  int gu_row;        // bytes of a gate/up row slot (4-bit row: H / 2)
  int gu_sc;         // bytes of a gate/up scale or bias segment slot
  int gu_bytes;      // bytes of one expert's gate/up slot
  int d_row;         // bytes of a down row (4-bit: I / 2)
  int d_sc;          // bytes of a down scale or bias segment slot
  int d_bytes;       // bytes of one expert's down slot
  int nbar;          // mbarriers: K (gate/up rows) + K (down rows)
  int off_xn, off_cand, off_misc, off_bar, off_gred, off_ycomb, off_gu, off_down;
  int smem_bytes;
};

struct FusedParams {
  int H, E, K, I;
  float eps;
  const void* x;
  int x_bf16;
  int add_residual;
  const float* gamma;
  const float* router_w;
  const float* offset;
  const qe_expert* experts;
  float* out;
  int32_t* topk_idx;
  float* topk_w;
  WsControl* ctl;
  unsigned long long* rec_logit;  // [kMaxGrid][8][2] per CTA line: {low half | tag, high half | tag} of each fp64 logit
  unsigned long long* rec_h;      // [K*I] {h bits | tag}
  unsigned long long* rec_done;   // {0 | tag} at c * kDoneStride: CTA c has read the launch epoch
  // routing decided beforehand (device [K] each), or null: the kernel then
  // skips the router and the top-K
  const int32_t* given_idx;
  const float* given_w;
  FusedGeometry g;
  unsigned long long budget_ns;
  int skip_cta;
  unsigned long long* trace;  // [grid][16] phase timestamps, or null
};

// Launch wrappers (defined in the .cu files).  Return cudaError_t.
cudaError_t launch_fused_layer(const FusedParams& p, cudaStream_t s);
int fused_geometry(int H, int E, int K, int I, int sms, int smem_optin, FusedGeometry* g);

struct RouteParams {
  int H, E, K, T;
  float eps;
  const void* x;
  int x_bf16;
  const float* gamma;
  const float* router_w;
  const float* offset;
  float* xn_out;    // may be null
  int32_t* idx;
  float* w;
  double* rinv;
  double* xg;
  double* logits;
  float* xn_ws;     // normalised activations kept for the expert path (may be null)
  uint16_t* xh;     // xn as fp16 bits [T][H] for the tensor-core path (may be null)
  float* xp4;       // may be null
  float* xp2;
  float* xsum;
  int* xexp;
  int* err;
};
cudaError_t launch_route(const RouteParams& p, cudaStream_t s);

struct FfnParams {
  int H, K, I, T;
  int mode;  // 4, 2 or 0 (each expert's own bits)
  const qe_expert* experts;
  const int32_t* idx;
  const float* xn;   // [T,H] (prep kernel input)
  float* xp4;
  float* xp2;
  float* xsum;
  int* xexp;
  float* h;
  float* hp;
  float* hsum;
  int* hexp;
  unsigned* hamax;
  float* y;          // [T,K,H]
  int* err;
  int skip_xprep;    // x' already prepared by the route step
};
cudaError_t launch_ffn(const FfnParams& p, cudaStream_t s);

cudaError_t launch_combine(const float* y, const float* w, const void* residual, int res_bf16, int T, int K,
                           int H, float* out, cudaStream_t s);

struct GroupedParams {
  int H, E, K, I, T;
  const qe_expert* experts;
  const int32_t* idx;
  const float* w;
  const float* xp4;
  const float* xp2;
  const float* xsum;
  const int* xexp;
  float* h;
  float* hp;
  float* hsum;
  int* hexp;
  unsigned* hamax;
  float* y;
  int* grp_count;     // [E + 8]: counts, then the grouping control words
  int* grp_start;     // [E + 1]
  int* grp_list;      // [T*K]
  int* grp_order;     // [E]
  const uint16_t* xh; // [T][H] fp16 bits of xn (tensor-core gate/up)
  const void* x;     // residual source
  int x_bf16;
  int add_residual;
  float* out;
  int* err;
  unsigned long long budget_ns;  // bounded waits of the tensor-core kernel
};
cudaError_t launch_grouped(const GroupedParams& p, cudaStream_t s);
// Tensor-core gate/up for experts with at least tc_min_tokens() tokens.
bool tc_eligible(int H, int I);
int tc_min_tokens();
cudaError_t launch_tc_gateup(const GroupedParams& gp, int* ctl, unsigned long long budget_ns, cudaStream_t s);


// ---- shared host helpers (qe_abi.cu)
struct DevInfo {
  int sms = 0, optin = 0;
};
DevInfo dev_info();
// GatedDeltaNet decode step (qe_gdn.cu): one launch over all heads.
cudaError_t launch_gdn_step(long long n_heads, int dk, int dv, float* S, const float* q, const float* k,
                            const float* v, const float* alpha, const float* beta, float* o, int sms,
                            cudaStream_t s);

int fail(int code, const char* fmt, ...);
int cuda_fail(cudaError_t e, const char* what);
int check_cfg(const qe_cfg* c);
int check_ptr(const void* p, const char* name, bool may_be_null = false, unsigned align = 4);
int check_ws(const qe_cfg* c, int T, void* ws, size_t bytes);
qe_expert pool_descriptor(const qe_cfg* c, void* base, int bits);
int route_impl(const qe_cfg* c, const void* x, int x_dtype, const float* gamma, const float* router_w,
               const float* offset, int T, float* xn, int32_t* idx, float* w, void* ws, size_t ws_bytes,
               bool want_xprime, cudaStream_t s);
bool fused_aligned(const void* x, int x_dtype, const float* gamma);
bool fused_fits(const qe_cfg* c, const void* x, int x_dtype, const float* gamma);
int fused_step(const qe_cfg* c, const qe_layer* layer, const void* x, int x_dtype, float* out, int add_residual,
               int32_t* topk_idx, float* topk_w, void* ws, const int32_t* given_idx, const float* given_w,
               cudaStream_t s);
int experts_and_combine(const qe_cfg* c, const qe_expert* experts, const int32_t* idx, const float* w, const void* x,
                        int x_dtype, int T, float* out, int add_residual, void* ws, cudaStream_t s);

}  // namespace qe
