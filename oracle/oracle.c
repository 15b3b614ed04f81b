/*
 * oracle.c -- TEST INFRASTRUCTURE.  A plain, slow, fp64 CPU statement of the
 * MoE expert step of Flash-MoE decode, and of the GatedDeltaNet decode step
 * that precedes it in 45 of the model's 60 layers, used only to check the
 * CUDA library.
 * Only the tests, the smoke check and the CPU-baseline leg of the benchmark
 * may load it; the product path never does.  It shares no code, header,
 * table or helper with the CUDA library.
 *
 * Sources (the Flash-MoE web pages; no code is printed there):
 *  [ARCH]  lilting.ch, "Flash-MoE: running a 397B-parameter model on a 48 GB
 *          MacBook", section "Model architecture": 512 experts per layer, 4
 *          active per token.  Same fact in tomo3141592653.github.io summary
 *          "Running a 400B-parameter LLM on iPhone 17 Pro", section "What is
 *          MoE".
 *  [SSD]   lilting.ch, same article, section "Core technique: SSD expert
 *          streaming": about 6.75 MB per 4-bit expert, 4 x 6.75 = 27 MB per
 *          token and layer.
 *  [METAL] lilting.ch, same article, section "Metal Compute Shaders" (kernel
 *          table): 4-bit and 2-bit matrix-vector products, RMS normalisation
 *          in two passes (sum of squares, then apply), MoE combine as a
 *          weighted sum of expert outputs; and the FMA rewrite of the dequant,
 *          (nibble*scale + bias)*x  ->  fma(nibble, scale*x, bias*x).
 *  [QUANT] tomo3141592653.github.io summary, section "Hybrid quantisation":
 *          MLX 4-bit quantisation of the experts.
 *  [GDN]   lilting.ch, same article, section "GatedDeltaNet acceleration":
 *          per layer a recurrent update of 64 heads x 128x128 state
 *          matrices, done with the BLAS calls scal, gemv and ger; and the
 *          tomo3141592653.github.io summary, section "GatedDeltaNet": a fixed,
 *          O(1) state in place of a KV cache.
 *
 * Readings where the pages are silent (each is a convention of the problem
 * statement this library implements; the pins in tests/ hold them):
 *  - affine dequant w = q*scale + bias, q unsigned, scale/bias bf16 per group
 *    of 64 consecutive input columns of a row (6.75 MiB per expert at
 *    hidden 4096 / intermediate 1024 fixes group 64 with 16-bit scale and bias);
 *  - element j of a uint32 word sits at bits [bits*j, bits*j + bits), low bits
 *    first, words run along the input (column) axis, rows are row-major;
 *  - RMSNorm xn = x / sqrt(mean(x^2) + eps) * gamma;
 *  - routing: softmax over all E logits, keep the K largest (ties -> lower
 *    expert index), renormalise the K weights to sum to 1;
 *  - SwiGLU h = silu(g) * u with silu(g) = g / (1 + exp(-g));
 *  - out = sum_k w_k * y_k (+ x when the residual is requested).
 *
 * All arithmetic is double precision and every dot product is summed
 * sequentially in index order.  OpenMP splits independent rows only, which
 * does not change any result.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  const uint32_t* wq;     /* [rows, cols*bits/32] packed q words        */
  const uint16_t* scales; /* [rows, cols/64] bf16 bit patterns           */
  const uint16_t* biases; /* [rows, cols/64] bf16 bit patterns           */
  int32_t bits;           /* 4 or 2                                      */
} or_qmat;

#define OR_GROUP 64

/* bf16 bit pattern -> its exact value. */
double or_bf16(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* q of element (r, c): word c / (32/bits) of row r, field c % (32/bits),
 * low bits first [QUANT, METAL]. */
unsigned or_q(const uint32_t* wq, int cols, int bits, int r, int c) {
  int per_word = 32 / bits;
  int words_per_row = cols / per_word;
  uint32_t w = wq[(size_t)r * words_per_row + c / per_word];
  return (w >> (bits * (c % per_word))) & ((1u << bits) - 1u);
}

/* Dequantised weight (r, c) = q * scale + bias of its group [METAL]. */
double or_dequant(const or_qmat* m, int cols, int r, int c) {
  int groups_per_row = cols / OR_GROUP;
  size_t gi = (size_t)r * groups_per_row + c / OR_GROUP;
  return (double)or_q(m->wq, cols, m->bits, r, c) * or_bf16(m->scales[gi]) +
         or_bf16(m->biases[gi]);
}

/* y = deq(W) x, y_r = sum_c w_rc x_c summed in column order [METAL]. */
void or_qmatvec(const or_qmat* m, int rows, int cols, const double* x, double* y,
                int nthreads) {
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(static) num_threads(nthreads)
  for (int r = 0; r < rows; ++r) {
    double acc = 0.0;
    for (int c = 0; c < cols; ++c) acc += or_dequant(m, cols, r, c) * x[c];
    y[r] = acc;
  }
}

/* The pages' FMA form of the same product, element by element:
 * y_r = sum_c fma(q, scale*x_c, bias*x_c) [METAL, the FMA dequant rewrite]. */
void or_qmatvec_fma_form(const or_qmat* m, int rows, int cols, const double* x,
                         double* y) {
  int groups_per_row = cols / OR_GROUP;
  for (int r = 0; r < rows; ++r) {
    double acc = 0.0;
    for (int c = 0; c < cols; ++c) {
      size_t gi = (size_t)r * groups_per_row + c / OR_GROUP;
      double q = (double)or_q(m->wq, cols, m->bits, r, c);
      double sx = or_bf16(m->scales[gi]) * x[c];
      double bx = or_bf16(m->biases[gi]) * x[c];
      acc += fma(q, sx, bx);
    }
    y[r] = acc;
  }
}

/* RMSNorm in two passes [METAL]: pass 1 reduces sum x^2, pass 2 applies
 * xn_c = x_c / sqrt(sum/H + eps) * gamma_c (gamma NULL means 1). */
void or_rmsnorm(const double* x, const double* gamma, int H, double eps, double* xn) {
  double ss = 0.0;
  for (int c = 0; c < H; ++c) ss += x[c] * x[c];
  double inv = 1.0 / sqrt(ss / (double)H + eps);
  for (int c = 0; c < H; ++c) xn[c] = x[c] * inv * (gamma ? gamma[c] : 1.0);
}

/* Router logits l_e = sum_c W[e,c] xn_c (+ offset_e) [ARCH]. */
void or_router(const float* W, const double* xn, const float* offset, int E, int H,
               double* logits, int nthreads) {
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(static) num_threads(nthreads)
  for (int e = 0; e < E; ++e) {
    double acc = 0.0;
    for (int c = 0; c < H; ++c) acc += (double)W[(size_t)e * H + c] * xn[c];
    logits[e] = acc + (offset ? (double)offset[e] : 0.0);
  }
}

/* Full softmax over all E logits (used to check the renormalisation). */
void or_softmax(const double* logits, int E, double* p) {
  double mx = logits[0];
  for (int e = 1; e < E; ++e) if (logits[e] > mx) mx = logits[e];
  double s = 0.0;
  for (int e = 0; e < E; ++e) { p[e] = exp(logits[e] - mx); s += p[e]; }
  for (int e = 0; e < E; ++e) p[e] /= s;
}

/* Top-K of E [ARCH]: K rounds, each taking the largest logit not yet taken,
 * the lower index winning a tie.  Weights are the softmax restricted to the K
 * kept experts, w_k = exp(l_k - l_max) / sum_j exp(l_j - l_max). */
void or_topk(const double* logits, int E, int K, int32_t* idx, double* w) {
  char* taken = (char*)calloc((size_t)E, 1);
  for (int k = 0; k < K; ++k) {
    int best = -1;
    for (int e = 0; e < E; ++e) {
      if (taken[e]) continue;
      if (best < 0 || logits[e] > logits[best]) best = e;
    }
    taken[best] = 1;
    idx[k] = best;
  }
  free(taken);
  double lmax = logits[idx[0]];
  double s = 0.0;
  for (int k = 0; k < K; ++k) { w[k] = exp(logits[idx[k]] - lmax); s += w[k]; }
  for (int k = 0; k < K; ++k) w[k] /= s;
}

/* silu(g) = g / (1 + exp(-g)). */
double or_silu(double g) { return g / (1.0 + exp(-g)); }

/* h = silu(g) * u, elementwise. */
void or_swiglu(const double* g, const double* u, int n, double* h) {
  for (int i = 0; i < n; ++i) h[i] = or_silu(g[i]) * u[i];
}

/* One expert: g = Wg xn, u = Wu xn, h = silu(g) u, y = Wd h.
 * gate/up are [I, H], down is [H, I]. */
void or_expert_ffn(const or_qmat* gate, const or_qmat* up, const or_qmat* down, int H,
                   int I, const double* xn, double* y, double* h_out, int nthreads) {
  double* g = (double*)malloc(sizeof(double) * (size_t)I);
  double* u = (double*)malloc(sizeof(double) * (size_t)I);
  double* h = (double*)malloc(sizeof(double) * (size_t)I);
  or_qmatvec(gate, I, H, xn, g, nthreads);
  or_qmatvec(up, I, H, xn, u, nthreads);
  or_swiglu(g, u, I, h);
  or_qmatvec(down, H, I, h, y, nthreads);
  if (h_out) memcpy(h_out, h, sizeof(double) * (size_t)I);
  free(g); free(u); free(h);
}

/* out_r = sum_k w_k y_k[r] (k ascending), plus residual_r if given [METAL,
 * MoE combine as a weighted sum]. */
void or_combine(const double* y, const double* w, int K, int H, const double* residual,
                double* out) {
  for (int r = 0; r < H; ++r) {
    double acc = 0.0;
    for (int k = 0; k < K; ++k) acc += w[k] * y[(size_t)k * H + r];
    out[r] = acc + (residual ? residual[r] : 0.0);
  }
}

/* One decode step of the gated delta rule for n_heads independent heads
 * [GDN].  The pages name the recurrence and its three BLAS calls but print
 * no formula; the reading taken here is the gated delta rule
 *   S' = alpha S (I - beta k k^T) + beta v k^T,   o = S' q,
 * carried out as the BLAS sequence the pages name, in this order:
 *   scal  S <- alpha S
 *   gemv  u <- S k                    (what the decayed state recalls for k)
 *   ger   S <- S + beta (v - u) k^T   (write the correction at key k)
 *   gemv  o <- S q                    (read out with the query)
 * S is [n_heads][dv][dk] row-major (row i answers value component i), q and
 * k are [n_heads][dk], v and o are [n_heads][dv], alpha and beta one value per
 * head.  S is updated in place. */
void or_gdn_step(int n_heads, int dk, int dv, double* S, const double* q, const double* k,
                 const double* v, const double* alpha, const double* beta, double* o) {
  double* u = (double*)malloc(sizeof(double) * (size_t)(dv > 0 ? dv : 1));
  for (int h = 0; h < n_heads; ++h) {
    double* Sh = S + (size_t)h * dv * dk;
    const double* qh = q + (size_t)h * dk;
    const double* kh = k + (size_t)h * dk;
    const double* vh = v + (size_t)h * dv;
    for (size_t e = 0; e < (size_t)dv * dk; ++e) Sh[e] *= alpha[h];
    for (int i = 0; i < dv; ++i) {
      double acc = 0.0;
      for (int j = 0; j < dk; ++j) acc += Sh[(size_t)i * dk + j] * kh[j];
      u[i] = acc;
    }
    for (int i = 0; i < dv; ++i) {
      const double c = beta[h] * (vh[i] - u[i]);
      for (int j = 0; j < dk; ++j) Sh[(size_t)i * dk + j] += c * kh[j];
    }
    for (int i = 0; i < dv; ++i) {
      double acc = 0.0;
      for (int j = 0; j < dk; ++j) acc += Sh[(size_t)i * dk + j] * qh[j];
      o[(size_t)h * dv + i] = acc;
    }
  }
  free(u);
}
