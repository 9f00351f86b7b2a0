/*
 * Plain CPU oracle of the MoE layer hot path: routing, dispatch layout,
 * permute, grouped SwiGLU experts, combine, and the backward of all of it.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the library path calls this file; the
 * tests, the smoke check and the benchmark's CPU-baseline leg do. It shares no
 * source, header, helper or constant with the CUDA library.
 *
 * What the pages fix and what is read into them
 * ---------------------------------------------
 * The pages name the steps of the layer, not their arithmetic:
 *   - "EP token dispatch, grouped expert compute" (leap-finetune PR #26 "Add
 *     MoE expert parallel training runtime", Summary / Major changes);
 *   - "grouped-GEMM" (ART issue #917 "Support combined expert and data
 *     parallelism in TrainerRank", Acceptance / Related);
 *   - expert-routing communication, expert communication groups, full
 *     source-order outputs, accumulation, uneven or empty work (ART issue
 *     #917, intro and Desired behavior).
 * Everything else takes the plainest reading: a dropless top-k softmax-gated
 * mixture of SwiGLU experts,
 *     Y_t = sum_{j<k} g_{t,j} * FFN_{S_{t,j}}(x_t),
 *     FFN_e(x) = (silu(x Wg_e^T) * (x Wu_e^T)) Wd_e^T,  silu(u) = u / (1 + e^-u),
 * with S_t the k largest router logits (ties to the lower expert index, slots
 * in descending order) and g_t the softmax over the k selected logits. The
 * backward is the exact gradient of that expression with S_t held fixed.
 *
 * Precision: every float result is computed in double from the exactly
 * up-converted inputs, with plain sequential sums. The one exception is the
 * router logit that decides the discrete top-k: it is computed in fp32 with
 * one fused multiply-add per input element in ascending element order, then
 * one fp32 add of the bias (orc_router_logits_f32), because a decision taken
 * from floats must be taken in the precision of the kernel that takes it.
 * orc_router_logits_f64 is the same definition in double (used by the
 * finite-difference checks).
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (no fast-math).
 * Parity status: every function below is pinned by a CPU test (brute force,
 * closed forms, invariants, finite differences); none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_FLAG_NONFINITE 1 /* a softmax over the selected logits was undefined */

/* ---------------------------------------------------------------- router */

/* Router logits, fp32, fixed order:
 *   acc = 0; for i = 0..d-1: acc = fmaf(x[t,i], Wr[e,i], acc); z[t,e] = acc + b[e].
 * The expert-routing step of ART issue #917 (intro). */
void orc_router_logits_f32(const float* x, const float* Wr, const float* b,
                           int64_t T, int d, int E, float* z) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      float acc = 0.0f;
      for (int i = 0; i < d; ++i)
        acc = fmaf(x[t * d + i], Wr[(int64_t)e * d + i], acc);
      z[t * E + e] = acc + b[e];
    }
  }
}

/* The same definition in double: z[t,e] = sum_i x[t,i] Wr[e,i] + b[e]. */
void orc_router_logits_f64(const double* x, const double* Wr, const double* b,
                           int64_t T, int d, int E, double* z) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += x[t * d + i] * Wr[(int64_t)e * d + i];
      z[t * E + e] = acc + b[e];
    }
  }
}

/* Ranking key: larger logit first; NaN after every number; equal keys go to
 * the lower expert index. Returns 1 when (za, ia) ranks before (zb, ib). */
static int ranks_before(double za, int ia, double zb, int ib) {
  int na = isnan(za), nb = isnan(zb);
  if (na != nb) return nb;
  if (!na && za != zb) return za > zb;
  return ia < ib;
}

/* Top-k selection and gate weights per token.
 * topk_idx[t,j] is the j-th ranked expert; topk_w[t,j] = softmax over the k
 * selected logits (equivalently, the softmax over all E renormalised to the
 * selected k), computed as exp(z_j - m) / sum_i exp(z_i - m) with m the
 * largest selected logit. A selected -inf next to a finite m is well defined
 * and gets exactly 0. The softmax is undefined only when m is not finite
 * (+inf gives inf - inf; m = -inf means every selected logit is -inf, 0/0)
 * or a selected logit is NaN (NaN ranks last, so then the k-th one is NaN):
 * only then are the weights 1/k each and the returned flag word has
 * ORC_FLAG_NONFINITE set.
 * Reads z in double (an fp32 logit converts exactly). */
int orc_route(const double* z, int64_t T, int E, int k, int32_t* topk_idx, double* topk_w) {
  int flags = 0;
#pragma omp parallel reduction(| : flags)
  {
    int* order = (int*)malloc(sizeof(int) * (size_t)(E > 0 ? E : 1));
#pragma omp for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
      const double* zt = z + t * E;
      /* insertion sort of the expert indices by the ranking key */
      for (int e = 0; e < E; ++e) {
        int p = e;
        while (p > 0 && ranks_before(zt[e], e, zt[order[p - 1]], order[p - 1])) {
          order[p] = order[p - 1];
          --p;
        }
        order[p] = e;
      }
      for (int j = 0; j < k; ++j) topk_idx[t * k + j] = order[j];
      const double m = zt[order[0]];
      if (!isfinite(m) || isnan(zt[order[k - 1]])) {
        flags |= ORC_FLAG_NONFINITE;
        for (int j = 0; j < k; ++j) topk_w[t * k + j] = 1.0 / k;
        continue;
      }
      double s = 0.0;
      for (int j = 0; j < k; ++j) s += exp(zt[order[j]] - m);
      for (int j = 0; j < k; ++j) topk_w[t * k + j] = exp(zt[order[j]] - m) / s;
    }
    free(order);
  }
  return flags;
}

/* Dispatch layout (the EP token dispatch of leap-finetune PR #26, Summary;
 * expert communication groups of ART issue #917, Desired behavior).
 *   counts[e]          number of (token, slot) pairs routed to e
 *   offsets[e]         exclusive prefix sum of counts, offsets[E] = T*k
 *   rows               pairs sorted by (expert, token), both ascending;
 *                      row_of_pair[t*k+j] is the row of pair (t,j) and
 *                      pair_of_row its inverse
 *   groups             expert e belongs to group e / (E/G) (contiguous blocks);
 *                      group_counts[g] = sum of its experts' counts,
 *                      group_offsets[g] = offsets[first expert of g]
 * Dropless: every pair gets a row. Returns -1 if E % G != 0, else 0. */
int orc_dispatch_layout(const int32_t* topk_idx, int64_t T, int E, int k, int G,
                        int32_t* counts, int64_t* offsets,
                        int32_t* group_counts, int64_t* group_offsets,
                        int32_t* row_of_pair, int32_t* pair_of_row) {
  if (G <= 0 || E % G != 0) return -1;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t p = 0; p < T * k; ++p) counts[topk_idx[p]] += 1;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int64_t* cursor = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
  for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
  /* visiting tokens in ascending order puts each expert's rows in token order */
  for (int64_t t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      int e = topk_idx[t * k + j];
      int64_t r = cursor[e]++;
      row_of_pair[t * k + j] = (int32_t)r;
      pair_of_row[r] = (int32_t)(t * k + j);
    }
  free(cursor);
  int per = E / G;
  for (int g = 0; g < G; ++g) {
    int64_t c = 0;
    for (int e = g * per; e < (g + 1) * per; ++e) c += counts[e];
    group_counts[g] = (int32_t)c;
    group_offsets[g] = offsets[g * per];
  }
  group_offsets[G] = offsets[E];
  return 0;
}

/* ------------------------------------------------------------- dispatch */

/* xp[r,:] = x[pair_of_row[r] / k, :]  (the token copy that dispatch sends) */
void orc_permute(const double* x, int64_t T, int d, int k, const int32_t* pair_of_row,
                 double* xp) {
  int64_t P = T * k;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < P; ++r) {
    int64_t t = pair_of_row[r] / k;
    memcpy(xp + r * d, x + t * d, sizeof(double) * (size_t)d);
  }
}

/* ------------------------------------------------------ expert compute */

static double silu(double u) { return u / (1.0 + exp(-u)); }
static double sigmoid(double u) { return 1.0 / (1.0 + exp(-u)); }
/* d/du silu(u) = s + u s (1 - s), s = sigmoid(u) */
static double silu_grad(double u) {
  double s = sigmoid(u);
  return s * (1.0 + u * (1.0 - s));
}

/* One expert's SwiGLU FFN on one row:
 *   h1 = Wg_e x, h2 = Wu_e x, a = silu(h1) * h2, y = Wd_e a.
 * Wg_e, Wu_e are [f, d]; Wd_e is [d, f]. */
static void ffn_row(const double* x, const double* Wg, const double* Wu, const double* Wd,
                    int d, int f, double* h1, double* h2, double* a, double* y) {
  for (int j = 0; j < f; ++j) {
    double s1 = 0.0, s2 = 0.0;
    for (int i = 0; i < d; ++i) {
      s1 += Wg[(int64_t)j * d + i] * x[i];
      s2 += Wu[(int64_t)j * d + i] * x[i];
    }
    h1[j] = s1;
    h2[j] = s2;
    a[j] = silu(s1) * s2;
  }
  for (int i = 0; i < d; ++i) {
    double s = 0.0;
    for (int j = 0; j < f; ++j) s += Wd[(int64_t)i * f + j] * a[j];
    y[i] = s;
  }
}

/* Grouped expert compute over the permuted rows: rows [offsets[e],
 * offsets[e+1]) go through expert e. An expert with no rows does nothing.
 * Wg, Wu: [E, f, d]; Wd: [E, d, f]; h1, h2, a: [P, f]; yp: [P, d]. */
void orc_expert_ffn_fwd(const double* xp, const double* Wg, const double* Wu, const double* Wd,
                        const int64_t* offsets, int E, int d, int f,
                        double* h1, double* h2, double* a, double* yp) {
  for (int e = 0; e < E; ++e) {
    const double* Wg_e = Wg + (int64_t)e * f * d;
    const double* Wu_e = Wu + (int64_t)e * f * d;
    const double* Wd_e = Wd + (int64_t)e * d * f;
#pragma omp parallel for schedule(static)
    for (int64_t r = offsets[e]; r < offsets[e + 1]; ++r)
      ffn_row(xp + r * d, Wg_e, Wu_e, Wd_e, d, f, h1 + r * f, h2 + r * f, a + r * f, yp + r * d);
  }
}

/* --------------------------------------------------------------- combine */

/* Y[t,:] = sum_{j<k} w[t,j] * yp[row_of_pair[t*k+j], :], j ascending.
 * Brings expert outputs back to source order (ART issue #917, Desired
 * behavior: full source-order outputs). */
void orc_combine(const double* yp, const double* w, const int32_t* row_of_pair,
                 int64_t T, int d, int k, double* Y) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t)
    for (int i = 0; i < d; ++i) {
      double s = 0.0;
      for (int j = 0; j < k; ++j) s += w[t * k + j] * yp[(int64_t)row_of_pair[t * k + j] * d + i];
      Y[t * d + i] = s;
    }
}

/* ------------------------------------------------------------- backward */

/* Combine backward: dyp[r] = w[t,j] dY[t];  dg[t,j] = <dY[t], yp[r]>. */
void orc_combine_bwd(const double* dY, const double* yp, const double* w,
                     const int32_t* row_of_pair, int64_t T, int d, int k,
                     double* dyp, double* dg) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      int64_t r = row_of_pair[t * k + j];
      double s = 0.0;
      for (int i = 0; i < d; ++i) {
        dyp[r * d + i] = w[t * k + j] * dY[t * d + i];
        s += dY[t * d + i] * yp[r * d + i];
      }
      dg[t * k + j] = s;
    }
}

/* Route backward through the softmax over the selected logits:
 *   dz[t, S_j] = g_j (dg_j - sum_m g_m dg_m), dz = 0 off the selection. */
void orc_route_bwd(const double* dg, const double* w, const int32_t* topk_idx,
                   int64_t T, int E, int k, double* dz) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    double s = 0.0;
    for (int j = 0; j < k; ++j) s += w[t * k + j] * dg[t * k + j];
    for (int e = 0; e < E; ++e) dz[t * E + e] = 0.0;
    for (int j = 0; j < k; ++j)
      dz[t * E + topk_idx[t * k + j]] = w[t * k + j] * (dg[t * k + j] - s);
  }
}

/* Grouped expert backward over the permuted rows, expert e on rows
 * [offsets[e], offsets[e+1]):
 *   da  = Wd_e^T dyp                     (dgrad of the down projection)
 *   dh1 = da * h2 * silu'(h1), dh2 = da * silu(h1)
 *   dxp = Wg_e^T dh1 + Wu_e^T dh2        (dgrad of gate / up)
 *   dWd_e += sum_r dyp_r a_r^T, dWg_e += sum_r dh1_r xp_r^T,
 *   dWu_e += sum_r dh2_r xp_r^T          (wgrad, accumulated)
 * An expert with no rows leaves its dW untouched. */
void orc_expert_ffn_bwd(const double* xp, const double* Wg, const double* Wu, const double* Wd,
                        const double* h1, const double* h2, const double* a, const double* dyp,
                        const int64_t* offsets, int E, int d, int f,
                        double* dxp, double* dWg, double* dWu, double* dWd) {
  int64_t P = offsets[E];
  double* dh1 = (double*)malloc(sizeof(double) * (size_t)(P > 0 ? P * f : 1));
  double* dh2 = (double*)malloc(sizeof(double) * (size_t)(P > 0 ? P * f : 1));
  for (int e = 0; e < E; ++e) {
    const double* Wg_e = Wg + (int64_t)e * f * d;
    const double* Wu_e = Wu + (int64_t)e * f * d;
    const double* Wd_e = Wd + (int64_t)e * d * f;
    int64_t r0 = offsets[e], r1 = offsets[e + 1];
#pragma omp parallel for schedule(static)
    for (int64_t r = r0; r < r1; ++r) {
      for (int j = 0; j < f; ++j) {
        double da = 0.0;
        for (int i = 0; i < d; ++i) da += Wd_e[(int64_t)i * f + j] * dyp[r * d + i];
        double u = h1[r * f + j];
        dh1[r * f + j] = da * h2[r * f + j] * silu_grad(u);
        dh2[r * f + j] = da * silu(u);
      }
      for (int i = 0; i < d; ++i) {
        double s = 0.0;
        for (int j = 0; j < f; ++j)
          s += Wg_e[(int64_t)j * d + i] * dh1[r * f + j] + Wu_e[(int64_t)j * d + i] * dh2[r * f + j];
        dxp[r * d + i] = s;
      }
    }
    if (r1 == r0) continue;
    double* dWg_e = dWg + (int64_t)e * f * d;
    double* dWu_e = dWu + (int64_t)e * f * d;
    double* dWd_e = dWd + (int64_t)e * d * f;
#pragma omp parallel for schedule(static)
    for (int j = 0; j < f; ++j)
      for (int i = 0; i < d; ++i) {
        double sg = 0.0, su = 0.0;
        for (int64_t r = r0; r < r1; ++r) {
          sg += dh1[r * f + j] * xp[r * d + i];
          su += dh2[r * f + j] * xp[r * d + i];
        }
        dWg_e[(int64_t)j * d + i] += sg;
        dWu_e[(int64_t)j * d + i] += su;
      }
#pragma omp parallel for schedule(static)
    for (int i = 0; i < d; ++i)
      for (int j = 0; j < f; ++j) {
        double s = 0.0;
        for (int64_t r = r0; r < r1; ++r) s += dyp[r * d + i] * a[r * f + j];
        dWd_e[(int64_t)i * f + j] += s;
      }
  }
  free(dh1);
  free(dh2);
}

/* Permute backward: dX[t] = sum_{j<k} dxp[row_of_pair[t*k+j]] (overwrites). */
void orc_permute_bwd(const double* dxp, const int32_t* row_of_pair, int64_t T, int d, int k,
                     double* dX) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t)
    for (int i = 0; i < d; ++i) {
      double s = 0.0;
      for (int j = 0; j < k; ++j) s += dxp[(int64_t)row_of_pair[t * k + j] * d + i];
      dX[t * d + i] = s;
    }
}

/* Router backward (z = x Wr^T + b):
 *   dX[t] += sum_e dz[t,e] Wr[e];  dWr[e] += sum_t dz[t,e] x[t];  db[e] += sum_t dz[t,e]. */
void orc_router_bwd(const double* x, const double* Wr, const double* dz,
                    int64_t T, int d, int E, double* dX, double* dWr, double* db) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t)
    for (int i = 0; i < d; ++i) {
      double s = 0.0;
      for (int e = 0; e < E; ++e) s += dz[t * E + e] * Wr[(int64_t)e * d + i];
      dX[t * d + i] += s;
    }
#pragma omp parallel for schedule(static)
  for (int e = 0; e < E; ++e) {
    for (int i = 0; i < d; ++i) {
      double s = 0.0;
      for (int64_t t = 0; t < T; ++t) s += dz[t * E + e] * x[t * d + i];
      dWr[(int64_t)e * d + i] += s;
    }
    double s = 0.0;
    for (int64_t t = 0; t < T; ++t) s += dz[t * E + e];
    db[e] += s;
  }
}

/* ----------------------------------------- auxiliary load-balancing loss */

/* Auxiliary load-balancing loss and routing metrics. The pages name MoE
 * losses and metrics without a formula (leap-finetune PR #26 "Add MoE expert
 * parallel training runtime", its MoE-loss tests); the plainest reading is the
 * Switch-Transformer balance loss:
 *   p[t,e] = softmax over all E experts of z[t,:]
 *   f_e    = counts[e] / (T k)          (fraction of routed pairs to e)
 *   P_e    = (1/T) sum_t p[t,e]         (importance)
 *   L      = alpha * E * sum_e f_e P_e
 *   H      = (1/T) sum_t (- sum_e p[t,e] ln p[t,e]),  0 ln 0 = 0
 *                                        (mean routing entropy)
 * f is a count, constant in z. Sums are sequential in t and e. */
static void orc_softmax_row(const double* z, int E, double* p) {
  double m = z[0];
  for (int e = 1; e < E; ++e)
    if (z[e] > m) m = z[e];
  double s = 0.0;
  for (int e = 0; e < E; ++e) {
    p[e] = exp(z[e] - m);
    s += p[e];
  }
  for (int e = 0; e < E; ++e) p[e] /= s;
}

void orc_aux_loss(const double* z, const int32_t* counts, int64_t T, int E, int k, double alpha,
                  double* importance, double* loss, double* entropy) {
  double* p = (double*)malloc(sizeof(double) * (size_t)E);
  double h = 0.0;
  for (int e = 0; e < E; ++e) importance[e] = 0.0;
  for (int64_t t = 0; t < T; ++t) {
    orc_softmax_row(z + t * E, E, p);
    for (int e = 0; e < E; ++e) {
      importance[e] += p[e];
      if (p[e] > 0.0) h -= p[e] * log(p[e]);
    }
  }
  double l = 0.0;
  for (int e = 0; e < E; ++e) {
    importance[e] = T > 0 ? importance[e] / (double)T : 0.0;
    const double fe = T > 0 ? (double)counts[e] / ((double)T * k) : 0.0;
    l += fe * importance[e];
  }
  *loss = alpha * E * l;
  *entropy = T > 0 ? h / (double)T : 0.0;
  free(p);
}

/* Gradient of the loss in z, f held constant (softmax Jacobian):
 *   dz[t,j] = dL * alpha * E / T * p[t,j] * (f_j - sum_e f_e p[t,e]). */
void orc_aux_loss_bwd(const double* z, const int32_t* counts, int64_t T, int E, int k,
                      double alpha, double dL, double* dz) {
#pragma omp parallel
  {
    double* p = (double*)malloc(sizeof(double) * (size_t)E);
#pragma omp for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
      orc_softmax_row(z + t * E, E, p);
      double s = 0.0;
      for (int e = 0; e < E; ++e) s += ((double)counts[e] / ((double)T * k)) * p[e];
      const double c = dL * alpha * E / (double)T;
      for (int j = 0; j < E; ++j)
        dz[t * E + j] = c * p[j] * ((double)counts[j] / ((double)T * k) - s);
    }
    free(p);
  }
}

/* ------------------------------------------- per-token brute force path */

/* The layer for a list of tokens, evaluated token by token with no
 * permutation (the brute-force form of the definition):
 *   Y_t = sum_j g_{t,j} FFN_{S_{t,j}}(x_t).
 * xs: [n, d] the tokens; idx, w: [n, k] their routing. Also returns the
 * per-slot expert outputs ys [n, k, d] (needed by the backward). */
void orc_tokens_fwd(const double* xs, const int32_t* idx, const double* w, int64_t n, int k,
                    const double* Wg, const double* Wu, const double* Wd, int d, int f,
                    double* Y, double* ys) {
#pragma omp parallel
  {
    double* h1 = (double*)malloc(sizeof(double) * (size_t)f);
    double* h2 = (double*)malloc(sizeof(double) * (size_t)f);
    double* a = (double*)malloc(sizeof(double) * (size_t)f);
#pragma omp for schedule(dynamic)
    for (int64_t t = 0; t < n; ++t) {
      for (int i = 0; i < d; ++i) Y[t * d + i] = 0.0;
      for (int j = 0; j < k; ++j) {
        int e = idx[t * k + j];
        double* y = ys + (t * k + j) * d;
        ffn_row(xs + t * d, Wg + (int64_t)e * f * d, Wu + (int64_t)e * f * d,
                Wd + (int64_t)e * d * f, d, f, h1, h2, a, y);
      }
      for (int i = 0; i < d; ++i) {
        double s = 0.0;
        for (int j = 0; j < k; ++j) s += w[t * k + j] * ys[(t * k + j) * d + i];
        Y[t * d + i] = s;
      }
    }
    free(h1);
    free(h2);
    free(a);
  }
}

/* Per-token backward for a list of tokens (brute force, no permutation):
 * given dY_t, returns dz_t [n, E] and the full input gradient
 *   dX_t = sum_j (Wg_e^T dh1 + Wu_e^T dh2)|_{e=S_j, dy=g_j dY_t} + sum_e dz_t[e] Wr[e].
 * ys are the per-slot expert outputs from orc_tokens_fwd. */
void orc_tokens_bwd(const double* xs, const double* dYs, const int32_t* idx, const double* w,
                    const double* ys, int64_t n, int k, int E,
                    const double* Wr, const double* Wg, const double* Wu, const double* Wd,
                    int d, int f, double* dz, double* dX) {
#pragma omp parallel
  {
    double* dg = (double*)malloc(sizeof(double) * (size_t)k);
#pragma omp for schedule(dynamic)
    for (int64_t t = 0; t < n; ++t) {
      const double* x = xs + t * d;
      const double* dY = dYs + t * d;
      for (int i = 0; i < d; ++i) dX[t * d + i] = 0.0;
      for (int j = 0; j < k; ++j) {
        double s = 0.0;
        for (int i = 0; i < d; ++i) s += dY[i] * ys[(t * k + j) * d + i];
        dg[j] = s;
      }
      double sg = 0.0;
      for (int j = 0; j < k; ++j) sg += w[t * k + j] * dg[j];
      for (int e = 0; e < E; ++e) dz[t * E + e] = 0.0;
      for (int j = 0; j < k; ++j) dz[t * E + idx[t * k + j]] = w[t * k + j] * (dg[j] - sg);
      for (int j = 0; j < k; ++j) {
        int e = idx[t * k + j];
        const double* Wg_e = Wg + (int64_t)e * f * d;
        const double* Wu_e = Wu + (int64_t)e * f * d;
        const double* Wd_e = Wd + (int64_t)e * d * f;
        double gj = w[t * k + j];
        for (int c = 0; c < f; ++c) {
          double h1 = 0.0, h2 = 0.0, da = 0.0;
          for (int i = 0; i < d; ++i) {
            h1 += Wg_e[(int64_t)c * d + i] * x[i];
            h2 += Wu_e[(int64_t)c * d + i] * x[i];
            da += Wd_e[(int64_t)i * f + c] * (gj * dY[i]);
          }
          double dh1 = da * h2 * silu_grad(h1);
          double dh2 = da * silu(h1);
          for (int i = 0; i < d; ++i)
            dX[t * d + i] += Wg_e[(int64_t)c * d + i] * dh1 + Wu_e[(int64_t)c * d + i] * dh2;
        }
      }
      for (int i = 0; i < d; ++i) {
        double s = 0.0;
        for (int e = 0; e < E; ++e) s += dz[t * E + e] * Wr[(int64_t)e * d + i];
        dX[t * d + i] += s;
      }
    }
    free(dg);
  }
}

/* Selected columns of one expert's weight gradients, summed over that
 * expert's rows (the wgrad of the grouped expert compute, restricted):
 * for each c in cols,
 *   dWg_e[c,:] = sum_r dh1_r[c] x_r,  dWu_e[c,:] = sum_r dh2_r[c] x_r,
 *   dWd_e[:,c] = sum_r dyp_r a_r[c],  dyp_r = g_r dY_r,
 * over the n rows given by their token activations xs [n,d], upstream
 * gradients dYs [n,d] and gate weights gs [n]. Rows are summed in the given
 * order. Wg_e, Wu_e [f,d]; Wd_e [d,f]. Outputs are [ncols, d]. */
void orc_wgrad_columns(const double* xs, const double* dYs, const double* gs, int64_t n,
                       const double* Wg_e, const double* Wu_e, const double* Wd_e, int d, int f,
                       const int32_t* cols, int ncols,
                       double* dWg_cols, double* dWu_cols, double* dWd_cols) {
#pragma omp parallel for schedule(dynamic)
  for (int q = 0; q < ncols; ++q) {
    int c = cols[q];
    double* og = dWg_cols + (int64_t)q * d;
    double* ou = dWu_cols + (int64_t)q * d;
    double* od = dWd_cols + (int64_t)q * d;
    for (int i = 0; i < d; ++i) og[i] = ou[i] = od[i] = 0.0;
    for (int64_t r = 0; r < n; ++r) {
      const double* x = xs + r * d;
      const double* dY = dYs + r * d;
      double h1 = 0.0, h2 = 0.0, da = 0.0;
      for (int i = 0; i < d; ++i) {
        h1 += Wg_e[(int64_t)c * d + i] * x[i];
        h2 += Wu_e[(int64_t)c * d + i] * x[i];
        da += Wd_e[(int64_t)i * f + c] * (gs[r] * dY[i]);
      }
      double a = silu(h1) * h2;
      double dh1 = da * h2 * silu_grad(h1);
      double dh2 = da * silu(h1);
      for (int i = 0; i < d; ++i) {
        og[i] += dh1 * x[i];
        ou[i] += dh2 * x[i];
        od[i] += gs[r] * dY[i] * a;
      }
    }
  }
}

int orc_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
