/*
 * LatentMoE forward oracle -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * A plain, slow, double-precision CPU restatement of what the LatentMoE
 * feed-forward layer computes.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no
 * code, header, table or helper with the CUDA library; the two meet only
 * through the seeded inputs of the `synth` module.
 *
 * Sources (the K3 repository pages):
 *   [sec07]  notes/sections/sec-07.tex, chapter "SiTU-GLU 与 Stable LatentMoE":
 *            the SiTU-GLU formula and its property table, the five-step compute
 *            flow (latent compression, K3 eq.13 routing, routed experts, shared
 *            experts, merge), the routing notes, and the sparse-dispatch
 *            subsection.
 *   [diff]   compare view 584f7e9..main, kda/layers/latent_moe.py:
 *            SiTU.forward, LatentMoE._route, LatentMoE._routed_u,
 *            LatentMoE.forward.
 *   [tests]  same compare view, tests/integration/test_k3_arch.py:
 *            _dense_moe_forward, test_moe_router_activates_topk_only and
 *            test_moe_aux_loss_penalizes_collapse.
 *   [prior]  the lines the compare view removes from LatentMoE.forward: the
 *            earlier router, TopK on the raw logits with the weights a
 *            softmax over the k selected logits.
 *
 * Precision: every input arrives as float (bf16 inputs are the exact bf16
 * values widened to float); every product and sum is formed in double and
 * the outputs are double.  No blocking, fusion or reordering beyond the
 * formulas: each token is computed on its own, slots in order i = 0..k-1.
 *
 * Readings where the pages leave a step open:
 *   - TopK order: keys sorted descending, a tie goes to the lower expert index
 *     ([diff] uses torch.topk, which returns values sorted descending).
 *   - RMSNorm (its file is not on the pages): u * (1/sqrt(mean(u^2) + eps)) * w.
 *   - The clamp of the routing denominator at 1e-9 is kept ([diff] _route).
 *   - Routed and shared experts may have different hidden widths (F and G).
 *
 * Parity pins for every function are in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int64_t n_tokens;  /* N = B*T                                   */
  int32_t d;         /* model width                               */
  int32_t latent;    /* l = d/2                                   */
  int32_t n_routed;  /* R                                         */
  int32_t top_k;     /* k                                         */
  int32_t n_shared;  /* S                                         */
  int32_t ff_routed; /* F: routed expert hidden width             */
  int32_t ff_shared; /* G: shared expert hidden width             */
  double beta1;      /* SiTU gate soft cap (4)                    */
  double beta2;      /* SiTU up soft cap (25)                     */
  double rms_eps;    /* RMSNorm epsilon                           */
  int32_t router;    /* 0: K3 sigmoid routing; 1: softmax over the top-k logits ([prior]) */
} orc_dims;

/* Logistic function.  The two branches are the same function; the second
 * avoids overflow of exp(-v) for very negative v. */
static double orc_sigmoid(double v) {
  if (v >= 0.0) return 1.0 / (1.0 + exp(-v));
  double e = exp(v);
  return e / (1.0 + e);
}

/* nn.Linear without bias: y[o] = sum_i W[o, i] * v[i], W stored [out, in]. */
static void orc_linear(const float* W, int64_t out, int64_t in, const double* v, double* y) {
  for (int64_t o = 0; o < out; ++o) {
    const float* row = W + o * in;
    double acc = 0.0;
    for (int64_t i = 0; i < in; ++i) acc += (double)row[i] * v[i];
    y[o] = acc;
  }
}

/* SiTU-GLU expert ([sec07] SiTU formula; [diff] SiTU.forward):
 *   a = W_g v,  c = W_u v,
 *   gate = beta1 * tanh(a / beta1) * sigmoid(a)      (sigmoid of a, not a/beta1)
 *   up   = beta2 * tanh(c / beta2)
 *   out  = W_o (gate * up)
 * w_g, w_u: [ff, dim_in]; w_o: [dim_in, ff].  `hidden` (optional) receives
 * gate*up, the quantity whose magnitude the property table bounds by beta1*beta2. */
void orc_situ(int32_t dim_in, int32_t ff, double beta1, double beta2,
              const float* w_g, const float* w_u, const float* w_o,
              const double* v, double* out, double* hidden) {
  double* a = (double*)malloc(sizeof(double) * (size_t)ff);
  double* c = (double*)malloc(sizeof(double) * (size_t)ff);
  double* h = (double*)malloc(sizeof(double) * (size_t)ff);
  orc_linear(w_g, ff, dim_in, v, a);
  orc_linear(w_u, ff, dim_in, v, c);
  for (int32_t j = 0; j < ff; ++j) {
    double gate = beta1 * tanh(a[j] / beta1) * orc_sigmoid(a[j]);
    double up = beta2 * tanh(c[j] / beta2);
    h[j] = gate * up;
  }
  orc_linear(w_o, dim_in, ff, h, out);
  if (hidden) memcpy(hidden, h, sizeof(double) * (size_t)ff);
  free(a);
  free(c);
  free(h);
}

/* Router for one token ([sec07] compute flow step 2, K3 eq.13; [diff] _route):
 *   l = W_r x,  s = sigmoid(l),  T = TopK(s + b, k),
 *   p_i = s_i / max(sum_{j in T} s_j, 1e-9).
 * The bias b enters the selection only; p uses the raw scores s.
 * router == 1 is the earlier router ([prior]): T = TopK(l, k) on the raw
 * logits (no bias), p = softmax over the k selected logits,
 *   p_i = exp(l_i - l_max) / sum_{j in T} exp(l_j - l_max).
 * ids/probs: [k] in slot order (key descending, ties to the lower index).
 * keys (optional): [R] receives the selection keys (s + b, or l). */
static void orc_route_token(int32_t d, int32_t R, int32_t k, int32_t router, const float* x,
                            const float* w_r, const float* bias, int32_t* ids, double* probs,
                            double* keys_out, double* scores_out) {
  double* l = (double*)malloc(sizeof(double) * (size_t)R);
  double* s = (double*)malloc(sizeof(double) * (size_t)R);
  double* key = (double*)malloc(sizeof(double) * (size_t)R);
  char* taken = (char*)calloc((size_t)R, 1);
  double* xv = (double*)malloc(sizeof(double) * (size_t)d);
  for (int32_t i = 0; i < d; ++i) xv[i] = (double)x[i];
  orc_linear(w_r, R, d, xv, l);
  for (int32_t e = 0; e < R; ++e) {
    s[e] = orc_sigmoid(l[e]);
    key[e] = router == 1 ? l[e] : s[e] + (bias ? (double)bias[e] : 0.0);
  }
  /* k rounds of "largest remaining key"; strict '>' keeps the lower index on a tie. */
  for (int32_t slot = 0; slot < k; ++slot) {
    int32_t best = -1;
    for (int32_t e = 0; e < R; ++e) {
      if (taken[e]) continue;
      if (best < 0 || key[e] > key[best]) best = e;
    }
    taken[best] = 1;
    ids[slot] = best;
  }
  if (router == 1) {
    /* softmax over the selected logits; slot 0 holds the largest */
    const double lmax = l[ids[0]];
    double den = 0.0;
    for (int32_t slot = 0; slot < k; ++slot) den += exp(l[ids[slot]] - lmax);
    for (int32_t slot = 0; slot < k; ++slot) probs[slot] = exp(l[ids[slot]] - lmax) / den;
  } else {
    double den = 0.0;
    for (int32_t slot = 0; slot < k; ++slot) den += s[ids[slot]];
    if (den < 1e-9) den = 1e-9;
    for (int32_t slot = 0; slot < k; ++slot) probs[slot] = s[ids[slot]] / den;
  }
  if (keys_out) memcpy(keys_out, key, sizeof(double) * (size_t)R);
  if (scores_out) memcpy(scores_out, s, sizeof(double) * (size_t)R);
  free(l);
  free(s);
  free(key);
  free(taken);
  free(xv);
}

/* Routing for all N tokens.  keys (optional): [N, R] = s + b.  scores
 * (optional): [N, R] = s. */
void orc_route(const orc_dims* dm, const float* x, const float* w_r, const float* bias,
               int32_t* ids, double* probs, double* keys, double* scores) {
  const int64_t N = dm->n_tokens;
  const int32_t d = dm->d, R = dm->n_routed, k = dm->top_k;
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t t = 0; t < N; ++t) {
    orc_route_token(d, R, k, dm->router, x + t * d, w_r, bias, ids + t * k, probs + t * k,
                    keys ? keys + t * R : NULL, scores ? scores + t * R : NULL);
  }
}

/* Token-expert pair permutation ([diff] _routed_u; [sec07] sparse dispatch,
 * step 1): the N*k pairs (t, ids[t, i]) are flattened token-major and sorted
 * by expert id with a stable sort, so that the pairs of one expert are
 * contiguous and, inside an expert, in ascending token order.
 *   counts[e]   = number of pairs with expert e          (bincount)
 *   offsets[e]  = sum_{e' < e} counts[e'], offsets[R] = N*k (cumsum - counts)
 *   perm_token[r] = token of the r-th pair in sorted order
 *   inv_pair[t*k + i] = sorted position r of the pair (t, ids[t, i])
 * Written as the textbook counting sort, which is a stable sort. */
void orc_permute(int64_t N, int32_t k, int32_t R, const int32_t* ids, int32_t* counts,
                 int32_t* offsets, int32_t* perm_token, int32_t* inv_pair) {
  for (int32_t e = 0; e < R; ++e) counts[e] = 0;
  for (int64_t p = 0; p < N * k; ++p) counts[ids[p]] += 1;
  offsets[0] = 0;
  for (int32_t e = 0; e < R; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)R);
  for (int32_t e = 0; e < R; ++e) cursor[e] = offsets[e];
  for (int64_t p = 0; p < N * k; ++p) { /* token-major order: p = t*k + i */
    int32_t e = ids[p];
    int32_t r = cursor[e]++;
    perm_token[r] = (int32_t)(p / k);
    inv_pair[p] = r;
  }
  free(cursor);
}

/* RMSNorm over one vector: out = u * (1/sqrt(mean(u^2) + eps)) * w. */
static void orc_rmsnorm(int32_t n, const double* u, const float* w, double eps, double* out) {
  double ms = 0.0;
  for (int32_t j = 0; j < n; ++j) ms += u[j] * u[j];
  ms /= (double)n;
  double inv = 1.0 / sqrt(ms + eps);
  for (int32_t j = 0; j < n; ++j) out[j] = u[j] * inv * (double)w[j];
}

/* Weights in the pages' nn.Linear layout ([out, in], K contiguous). */
typedef struct {
  const float* w_down;     /* [l, d]      W_down: d -> l                    */
  const float* w_router;   /* [R, d]      W_r                               */
  const float* w_up;       /* [d, l]      W_up: l -> d                      */
  const float* rms_weight; /* [l]                                           */
  const float* expert_bias;/* [R] or NULL (= 0)                             */
  const float* w_g;        /* [R, F, l]   routed gate projections           */
  const float* w_u;        /* [R, F, l]   routed up projections             */
  const float* w_o;        /* [R, l, F]   routed output projections         */
  const float* ws_g;       /* [S, G, d]   shared gate projections           */
  const float* ws_u;       /* [S, G, d]   shared up projections             */
  const float* ws_o;       /* [S, d, G]   shared output projections         */
} orc_weights;

/* Per-token forward ([sec07] compute flow, five steps; [diff] LatentMoE.forward):
 *   1. z = W_down x
 *   2. routing (K3 eq.13), see orc_route_token
 *   3. u = sum_{i in T} p_i * E_i(z)           (routed SiTU experts in l)
 *   4. s_sh = sum_j E^sh_j(x)                  (shared SiTU experts in d)
 *   5. y = s_sh + W_up RMSNorm(u)
 * Optional outputs (NULL to skip): z [N,l], u [N,l], uhat [N,l], shared [N,d],
 * routed_out [N,k,l] (E_{ids[t,i]}(z_t) before weighting). */
static void orc_forward_token(const orc_dims* dm, const orc_weights* w, const float* x_t,
                              double* y_t, int32_t* ids_t, double* probs_t, double* z_t_out,
                              double* u_t_out, double* uhat_t_out, double* sh_t_out,
                              double* routed_t_out) {
  const int32_t d = dm->d, L = dm->latent, R = dm->n_routed, k = dm->top_k;
  const int32_t F = dm->ff_routed, S = dm->n_shared, G = dm->ff_shared;
  double* xv = (double*)malloc(sizeof(double) * (size_t)d);
  double* z = (double*)malloc(sizeof(double) * (size_t)L);
  double* u = (double*)calloc((size_t)L, sizeof(double));
  double* e_out = (double*)malloc(sizeof(double) * (size_t)L);
  double* uhat = (double*)malloc(sizeof(double) * (size_t)L);
  double* sh = (double*)calloc((size_t)d, sizeof(double));
  double* sh_j = (double*)malloc(sizeof(double) * (size_t)d);
  double* up = (double*)malloc(sizeof(double) * (size_t)d);

  for (int32_t i = 0; i < d; ++i) xv[i] = (double)x_t[i];
  /* step 1: latent compression */
  orc_linear(w->w_down, L, d, xv, z);
  /* step 2: routing on the full-width x (not z) */
  orc_route_token(d, R, k, dm->router, x_t, w->w_router, w->expert_bias, ids_t, probs_t, NULL,
                  NULL);
  /* step 3: routed experts, slots in order */
  for (int32_t slot = 0; slot < k; ++slot) {
    const int64_t e = ids_t[slot];
    orc_situ(L, F, dm->beta1, dm->beta2, w->w_g + e * F * L, w->w_u + e * F * L,
             w->w_o + e * L * F, z, e_out, NULL);
    for (int32_t j = 0; j < L; ++j) u[j] += probs_t[slot] * e_out[j];
    if (routed_t_out) memcpy(routed_t_out + (int64_t)slot * L, e_out, sizeof(double) * (size_t)L);
  }
  /* step 4: shared experts on x */
  for (int32_t j = 0; j < S; ++j) {
    orc_situ(d, G, dm->beta1, dm->beta2, w->ws_g + (int64_t)j * G * d,
             w->ws_u + (int64_t)j * G * d, w->ws_o + (int64_t)j * d * G, xv, sh_j, NULL);
    for (int32_t i = 0; i < d; ++i) sh[i] += sh_j[i];
  }
  /* step 5: merge */
  orc_rmsnorm(L, u, w->rms_weight, dm->rms_eps, uhat);
  orc_linear(w->w_up, d, L, uhat, up);
  for (int32_t i = 0; i < d; ++i) y_t[i] = sh[i] + up[i];

  if (z_t_out) memcpy(z_t_out, z, sizeof(double) * (size_t)L);
  if (u_t_out) memcpy(u_t_out, u, sizeof(double) * (size_t)L);
  if (uhat_t_out) memcpy(uhat_t_out, uhat, sizeof(double) * (size_t)L);
  if (sh_t_out) memcpy(sh_t_out, sh, sizeof(double) * (size_t)d);
  free(xv);
  free(z);
  free(u);
  free(e_out);
  free(uhat);
  free(sh);
  free(sh_j);
  free(up);
}

void orc_forward(const orc_dims* dm, const orc_weights* w, const float* x, double* y,
                 int32_t* ids, double* probs, double* z_out, double* u_out, double* uhat_out,
                 double* shared_out, double* routed_out) {
  const int64_t N = dm->n_tokens;
  const int32_t d = dm->d, L = dm->latent, k = dm->top_k;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t t = 0; t < N; ++t) {
    orc_forward_token(dm, w, x + t * d, y + t * d, ids + t * k, probs + t * k,
                      z_out ? z_out + t * L : NULL, u_out ? u_out + t * L : NULL,
                      uhat_out ? uhat_out + t * L : NULL, shared_out ? shared_out + t * d : NULL,
                      routed_out ? routed_out + t * (int64_t)k * L : NULL);
  }
}

/* Dense evaluation ([tests] _dense_moe_forward; the removed forward in
 * [diff]): every routed expert runs on every token, all_out[t, e] = E_e(z_t),
 * then u_t = sum_i p_i * all_out[t, ids[t, i]].  The pages test that it
 * equals the sparse dispatch.  ids/probs come from the same router. */
void orc_forward_dense(const orc_dims* dm, const orc_weights* w, const float* x, double* y,
                       double* u_out) {
  const int64_t N = dm->n_tokens;
  const int32_t d = dm->d, L = dm->latent, R = dm->n_routed, k = dm->top_k;
  const int32_t F = dm->ff_routed, S = dm->n_shared, G = dm->ff_shared;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t t = 0; t < N; ++t) {
    const float* x_t = x + t * d;
    double* xv = (double*)malloc(sizeof(double) * (size_t)d);
    double* z = (double*)malloc(sizeof(double) * (size_t)L);
    double* all_out = (double*)malloc(sizeof(double) * (size_t)R * (size_t)L);
    double* u = (double*)calloc((size_t)L, sizeof(double));
    double* uhat = (double*)malloc(sizeof(double) * (size_t)L);
    double* sh = (double*)calloc((size_t)d, sizeof(double));
    double* tmp = (double*)malloc(sizeof(double) * (size_t)d);
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    double* probs = (double*)malloc(sizeof(double) * (size_t)k);
    for (int32_t i = 0; i < d; ++i) xv[i] = (double)x_t[i];
    orc_linear(w->w_down, L, d, xv, z);
    orc_route_token(d, R, k, dm->router, x_t, w->w_router, w->expert_bias, ids, probs, NULL,
                    NULL);
    for (int32_t e = 0; e < R; ++e)
      orc_situ(L, F, dm->beta1, dm->beta2, w->w_g + (int64_t)e * F * L,
               w->w_u + (int64_t)e * F * L, w->w_o + (int64_t)e * L * F, z,
               all_out + (int64_t)e * L, NULL);
    for (int32_t slot = 0; slot < k; ++slot)
      for (int32_t j = 0; j < L; ++j) u[j] += probs[slot] * all_out[(int64_t)ids[slot] * L + j];
    for (int32_t j = 0; j < S; ++j) {
      orc_situ(d, G, dm->beta1, dm->beta2, w->ws_g + (int64_t)j * G * d,
               w->ws_u + (int64_t)j * G * d, w->ws_o + (int64_t)j * d * G, xv, tmp, NULL);
      for (int32_t i = 0; i < d; ++i) sh[i] += tmp[i];
    }
    orc_rmsnorm(L, u, w->rms_weight, dm->rms_eps, uhat);
    orc_linear(w->w_up, d, L, uhat, tmp);
    for (int32_t i = 0; i < d; ++i) y[t * d + i] = sh[i] + tmp[i];
    if (u_out) memcpy(u_out + t * L, u, sizeof(double) * (size_t)L);
    free(xv);
    free(z);
    free(all_out);
    free(u);
    free(uhat);
    free(sh);
    free(tmp);
    free(ids);
    free(probs);
  }
}

/* Standalone RMSNorm over N rows of width n (for pins). */
void orc_rmsnorm_rows(int64_t N, int32_t n, const double* u, const float* w, double eps,
                      double* out) {
  for (int64_t t = 0; t < N; ++t) orc_rmsnorm(n, u + t * n, w, eps, out + t * n);
}

/* Router balancing losses ([diff] LatentMoE._balancing_losses; [tests]
 * test_moe_aux_loss_penalizes_collapse), before their coefficients:
 *   counts_e    = number of pairs routed to expert e        (bincount of ids)
 *   frac_e      = counts_e / max(sum_e counts_e, 1)
 *   prob_mean_e = mean over tokens of sigmoid(l_te)         (l = W_r x)
 *   aux         = R * sum_e frac_e * prob_mean_e            (Switch/GShard form on sigmoid scores)
 *   z           = mean over tokens of logsumexp_e(l_te)^2   (z-loss on the raw logits)
 * out: [2 + 2R] = aux, z, frac[R], prob_mean[R].  logsumexp is formed as
 * m + log(sum exp(l - m)) with m the row maximum. */
void orc_router_losses(const orc_dims* dm, const float* x, const float* w_r, const int32_t* ids,
                       double* out) {
  const int64_t N = dm->n_tokens;
  const int32_t d = dm->d, R = dm->n_routed, k = dm->top_k;
  double* frac = out + 2;
  double* pmean = out + 2 + R;
  double* l = (double*)malloc(sizeof(double) * (size_t)R);
  double* xv = (double*)malloc(sizeof(double) * (size_t)d);
  double z = 0.0, total = 0.0;
  for (int32_t e = 0; e < R; ++e) frac[e] = pmean[e] = 0.0;
  for (int64_t i = 0; i < N * k; ++i) frac[ids[i]] += 1.0;
  for (int32_t e = 0; e < R; ++e) total += frac[e];
  if (total < 1.0) total = 1.0;
  for (int32_t e = 0; e < R; ++e) frac[e] /= total;
  for (int64_t t = 0; t < N; ++t) {
    for (int32_t i = 0; i < d; ++i) xv[i] = (double)x[t * d + i];
    orc_linear(w_r, R, d, xv, l);
    double m = l[0], se = 0.0;
    for (int32_t e = 1; e < R; ++e) m = l[e] > m ? l[e] : m;
    for (int32_t e = 0; e < R; ++e) {
      se += exp(l[e] - m);
      pmean[e] += orc_sigmoid(l[e]);
    }
    const double lse = m + log(se);
    z += lse * lse;
  }
  double aux = 0.0;
  for (int32_t e = 0; e < R; ++e) {
    pmean[e] = N > 0 ? pmean[e] / (double)N : 0.0;
    aux += frac[e] * pmean[e];
  }
  out[0] = (double)R * aux;
  out[1] = N > 0 ? z / (double)N : 0.0;
  free(l);
  free(xv);
}

/* ------------------------------------------------------------------ backward
 * Gradients of the layer for an upstream gradient dy [N, d] (the pages' tests
 * train the layer: test_moe_unselected_experts_have_zero_grad and the sparse
 * == dense gradient checks of [tests]), by the chain rule through the five
 * steps of the forward, token by token, in double:
 *   y = s_sh + W_up uhat          dW_up += dy uhat^T,  duhat = W_up^T dy
 *   uhat = u r w, r = (mean u^2 + eps)^(-1/2)
 *                                 dw += duhat u r,  du = r w duhat - u r^3/l sum_j w_j duhat_j u_j
 *   u = sum_i p_i E_i(z)          dp_i = <du, E_i(z)>,  dE_i = p_i du
 *   E(v) = W_o h, h = g(a) up(c), a = W_g v, c = W_u v
 *     g(a) = b1 tanh(a/b1) sigmoid(a),   g'(a) = sech^2(a/b1) sigmoid(a) + g(a) (1 - sigmoid(a))
 *     up(c) = b2 tanh(c/b2),             up'(c) = sech^2(c/b2)
 *                                 dW_o += dE h^T, dh = W_o^T dE, da = dh up g', dc = dh g up',
 *                                 dW_g += da v^T, dW_u += dc v^T, dv += W_g^T da + W_u^T dc
 *   routing (ids fixed: they are not differentiable; b enters no gradient):
 *     K3: p_i = s_i / S, S = sum_T s (clamped at 1e-9), s = sigmoid(l):
 *         ds_i = (dp_i - sum_j p_j dp_j) / S   (dp_i / 1e-9 when clamped),
 *         dl_i = ds_i s_i (1 - s_i)
 *     softmax over the top-k logits: dl_i = p_i (dp_i - sum_j p_j dp_j)
 *                                 dW_r[e_i] += dl_i x,  dx += dl_i W_r[e_i]
 *   z = W_down x                  dW_down += dz x^T,  dx += W_down^T dz
 *   s_sh = sum_j E^sh_j(x)        E^sh backward with dE = dy and v = x
 * Every output is overwritten.  Weight gradients of experts no token selected
 * stay exactly 0. */
static void orc_situ_backward(int32_t dim_in, int32_t ff, double beta1, double beta2,
                              const float* w_g, const float* w_u, const float* w_o,
                              const double* v, const double* dout, double* dv, double* dw_g,
                              double* dw_u, double* dw_o, double* out) {
  double* a = (double*)malloc(sizeof(double) * (size_t)ff);
  double* c = (double*)malloc(sizeof(double) * (size_t)ff);
  double* h = (double*)malloc(sizeof(double) * (size_t)ff);
  double* dh = (double*)calloc((size_t)ff, sizeof(double));
  orc_linear(w_g, ff, dim_in, v, a);
  orc_linear(w_u, ff, dim_in, v, c);
  for (int32_t f = 0; f < ff; ++f) {
    const double tg = tanh(a[f] / beta1), sg = orc_sigmoid(a[f]), tu = tanh(c[f] / beta2);
    h[f] = beta1 * tg * sg * beta2 * tu;
  }
  if (out) orc_linear(w_o, dim_in, ff, h, out);
  for (int32_t i = 0; i < dim_in; ++i) {
    const float* row = w_o + (int64_t)i * ff;
    for (int32_t f = 0; f < ff; ++f) {
      dh[f] += (double)row[f] * dout[i];
      dw_o[(int64_t)i * ff + f] += dout[i] * h[f];
    }
  }
  for (int32_t f = 0; f < ff; ++f) {
    const double tg = tanh(a[f] / beta1), sg = orc_sigmoid(a[f]), tu = tanh(c[f] / beta2);
    const double g = beta1 * tg * sg, up = beta2 * tu;
    const double dg = (1.0 - tg * tg) * sg + g * (1.0 - sg);
    const double du = 1.0 - tu * tu;
    const double da = dh[f] * up * dg, dc = dh[f] * g * du;
    const float* rg = w_g + (int64_t)f * dim_in;
    const float* ru = w_u + (int64_t)f * dim_in;
    double* gg = dw_g + (int64_t)f * dim_in;
    double* gu = dw_u + (int64_t)f * dim_in;
    for (int32_t j = 0; j < dim_in; ++j) {
      gg[j] += da * v[j];
      gu[j] += dc * v[j];
      dv[j] += (double)rg[j] * da + (double)ru[j] * dc;
    }
  }
  free(a);
  free(c);
  free(h);
  free(dh);
}

void orc_backward(const orc_dims* dm, const orc_weights* w, const float* x, const float* dy,
                  double* dx, double* dw_down, double* dw_router, double* dw_up, double* drms,
                  double* dw_g, double* dw_u, double* dw_o, double* dws_g, double* dws_u,
                  double* dws_o) {
  const int64_t N = dm->n_tokens;
  const int32_t d = dm->d, L = dm->latent, R = dm->n_routed, k = dm->top_k;
  const int32_t F = dm->ff_routed, S = dm->n_shared, G = dm->ff_shared;
  memset(dx, 0, sizeof(double) * (size_t)(N * d));
  memset(dw_down, 0, sizeof(double) * (size_t)L * d);
  memset(dw_router, 0, sizeof(double) * (size_t)R * d);
  memset(dw_up, 0, sizeof(double) * (size_t)d * L);
  memset(drms, 0, sizeof(double) * (size_t)L);
  memset(dw_g, 0, sizeof(double) * (size_t)R * F * L);
  memset(dw_u, 0, sizeof(double) * (size_t)R * F * L);
  memset(dw_o, 0, sizeof(double) * (size_t)R * L * F);
  if (S > 0) {
    memset(dws_g, 0, sizeof(double) * (size_t)S * G * d);
    memset(dws_u, 0, sizeof(double) * (size_t)S * G * d);
    memset(dws_o, 0, sizeof(double) * (size_t)S * d * G);
  }
  double* xv = (double*)malloc(sizeof(double) * (size_t)d);
  double* dyv = (double*)malloc(sizeof(double) * (size_t)d);
  double* z = (double*)malloc(sizeof(double) * (size_t)L);
  double* dz = (double*)malloc(sizeof(double) * (size_t)L);
  double* eo = (double*)malloc(sizeof(double) * (size_t)k * L);
  double* u = (double*)malloc(sizeof(double) * (size_t)L);
  double* uhat = (double*)malloc(sizeof(double) * (size_t)L);
  double* duhat = (double*)malloc(sizeof(double) * (size_t)L);
  double* du = (double*)malloc(sizeof(double) * (size_t)L);
  double* dE = (double*)malloc(sizeof(double) * (size_t)L);
  double* l = (double*)malloc(sizeof(double) * (size_t)R);
  double* dp = (double*)malloc(sizeof(double) * (size_t)k);
  double* probs = (double*)malloc(sizeof(double) * (size_t)k);
  int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
  for (int64_t t = 0; t < N; ++t) {
    const float* x_t = x + t * d;
    double* dx_t = dx + t * d;
    for (int32_t i = 0; i < d; ++i) {
      xv[i] = (double)x_t[i];
      dyv[i] = (double)dy[t * d + i];
    }
    /* forward of this token */
    orc_linear(w->w_down, L, d, xv, z);
    orc_linear(w->w_router, R, d, xv, l);
    orc_route_token(d, R, k, dm->router, x_t, w->w_router, w->expert_bias, ids, probs, NULL,
                    NULL);
    for (int32_t j = 0; j < L; ++j) u[j] = 0.0;
    for (int32_t slot = 0; slot < k; ++slot) {
      const int64_t e = ids[slot];
      orc_situ(L, F, dm->beta1, dm->beta2, w->w_g + e * F * L, w->w_u + e * F * L,
               w->w_o + e * L * F, z, eo + (int64_t)slot * L, NULL);
      for (int32_t j = 0; j < L; ++j) u[j] += probs[slot] * eo[(int64_t)slot * L + j];
    }
    double ms = 0.0;
    for (int32_t j = 0; j < L; ++j) ms += u[j] * u[j];
    const double r = 1.0 / sqrt(ms / (double)L + dm->rms_eps);
    for (int32_t j = 0; j < L; ++j) uhat[j] = u[j] * r * (double)w->rms_weight[j];
    /* step 5: y = s_sh + W_up uhat */
    for (int32_t j = 0; j < L; ++j) duhat[j] = 0.0;
    for (int32_t i = 0; i < d; ++i) {
      const float* row = w->w_up + (int64_t)i * L;
      for (int32_t j = 0; j < L; ++j) {
        dw_up[(int64_t)i * L + j] += dyv[i] * uhat[j];
        duhat[j] += (double)row[j] * dyv[i];
      }
    }
    /* RMSNorm */
    double wdu = 0.0;
    for (int32_t j = 0; j < L; ++j) {
      drms[j] += duhat[j] * u[j] * r;
      wdu += (double)w->rms_weight[j] * duhat[j] * u[j];
    }
    for (int32_t j = 0; j < L; ++j)
      du[j] = r * (double)w->rms_weight[j] * duhat[j] - u[j] * r * r * r / (double)L * wdu;
    /* routed experts and their weights p */
    for (int32_t j = 0; j < L; ++j) dz[j] = 0.0;
    for (int32_t slot = 0; slot < k; ++slot) {
      const int64_t e = ids[slot];
      double acc = 0.0;
      for (int32_t j = 0; j < L; ++j) {
        acc += du[j] * eo[(int64_t)slot * L + j];
        dE[j] = probs[slot] * du[j];
      }
      dp[slot] = acc;
      orc_situ_backward(L, F, dm->beta1, dm->beta2, w->w_g + e * F * L, w->w_u + e * F * L,
                        w->w_o + e * L * F, z, dE, dz, dw_g + e * F * L, dw_u + e * F * L,
                        dw_o + e * L * F, NULL);
    }
    /* router, through p only */
    double pdp = 0.0, ssum = 0.0;
    for (int32_t slot = 0; slot < k; ++slot) {
      pdp += probs[slot] * dp[slot];
      ssum += orc_sigmoid(l[ids[slot]]);
    }
    for (int32_t slot = 0; slot < k; ++slot) {
      const int32_t e = ids[slot];
      double dl;
      if (dm->router == 1) {
        dl = probs[slot] * (dp[slot] - pdp);
      } else {
        const double s = orc_sigmoid(l[e]);
        const double ds = ssum >= 1e-9 ? (dp[slot] - pdp) / ssum : dp[slot] / 1e-9;
        dl = ds * s * (1.0 - s);
      }
      const float* row = w->w_router + (int64_t)e * d;
      double* grow = dw_router + (int64_t)e * d;
      for (int32_t i = 0; i < d; ++i) {
        grow[i] += dl * xv[i];
        dx_t[i] += dl * (double)row[i];
      }
    }
    /* step 1: z = W_down x */
    for (int32_t j = 0; j < L; ++j) {
      const float* row = w->w_down + (int64_t)j * d;
      double* grow = dw_down + (int64_t)j * d;
      for (int32_t i = 0; i < d; ++i) {
        grow[i] += dz[j] * xv[i];
        dx_t[i] += (double)row[i] * dz[j];
      }
    }
    /* step 4: shared experts, dE = dy */
    for (int32_t j = 0; j < S; ++j)
      orc_situ_backward(d, G, dm->beta1, dm->beta2, w->ws_g + (int64_t)j * G * d,
                        w->ws_u + (int64_t)j * G * d, w->ws_o + (int64_t)j * d * G, xv, dyv,
                        dx_t, dws_g + (int64_t)j * G * d, dws_u + (int64_t)j * G * d,
                        dws_o + (int64_t)j * d * G, NULL);
  }
  free(xv);
  free(dyv);
  free(z);
  free(dz);
  free(eo);
  free(u);
  free(uhat);
  free(duhat);
  free(du);
  free(dE);
  free(l);
  free(dp);
  free(probs);
  free(ids);
}
