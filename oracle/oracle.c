/*
 * oracle.c -- plain CPU reference of the inference MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check of the graft
 * entry point and the CPU-baseline leg of bench.py may load this library.  The
 * product (the CUDA library and its Python binding) never calls it, and this
 * file shares no code, header or table with the product.
 *
 * What it computes is the plain definition of each step, written out in the
 * order the pages give it, with dot products accumulated in double (bf16 x bf16
 * and bf16 x fp32 products are exact in double) and rounded once to the dtype
 * the page's tensor has at that point:
 *
 *   gate logits, sigmoid (or softmax), biased choice score, group top-2 score
 *   (or group maximum), group and expert top-k, unbiased weights,
 *   renormalisation, route scale
 *       -- "Kimi K2 · Affinities", gate-forward excerpt (MoEGate.forward,
 *          noaux_tc) and "DeepSeek-V3.2-Exp · Affinities", gate-forward
 *          excerpt (Gate.forward)
 *   counts, stable slot sort, gather, per-expert MLP, unpermute, combine
 *       -- "Kimi K3 · Add shared output", moe-forward excerpt (moe_infer)
 *   expert MLP, SiLU-and-mul, SiTU
 *       -- "Kimi K3 · Gate features", expert excerpt (KimiBlockSparseMLP) and
 *          situ excerpt (SituAndMul, _get_situ_activation_params)
 *   latent down/up projections, routed-expert norm, shared-expert add
 *       -- "Kimi K3 · Add shared output", moe-forward excerpt
 *          (KimiSparseMoeBlock.forward)
 *
 * Readings where the pages are silent or disagree (each also listed in the
 * design notes):
 *   - masked groups are filled with -inf (the DeepSeek page) rather than 0.0
 *     (the Kimi page); both agree whenever the kept groups hold >= K positive
 *     scores;
 *   - every top-k breaks ties towards the lower index and emits its result in
 *     (value descending, index ascending) order;
 *   - sums over k (weight normaliser, combine) run sequentially k = 0..K-1;
 *   - the slot sort is stable (slots of one expert keep ascending slot order);
 *   - the sigmoid is the fp32 rounding of 1/(1+exp(-L)) evaluated in double;
 *   - the routed-expert norm is an RMSNorm (see oracle_rms_norm); the latent
 *     projections are bias-free; the shared experts are one gated MLP of the
 *     experts' kind on the full width (oracle_expert_ffn on every token).
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fopenmp (no x87: x86-64 SSE
 * arithmetic, so every float operation below is one IEEE fp32 operation).
 * OpenMP only splits independent tokens or rows between threads; the result
 * is bit-identical for any thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef uint16_t bf16_t;

enum { ORACLE_ACT_SILU = 0, ORACLE_ACT_SITU = 1 };

/* ----------------------------------------------------------- number formats */

static float bf16_value(bf16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Nearest-even bf16 of a float. */
static bf16_t bf16_round_f(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (bf16_t)((u >> 16) | 0x0040u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (bf16_t)(u >> 16);
}

/* Nearest-even bf16 of a double, rounded once (no detour through fp32).
 * Values below the fp32 normal range go through fp32 (irrelevant here). */
static bf16_t bf16_round_d(double d) {
  if (d != d) return 0x7FC0u;
  double a = fabs(d);
  if (a < 0x1p-126) return bf16_round_f((float)d);
  uint64_t u;
  memcpy(&u, &d, 8);
  /* keep 7 explicit mantissa bits of 52: drop 45 with round-half-even */
  uint64_t drop = 45;
  uint64_t half = 1ULL << (drop - 1);
  uint64_t lsb = (u >> drop) & 1ULL;
  u += (half - 1ULL) + lsb;
  u &= ~((1ULL << drop) - 1ULL);
  double r;
  memcpy(&r, &u, 8);
  if (fabs(r) >= 0x1p128) return (bf16_t)(d < 0 ? 0xFF80u : 0x7F80u);
  return bf16_round_f((float)r); /* exact: r has 8 significant bits */
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* -------------------------------------------------------------- the router */

/* logits[t,e] = fp32( sum_j x[t,j] * W[e,j] ): F.linear of the fp32-upcast
 * hidden states with the fp32 gate weight ("Kimi K2 · Affinities",
 * gate-forward: the F.linear call; "DeepSeek-V3.2-Exp · Affinities":
 * linear(x.float(), weight.float())). */
void oracle_gate_logits(const bf16_t* x, int64_t N, int d, const float* W, int E,
                        float* logits) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < N; ++t) {
    const bf16_t* xr = x + t * (int64_t)d;
    for (int e = 0; e < E; ++e) {
      const float* wr = W + (int64_t)e * d;
      double acc = 0.0;
      for (int j = 0; j < d; ++j) acc += (double)bf16_value(xr[j]) * (double)wr[j];
      logits[t * (int64_t)E + e] = (float)acc;
    }
  }
}

/* Sigmoid affinity (both router pages: scores = logits.sigmoid()). */
float oracle_sigmoid(float L) {
  return (float)(1.0 / (1.0 + exp(-(double)L)));
}

/* "a ranks before b": larger value first, then lower index. */
static int ranks_before(float a, int ia, float b, int ib) {
  return a > b || (a == b && ia < ib);
}

/* Group score of group g: sum of its two largest choice scores
 * (topk(2).sum on the [n, n_group, E/n_group] view).  One fp32 add. */
static float group_top2(const float* c, int gsz) {
  int i1 = 0;
  for (int i = 1; i < gsz; ++i)
    if (ranks_before(c[i], i, c[i1], i1)) i1 = i;
  int i2 = -1;
  for (int i = 0; i < gsz; ++i) {
    if (i == i1) continue;
    if (i2 < 0 || ranks_before(c[i], i, c[i2], i2)) i2 = i;
  }
  return c[i1] + c[i2];
}

/* Group score when the group has no top-2 sum: its largest choice score
 * ("DeepSeek-V3.2-Exp · Affinities", gate-forward: scores.amax(dim=-1), the
 * form that page uses when there is no correction bias). */
static float group_max(const float* c, int gsz) {
  float m = c[0];
  for (int i = 1; i < gsz; ++i)
    if (c[i] > m) m = c[i];
  return m;
}

enum { ORACLE_GROUP_TOP2_SUM = 0, ORACLE_GROUP_MAX = 1 };
enum { ORACLE_SCORE_SIGMOID = 0, ORACLE_SCORE_SOFTMAX = 1 };

static float group_score(const float* c, int gsz, int mode) {
  return mode == ORACLE_GROUP_MAX ? group_max(c, gsz) : group_top2(c, gsz);
}

void oracle_group_scores_ex(const float* c, int64_t N, int E, int G, int mode, float* gs) {
  const int gsz = E / G;
  for (int64_t t = 0; t < N; ++t)
    for (int g = 0; g < G; ++g) gs[t * G + g] = group_score(c + t * (int64_t)E + g * gsz, gsz, mode);
}

void oracle_group_scores(const float* c, int64_t N, int E, int G, float* gs) {
  oracle_group_scores_ex(c, N, E, G, ORACLE_GROUP_TOP2_SUM, gs);
}

/* Affinity scores of one token: sigmoid of each logit (both router pages), or
 * the softmax over all experts ("DeepSeek-V3.2-Exp · Affinities",
 * gate-forward: scores.softmax(dim=-1)), evaluated in double with the row
 * maximum subtracted, each rounded once to fp32. */
static void token_scores(const float* L, int E, int score_func, float* s) {
  if (score_func == ORACLE_SCORE_SOFTMAX) {
    double m = (double)L[0];
    for (int e = 1; e < E; ++e)
      if ((double)L[e] > m) m = (double)L[e];
    double sum = 0.0;
    for (int e = 0; e < E; ++e) sum += exp((double)L[e] - m);
    for (int e = 0; e < E; ++e) s[e] = (float)(exp((double)L[e] - m) / sum);
  } else {
    for (int e = 0; e < E; ++e) s[e] = oracle_sigmoid(L[e]);
  }
}

/* Selection and weights for one token, from its logits.
 *   s = sigmoid(L); c = s + bias (bias only steers the choice);
 *   if G > 1: group scores, keep the top TG groups, other experts get -inf;
 *   idx = top-K of c; w = s[idx]; if K > 1 and norm: w /= (sum w + 1e-20);
 *   w *= route_scale.
 * margin (optional) = min(gs_(TG) - gs_(TG+1), c_(K) - c_(K+1)) in double,
 * +inf where a boundary does not exist. */
static void route_token(const float* L, int E, const float* bias, int G, int TG, int K,
                        int norm, float route_scale, int score_func, int group_mode,
                        int32_t* idx, float* w, double* margin, float* s, float* c, float* gs,
                        unsigned char* used) {
  token_scores(L, E, score_func, s);
  for (int e = 0; e < E; ++e) c[e] = bias ? s[e] + bias[e] : s[e];
  double m_g = INFINITY, m_e = INFINITY;
  if (G > 1) {
    const int gsz = E / G;
    for (int g = 0; g < G; ++g) gs[g] = group_score(c + g * gsz, gsz, group_mode);
    /* top-TG groups by (gs desc, g asc) */
    memset(used, 0, (size_t)G);
    float last_kept = 0.0f;
    for (int r = 0; r < TG; ++r) {
      int best = -1;
      for (int g = 0; g < G; ++g)
        if (!used[g] && (best < 0 || ranks_before(gs[g], g, gs[best], best))) best = g;
      used[best] = 1;
      last_kept = gs[best];
    }
    if (TG < G) {
      int nxt = -1;
      for (int g = 0; g < G; ++g)
        if (!used[g] && (nxt < 0 || ranks_before(gs[g], g, gs[nxt], nxt))) nxt = g;
      m_g = (double)last_kept - (double)gs[nxt];
    }
    for (int g = 0; g < G; ++g)
      if (!used[g])
        for (int i = 0; i < gsz; ++i) c[g * gsz + i] = -INFINITY;
  }
  /* top-K experts by (c desc, e asc) */
  memset(used, 0, (size_t)E);
  for (int k = 0; k < K; ++k) {
    int best = -1;
    for (int e = 0; e < E; ++e)
      if (!used[e] && (best < 0 || ranks_before(c[e], e, c[best], best))) best = e;
    used[best] = 1;
    idx[k] = best;
  }
  {
    int nxt = -1;
    for (int e = 0; e < E; ++e)
      if (!used[e] && c[e] != -INFINITY && (nxt < 0 || ranks_before(c[e], e, c[nxt], nxt)))
        nxt = e;
    if (nxt >= 0) m_e = (double)c[idx[K - 1]] - (double)c[nxt];
  }
  /* unbiased weights, renormalised, scaled */
  for (int k = 0; k < K; ++k) w[k] = s[idx[k]];
  if (K > 1 && norm) {
    float den = w[0];
    for (int k = 1; k < K; ++k) den = den + w[k];
    den = den + 1e-20f;
    for (int k = 0; k < K; ++k) w[k] = w[k] / den;
  }
  for (int k = 0; k < K; ++k) w[k] = w[k] * route_scale;
  if (margin) *margin = m_g < m_e ? m_g : m_e;
}

void oracle_route_from_logits_ex(const float* logits, int64_t N, int E, const float* bias,
                                 int G, int TG, int K, int norm, float route_scale,
                                 int score_func, int group_mode, int32_t* idx, float* w,
                                 double* margin) {
#pragma omp parallel
  {
    float* s = (float*)malloc(sizeof(float) * (size_t)E);
    float* c = (float*)malloc(sizeof(float) * (size_t)E);
    float* gs = (float*)malloc(sizeof(float) * (size_t)(G > 0 ? G : 1));
    unsigned char* used = (unsigned char*)malloc((size_t)(E > G ? E : G));
#pragma omp for schedule(static)
    for (int64_t t = 0; t < N; ++t)
      route_token(logits + t * (int64_t)E, E, bias, G, TG, K, norm, route_scale, score_func,
                  group_mode, idx + t * (int64_t)K, w + t * (int64_t)K,
                  margin ? margin + t : NULL, s, c, gs, used);
    free(s); free(c); free(gs); free(used);
  }
}

void oracle_route_from_logits(const float* logits, int64_t N, int E, const float* bias, int G,
                              int TG, int K, int norm, float route_scale, int32_t* idx,
                              float* w, double* margin) {
  oracle_route_from_logits_ex(logits, N, E, bias, G, TG, K, norm, route_scale,
                              ORACLE_SCORE_SIGMOID, ORACLE_GROUP_TOP2_SUM, idx, w, margin);
}

/* Biased choice scores with the non-kept groups masked to -inf (for tests). */
void oracle_choice_scores_ex(const float* logits, int64_t N, int E, const float* bias, int G,
                             int TG, int score_func, int group_mode, float* c_out) {
  float* gs = (float*)malloc(sizeof(float) * (size_t)(G > 0 ? G : 1));
  unsigned char* used = (unsigned char*)malloc((size_t)(G > 0 ? G : 1));
  float* sc = (float*)malloc(sizeof(float) * (size_t)E);
  for (int64_t t = 0; t < N; ++t) {
    float* c = c_out + t * (int64_t)E;
    token_scores(logits + t * (int64_t)E, E, score_func, sc);
    for (int e = 0; e < E; ++e) c[e] = bias ? sc[e] + bias[e] : sc[e];
    if (G > 1) {
      const int gsz = E / G;
      for (int g = 0; g < G; ++g) gs[g] = group_score(c + g * gsz, gsz, group_mode);
      memset(used, 0, (size_t)G);
      for (int r = 0; r < TG; ++r) {
        int best = -1;
        for (int g = 0; g < G; ++g)
          if (!used[g] && (best < 0 || ranks_before(gs[g], g, gs[best], best))) best = g;
        used[best] = 1;
      }
      for (int g = 0; g < G; ++g)
        if (!used[g])
          for (int i = 0; i < gsz; ++i) c[g * gsz + i] = -INFINITY;
    }
  }
  free(gs); free(used); free(sc);
}

void oracle_choice_scores(const float* logits, int64_t N, int E, const float* bias, int G,
                          int TG, float* c_out) {
  oracle_choice_scores_ex(logits, N, E, bias, G, TG, ORACLE_SCORE_SIGMOID,
                          ORACLE_GROUP_TOP2_SUM, c_out);
}

/* ------------------------------------------------------------- moe_infer */

/* Per-expert counts, exclusive offsets and the stable sort of the flat slots
 * t*K+k by expert: perm[j] = slot at sorted position j, pos[slot] = j
 * ("Kimi K3 · Add shared output", moe_infer: cnts/scatter_/sum, argsort). */
void oracle_dispatch(const int32_t* idx, int64_t N, int K, int E, int32_t* counts,
                     int32_t* offsets, int32_t* perm, int32_t* pos) {
  const int64_t S = N * (int64_t)K;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t i = 0; i < S; ++i) counts[idx[i]] += 1;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
  for (int64_t i = 0; i < S; ++i) {
    int32_t p = cursor[idx[i]]++;
    perm[p] = (int32_t)i;
    pos[i] = p;
  }
  free(cursor);
}

/* sorted_tokens = x[idxs // K] */
void oracle_gather(const bf16_t* x, int d, const int32_t* perm, int64_t S, int K, bf16_t* xs) {
  for (int64_t j = 0; j < S; ++j)
    memcpy(xs + j * (int64_t)d, x + (int64_t)(perm[j] / K) * d, sizeof(bf16_t) * (size_t)d);
}

/* One expert's gated MLP on n rows ("Kimi K3 · Gate features", expert and situ
 * excerpts).  w1, w3: [F, d] (gate, up); w2: [d, F] (down); all bf16.
 *   g = bf16(x . w1^T), u = bf16(x . w3^T)       (bf16 nn.Linear outputs)
 *   SiLU-and-mul: h = bf16( bf16(silu(g)) * u ),  silu(g) = g * sigmoid(g)
 *   SiTU:         h = bf16( beta*tanh(g/beta)*sigmoid(g) * u' ),
 *                 u' = lbeta*tanh(u/lbeta) when lbeta is set, else u
 *   y = bf16(h . w2^T)
 * beta == 0 or NaN means 1.0 (the page's "beta or 1.0"); lbeta == 0 or NaN
 * means "not set".  Transcendentals are evaluated in double and rounded once
 * to bf16 (the page evaluates SiTU in fp32 and casts once to bf16). */
void oracle_expert_ffn(const bf16_t* xs, int64_t n, int d, int F, const bf16_t* w1,
                       const bf16_t* w3, const bf16_t* w2, int act, float beta, float lbeta,
                       bf16_t* y) {
  const double b = (beta == 0.0f || beta != beta) ? 1.0 : (double)beta;
  const int has_lb = !(lbeta == 0.0f || lbeta != lbeta);
  const double lb = (double)lbeta;
#pragma omp parallel
  {
    float* h = (float*)malloc(sizeof(float) * (size_t)F);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
      const bf16_t* xr = xs + r * (int64_t)d;
      for (int f = 0; f < F; ++f) {
        double ag = 0.0, au = 0.0;
        const bf16_t* r1 = w1 + (int64_t)f * d;
        const bf16_t* r3 = w3 + (int64_t)f * d;
        for (int j = 0; j < d; ++j) {
          double xv = (double)bf16_value(xr[j]);
          ag += xv * (double)bf16_value(r1[j]);
          au += xv * (double)bf16_value(r3[j]);
        }
        double g = (double)bf16_value(bf16_round_d(ag));
        double u = (double)bf16_value(bf16_round_d(au));
        double hv;
        if (act == ORACLE_ACT_SILU) {
          double a = (double)bf16_value(bf16_round_d(g / (1.0 + exp(-g))));
          hv = a * u; /* exact: a product of two bf16 values */
        } else {
          double up = has_lb ? lb * tanh(u / lb) : u;
          hv = b * tanh(g / b) * (1.0 / (1.0 + exp(-g))) * up;
        }
        h[f] = bf16_value(bf16_round_d(hv));
      }
      bf16_t* yr = y + r * (int64_t)d;
      for (int i = 0; i < d; ++i) {
        const bf16_t* r2 = w2 + (int64_t)i * F;
        double acc = 0.0;
        for (int f = 0; f < F; ++f) acc += (double)h[f] * (double)bf16_value(r2[f]);
        yr[i] = bf16_round_d(acc);
      }
    }
    free(h);
  }
}

/* Unpermute + combine: out[t] = bf16( sum_k fp32(y[pos[t*K+k]]) * w[t,k] ),
 * each product rounded to fp32, summed in fp32 for k = 0..K-1
 * (moe_infer: new_x[idxs] = outs; .type(fp32).mul_(w).sum(dim=1).type(bf16)). */
void oracle_combine(const bf16_t* y, const int32_t* pos, const float* w, int64_t N, int K,
                    int d, bf16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < N; ++t) {
    for (int i = 0; i < d; ++i) {
      float acc = bf16_value(y[(int64_t)pos[t * K] * d + i]) * w[t * K];
      for (int k = 1; k < K; ++k) {
        float p = bf16_value(y[(int64_t)pos[t * K + k] * d + i]) * w[t * K + k];
        acc = acc + p;
      }
      out[t * (int64_t)d + i] = bf16_round_f(acc);
    }
  }
}

/* The whole moe_infer on stacked expert weights (w1, w3: [E, F, d], w2:
 * [E, d, F]), following the page: dispatch, gather, per-expert MLP over each
 * non-empty segment, unpermute, combine.  ws must hold 2*S int32 + E + (E+1)
 * int32 and 2*S*d bf16 (see oracle_moe_infer_ws_bytes). */
size_t oracle_moe_infer_ws_bytes(int64_t N, int K, int E, int d) {
  const int64_t S = N * (int64_t)K;
  return sizeof(int32_t) * (size_t)(2 * S + 2 * E + 1) + sizeof(bf16_t) * (size_t)(2 * S * d);
}

void oracle_moe_infer(const bf16_t* x, int64_t N, int d, const int32_t* idx, const float* w,
                      int K, int E, int F, const bf16_t* w1, const bf16_t* w3, const bf16_t* w2,
                      int act, float beta, float lbeta, bf16_t* out, void* ws) {
  const int64_t S = N * (int64_t)K;
  int32_t* counts = (int32_t*)ws;
  int32_t* offsets = counts + E;
  int32_t* perm = offsets + E + 1;
  int32_t* pos = perm + S;
  bf16_t* xs = (bf16_t*)(pos + S);
  bf16_t* ys = xs + S * (int64_t)d;
  oracle_dispatch(idx, N, K, E, counts, offsets, perm, pos);
  oracle_gather(x, d, perm, S, K, xs);
  for (int e = 0; e < E; ++e) {
    const int64_t n = counts[e];
    if (n == 0) continue;
    const int64_t o = offsets[e];
    oracle_expert_ffn(xs + o * d, n, d, F, w1 + (int64_t)e * F * d, w3 + (int64_t)e * F * d,
                      w2 + (int64_t)e * d * F, act, beta, lbeta, ys + o * d);
  }
  oracle_combine(ys, pos, w, N, K, d, out);
}

/* The same layer as a per-token dense loop: for each token t and each k, run
 * expert idx[t,k] on x[t] directly, then combine as above.  No sort at all. */
void oracle_moe_dense(const bf16_t* x, int64_t N, int d, const int32_t* idx, const float* w,
                      int K, int F, const bf16_t* w1, const bf16_t* w3, const bf16_t* w2, int act,
                      float beta, float lbeta, bf16_t* out) {
  bf16_t* yk = (bf16_t*)malloc(sizeof(bf16_t) * (size_t)K * (size_t)d);
  int32_t* posk = (int32_t*)malloc(sizeof(int32_t) * (size_t)K);
  for (int64_t t = 0; t < N; ++t) {
    for (int k = 0; k < K; ++k) {
      const int64_t e = idx[t * K + k];
      oracle_expert_ffn(x + t * (int64_t)d, 1, d, F, w1 + e * F * d, w3 + e * F * d,
                        w2 + e * d * F, act, beta, lbeta, yk + (int64_t)k * d);
      posk[k] = k;
    }
    oracle_combine(yk, posk, w + t * K, 1, K, d, out + t * (int64_t)d);
  }
  free(yk);
  free(posk);
}

/* ------------------------------------------------- the block around moe_infer */

/* Bias-free bf16 nn.Linear: y[m,n] = bf16( sum_k x[m,k] * W[n,k] ), the sum in
 * double and rounded once.  routed_expert_down_proj and routed_expert_up_proj
 * of the latent block ("Kimi K3 · Add shared output", moe-forward excerpt,
 * KimiSparseMoeBlock.forward); their bias-free form is a reading, the same as
 * the experts' own Linear layers ("Kimi K3 · Gate features", expert excerpt). */
void oracle_linear(const bf16_t* x, int64_t M, int K, const bf16_t* W, int Nout, bf16_t* y) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t m = 0; m < M; ++m) {
    const bf16_t* xr = x + m * (int64_t)K;
    for (int n = 0; n < Nout; ++n) {
      const bf16_t* wr = W + (int64_t)n * K;
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += (double)bf16_value(xr[k]) * (double)bf16_value(wr[k]);
      y[m * (int64_t)Nout + n] = bf16_round_d(acc);
    }
  }
}

/* out = bf16( a + b ) elementwise for bf16 a, b: the exact sum rounded once
 * (the block's final y + shared_experts(identity)). */
void oracle_add(const bf16_t* a, const bf16_t* b, int64_t n, bf16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = bf16_round_d((double)bf16_value(a[i]) + (double)bf16_value(b[i]));
}

/* routed_expert_norm of the latent block, whose kind the pages do not show;
 * read as the RMSNorm the model family uses elsewhere (DeepseekV3RMSNorm in
 * "Kimi K2 · Masked scores", transformer excerpt): per row,
 *   r = 1 / sqrt( mean_i y_i^2 + eps )          (double)
 *   n_i = bf16( y_i * r )                         (normalised, cast back)
 *   out_i = bf16( w_i * n_i )                     (bf16 weight times bf16) */
void oracle_rms_norm(const bf16_t* x, int64_t N, int d, const bf16_t* w, float eps,
                     bf16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < N; ++t) {
    const bf16_t* xr = x + t * (int64_t)d;
    double ss = 0.0;
    for (int i = 0; i < d; ++i) {
      const double v = (double)bf16_value(xr[i]);
      ss += v * v;
    }
    const double r = 1.0 / sqrt(ss / (double)d + (double)eps);
    for (int i = 0; i < d; ++i) {
      const double nv = (double)bf16_value(bf16_round_d((double)bf16_value(xr[i]) * r));
      out[t * (int64_t)d + i] = bf16_round_d((double)bf16_value(w[i]) * nv);
    }
  }
}

/* Rounding helpers, exported so that tests can pin them. */
uint16_t oracle_bf16_round_double(double d) { return bf16_round_d(d); }
uint16_t oracle_bf16_round_float(float f) { return bf16_round_f(f); }
