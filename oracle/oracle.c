/*
 * ORACLE for the Mixture-of-Experts FFN layer -- test infrastructure only.
 *
 * A plain, slow, obviously correct CPU statement of what the layer computes,
 * accumulated in f64.  Only the tests, the smoke check and the benchmark's CPU
 * baseline call it; the product library never links, loads or runs it, and
 * this file shares no code, header, table or helper with the CUDA sources.
 *
 * Steps (notation: T tokens, H hidden, E experts, K selected per token,
 * I expert intermediate, Is shared intermediate; weights are out x in):
 *   1. logits   l[t,e] = sum_h x[t,h] W_r[e,h] (+ b_e)
 *               (hf2q qwen35/gpu_ffn.rs, build_moe_ffn_layer_gpu, router step;
 *                ferrox-models decoder.rs, gpt_oss_ffn: bias added to logits)
 *   2. select   experts ordered by (l descending, e ascending); ids = first K
 *               (hf2q qwen35/gpu_ffn.rs, softmax_topk_renorm_cpu: full stable
 *                sort of all experts, then the first K).
 *               Group-limited (ferrox-models decoder.rs calls
 *               route_top_k_grouped(logits, n_groups, groups used, K, ...)
 *               when the model has expert groups; its body is not printed):
 *               the E experts form n_groups contiguous groups of E/n_groups;
 *               a group's score is its largest logit; the topk_groups groups
 *               with the highest scores (lower group index first on ties)
 *               stay eligible and the K experts are chosen among them.
 *   3. weights  softmax gating: p_e = exp(l_e - m) / sum_j exp(l_j - m),
 *               m = max_e l_e; sigmoid gating (GatingFunction, the other
 *               router the pages name): p_e = 1 / (1 + exp(-l_e));
 *               renormalised: w_k = p_id_k / sum_k' p_id_k'; else w_k = p_id_k
 *               (softmax_topk_renorm_cpu; its 1e-20 guards are kept)
 *   4. permute  counts[e], exclusive offsets, pair ids p = t K + k stably
 *               sorted by expert, and the inverse pair_pos
 *               (DS4Server qwen_mtplx.rs, gather_sort: argsort of the flat
 *                expert ids and its inverse)
 *   5. experts  g = W_gate[e] x, u = W_up[e] x, a = act(g) * u, y = W_down[e] a,
 *               out[t] += w_k y summed in k order
 *               (mlx-native moe_dispatch.rs, moe_dispatch per-expert loop and
 *                moe_weighted_sum; hf2q qwen35/gpu_ffn.rs, silu_mul_cpu)
 *               act = SiLU g/(1+e^-g) (hf2q, silu_mul_cpu) or the tanh GELU
 *               0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3)))
 *               (mlx-native moe_dispatch.rs, tests, cpu_gelu)
 *   6. shared   s = sigmoid(w_s . x) when gated, else 1;
 *               out[t] += s * W_sdown (act(W_sgate x) * (W_sup x))
 *               (hf2q qwen35/gpu_ffn.rs, build_moe_ffn_layer_gpu, shared expert)
 *
 * Backward of two steps (mlx-native moe_dispatch.rs, the backward kernels of
 * moe_weighted_sum_seq and moe_swiglu_seq), for a loss L with dL/dout given:
 *   combine     out[t,d] = sum_k y[t,k,d] w[t,k]:
 *               d_y[t,k,d] = w[t,k] d_out[t,d];  d_w[t,k] = sum_d y[t,k,d] d_out[t,d]
 *   act * up    h[p,i] = act(g[p,i]) u[p,i], gate_up rows [g | u] of 2I:
 *               d_g = d_h u act'(g);  d_u = d_h act(g)
 *               act'(g) for SiLU: s (1 + g (1 - s)), s = 1/(1+e^-g);
 *               for the tanh GELU with z = c (g + a g^3), c = sqrt(2/pi),
 *               a = 0.044715: 0.5 (1 + tanh z) + 0.5 g (1 - tanh^2 z) c (1 + 3 a g^2)
 *
 * Storage formats read (converted exactly to f64): f32; bf16 (upper half of an
 * f32); Q8_0 GGML blocks {fp16 d; int8 q[32]} along the input dimension, value
 * = fp16(d) * q.  The k-quant stacks of the pages' Metal MoE providers
 * (ferrum-kernels vnext MoE: Q4_K and Q6_K blocks of 256 values, 144 and 210
 * bytes; their byte layout is GGML's, which the pages name but do not print):
 *   Q4_K {fp16 d; fp16 dmin; u8 scales[12]; u8 qs[128]}: eight sub-blocks of
 *     32 values, sub-block j with a 6-bit scale s_j and 6-bit min m_j packed in
 *     scales[] (j < 4: s = scales[j] & 63, m = scales[j+4] & 63; j >= 4:
 *     s = (scales[j+4] & 15) | (scales[j-4] >> 6) << 4,
 *     m = (scales[j+4] >> 4) | (scales[j] >> 6) << 4); value 32j + l is the
 *     low nibble of qs[32 (j/2) + l] for even j, the high nibble for odd j;
 *     value = d s_j q - dmin m_j.
 *   Q6_K {u8 ql[128]; u8 qh[64]; i8 scales[16]; fp16 d}: two halves of 128
 *     values; in half n, value 128n + 32i + l (i = 0..3, l = 0..31) has low
 *     four bits from ql[64n + l + 32 (i & 1)] (low nibble for i < 2, high for
 *     i >= 2) and high two bits (qh[32n + l] >> 2i) & 3; value =
 *     d scales[8n + (32i + l)/16] (q - 32).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Storage formats.  ORA_Q4_K_Q6_K is a layer format: gate/up rows in Q4_K,
 * down rows in Q6_K.  ORA_Q6_K is a row format only. */
enum { ORA_F32 = 0, ORA_BF16 = 1, ORA_Q8_0 = 2, ORA_Q4_K = 3, ORA_Q4_K_Q6_K = 4, ORA_Q6_K = 5 };
enum { ORA_SILU = 0, ORA_GELU_TANH = 1 };

enum { ORA_GATING_SOFTMAX = 0, ORA_GATING_SIGMOID = 1 };

typedef struct {
  int64_t T, H, E, I, K;
  int32_t act, renormalize;
  int32_t act_dtype, w_dtype, router_dtype;
  int32_t has_router_bias;
  int64_t shared_I;
  int32_t has_shared_gate;
  int32_t gating;                /* ORA_GATING_* */
  int64_t n_groups, topk_groups; /* group-limited selection when n_groups > 1 */
} ora_desc;

/* How one token's experts are chosen and weighted. */
typedef struct {
  int64_t E, K;
  int renorm, gating;
  int64_t n_groups, topk_groups;
} ora_route;

typedef struct {
  const void* x;          /* [T,H] act_dtype */
  const void* router;     /* [E,H] router_dtype */
  const float* bias;      /* [E] f32 or NULL */
  const void* gate;       /* [E,I,H] w_dtype */
  const void* up;         /* [E,I,H] */
  const void* down;       /* [E,H,I] */
  const void* sh_gate;    /* [Is,H] */
  const void* sh_up;      /* [Is,H] */
  const void* sh_down;    /* [H,Is] */
  const void* sh_gate_w;  /* [H] router_dtype */
} ora_tensors;

/* ---- exact conversions to f64 ---- */

double ora_fp16_to_double(uint16_t h) {
  int sign = (h >> 15) & 1, ex = (h >> 10) & 31, man = h & 1023;
  double v;
  if (ex == 0)
    v = ldexp((double)man, -24);                 /* zero and subnormals */
  else if (ex == 31)
    v = man ? NAN : INFINITY;
  else
    v = ldexp(1024.0 + man, ex - 25);            /* (1 + man/1024) 2^(ex-15) */
  return sign ? -v : v;
}

static inline double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Row r (of `cols` elements) of a row-major matrix stored in dtype, as f64. */
static void load_row(const void* base, int dtype, int64_t r, int64_t cols, double* out) {
  if (dtype == ORA_F32) {
    const float* p = (const float*)base + r * cols;
    for (int64_t c = 0; c < cols; ++c) out[c] = (double)p[c];
  } else if (dtype == ORA_BF16) {
    const uint16_t* p = (const uint16_t*)base + r * cols;
    for (int64_t c = 0; c < cols; ++c) out[c] = bf16_to_double(p[c]);
  } else if (dtype == ORA_Q4_K) {
    const uint8_t* p = (const uint8_t*)base + r * (cols / 256) * 144;
    for (int64_t b = 0; b < cols / 256; ++b) {
      const uint8_t* blk = p + b * 144;
      uint16_t db, mb;
      memcpy(&db, blk, 2);
      memcpy(&mb, blk + 2, 2);
      const double d = ora_fp16_to_double(db), dmin = ora_fp16_to_double(mb);
      const uint8_t* sc = blk + 4;
      const uint8_t* qs = blk + 16;
      for (int j = 0; j < 8; ++j) {
        int s, m;
        if (j < 4) {
          s = sc[j] & 63;
          m = sc[j + 4] & 63;
        } else {
          s = (sc[j + 4] & 15) | ((sc[j - 4] >> 6) << 4);
          m = (sc[j + 4] >> 4) | ((sc[j] >> 6) << 4);
        }
        for (int l = 0; l < 32; ++l) {
          const uint8_t byte = qs[32 * (j / 2) + l];
          const int q = (j % 2 == 0) ? (byte & 15) : (byte >> 4);
          out[b * 256 + 32 * j + l] = d * s * q - dmin * m;
        }
      }
    }
  } else if (dtype == ORA_Q6_K) {
    const uint8_t* p = (const uint8_t*)base + r * (cols / 256) * 210;
    for (int64_t b = 0; b < cols / 256; ++b) {
      const uint8_t* ql = p + b * 210;
      const uint8_t* qh = ql + 128;
      const int8_t* sc = (const int8_t*)(ql + 192);
      uint16_t db;
      memcpy(&db, ql + 208, 2);
      const double d = ora_fp16_to_double(db);
      for (int n = 0; n < 2; ++n)
        for (int i = 0; i < 4; ++i)
          for (int l = 0; l < 32; ++l) {
            const uint8_t lowb = ql[64 * n + l + 32 * (i & 1)];
            const int lo = i < 2 ? (lowb & 15) : (lowb >> 4);
            const int hi = (qh[32 * n + l] >> (2 * i)) & 3;
            const int q = lo | (hi << 4);
            const int j = 32 * i + l;
            out[b * 256 + 128 * n + j] = d * sc[8 * n + j / 16] * (q - 32);
          }
    }
  } else { /* Q8_0: 34-byte blocks, 32 values each */
    const uint8_t* p = (const uint8_t*)base + r * (cols / 32) * 34;
    for (int64_t b = 0; b < cols / 32; ++b) {
      uint16_t dbits;
      memcpy(&dbits, p + b * 34, 2);
      double d = ora_fp16_to_double(dbits);
      for (int j = 0; j < 32; ++j) out[b * 32 + j] = d * (double)(int8_t)p[b * 34 + 2 + j];
    }
  }
}

static double dot(const double* a, const double* b, int64_t n) {
  double s = 0.0;
  for (int64_t i = 0; i < n; ++i) s += a[i] * b[i];
  return s;
}

double ora_act(int act, double g) {
  if (act == ORA_SILU) return g / (1.0 + exp(-g));
  const double c = sqrt(2.0 / M_PI);
  return 0.5 * g * (1.0 + tanh(c * (g + 0.044715 * g * g * g)));
}

/* ---- step 1: router logits of one token ---- */
static void logits_one(const ora_desc* d, const ora_tensors* w, const double* xt, double* wrow, double* l,
                       double* absmax) {
  double am = 0.0;
  for (int64_t e = 0; e < d->E; ++e) {
    load_row(w->router, d->router_dtype, e, d->H, wrow);
    double s = 0.0, a = 0.0;
    for (int64_t h = 0; h < d->H; ++h) {
      s += xt[h] * wrow[h];
      a += fabs(xt[h] * wrow[h]);
    }
    if (d->has_router_bias) {
      s += (double)w->bias[e];
      a += fabs((double)w->bias[e]);
    }
    l[e] = s;
    if (a > am) am = a;
  }
  if (absmax) *absmax = am;
}

/* ---- steps 2-3: selection and weights from one token's logits ---- */
typedef struct {
  double l;
  int32_t e;
} ora_key;

static int by_logit_desc_index_asc(const void* pa, const void* pb) {
  const ora_key* a = (const ora_key*)pa;
  const ora_key* b = (const ora_key*)pb;
  if (a->l > b->l) return -1;
  if (a->l < b->l) return 1;
  return (a->e > b->e) - (a->e < b->e);
}

/* Gate values of all experts: max-subtracted softmax, or elementwise sigmoid. */
static void gate_all(const double* l, int64_t E, int gating, double* p) {
  if (gating == ORA_GATING_SIGMOID) {
    for (int64_t e = 0; e < E; ++e) p[e] = 1.0 / (1.0 + exp(-l[e]));
    return;
  }
  double m = -INFINITY;
  for (int64_t e = 0; e < E; ++e)
    if (l[e] > m) m = l[e];
  double denom = 0.0;
  for (int64_t e = 0; e < E; ++e) {
    p[e] = exp(l[e] - m);
    denom += p[e];
  }
  double inv = denom > 1e-20 ? 1.0 / denom : 1.0;
  for (int64_t e = 0; e < E; ++e) p[e] *= inv;
}

/* Weights of a given selection (ids[K]) from the probabilities. */
static void weights_of(const double* p, const int32_t* ids, int64_t K, int renorm, double* w) {
  if (!renorm) {
    for (int64_t k = 0; k < K; ++k) w[k] = p[ids[k]];
    return;
  }
  double sum_sel = 0.0;
  for (int64_t k = 0; k < K; ++k) sum_sel += p[ids[k]];
  double inv = sum_sel > 1e-20 ? 1.0 / sum_sel : 1.0 / (double)K;
  for (int64_t k = 0; k < K; ++k) w[k] = p[ids[k]] * inv;
}

/* keys[E] scratch; with groups, the experts of groups that are not among the
 * topk_groups best are left out of the sort. */
static void select_one(const double* l, const ora_route* r, ora_key* keys, double* p, int32_t* ids, double* w) {
  const int64_t E = r->E, K = r->K;
  int64_t n = 0;
  if (r->n_groups > 1) {
    const int64_t gs = E / r->n_groups;
    ora_key* gkeys = keys; /* group scores first, in the same scratch */
    for (int64_t g = 0; g < r->n_groups; ++g) {
      double m = -INFINITY;
      for (int64_t e = g * gs; e < (g + 1) * gs; ++e)
        if (l[e] > m) m = l[e];
      gkeys[g].l = m;
      gkeys[g].e = (int32_t)g;
    }
    qsort(gkeys, (size_t)r->n_groups, sizeof(ora_key), by_logit_desc_index_asc);
    char* keep = (char*)calloc((size_t)r->n_groups, 1);
    for (int64_t i = 0; i < r->topk_groups; ++i) keep[gkeys[i].e] = 1;
    for (int64_t e = 0; e < E; ++e)
      if (keep[e / gs]) {
        keys[n].l = l[e];
        keys[n].e = (int32_t)e;
        ++n;
      }
    free(keep);
  } else {
    for (int64_t e = 0; e < E; ++e) {
      keys[e].l = l[e];
      keys[e].e = (int32_t)e;
    }
    n = E;
  }
  qsort(keys, (size_t)n, sizeof(ora_key), by_logit_desc_index_asc);
  for (int64_t k = 0; k < K; ++k) ids[k] = keys[k].e;
  gate_all(l, E, r->gating, p);
  weights_of(p, ids, K, r->renorm, w);
}

/* Selection + weights for n tokens from given logits [n,E] (e.g. the GPU's f32 logits widened to f64). */
void ora_select(const double* logits, int64_t n, const ora_route* r, int32_t* ids, double* w) {
  const int64_t E = r->E, K = r->K;
#pragma omp parallel
  {
    ora_key* keys = (ora_key*)malloc(sizeof(ora_key) * E);
    double* p = (double*)malloc(sizeof(double) * E);
#pragma omp for schedule(static)
    for (int64_t t = 0; t < n; ++t) select_one(logits + t * E, r, keys, p, ids + t * K, w + t * K);
    free(keys);
    free(p);
  }
}

/* Weights of a forced selection ids[n,K] from logits [n,E]. */
void ora_weights_for(const double* logits, int64_t n, const ora_route* r, const int32_t* ids, double* w) {
  double* p = (double*)malloc(sizeof(double) * r->E);
  for (int64_t t = 0; t < n; ++t) {
    gate_all(logits + t * r->E, r->E, r->gating, p);
    weights_of(p, ids + t * r->K, r->K, r->renorm, w + t * r->K);
  }
  free(p);
}

static ora_route route_of(const ora_desc* d) {
  ora_route r;
  r.E = d->E;
  r.K = d->K;
  r.renorm = d->renormalize;
  r.gating = d->gating;
  r.n_groups = d->n_groups;
  r.topk_groups = d->topk_groups;
  return r;
}

/* ---- step 4: stable permutation of pair ids by expert (counting sort) ---- */
int ora_permute(const int32_t* ids, int64_t P, int64_t E, int32_t* counts, int32_t* offsets, int32_t* sorted_pairs,
                int32_t* pair_pos) {
  if (E < 1 || P < 0) return -1;
  for (int64_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t p = 0; p < P; ++p) {
    if (ids[p] < 0 || ids[p] >= E) return -1;
    counts[ids[p]]++;
  }
  offsets[0] = 0;
  for (int64_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
  for (int64_t p = 0; p < P; ++p) {
    int32_t e = ids[p];
    int32_t pos = offsets[e] + fill[e]++;
    sorted_pairs[pos] = (int32_t)p;
    pair_pos[p] = pos;
  }
  free(fill);
  return 0;
}

/* ---- step 5/6 building block: one gated FFN on one token ---- */
/* y[Hout] = Wd (act(Wg xt) * (Wu xt)); Wg, Wu are [F, Hin] rows at row0, Wd is [Hout, F] rows at drow0. */
/* Row formats of the gate/up and of the down projections of a layer format. */
static int gu_format(int w_dtype) { return w_dtype == ORA_Q4_K_Q6_K ? ORA_Q4_K : w_dtype; }
static int down_format(int w_dtype) { return w_dtype == ORA_Q4_K_Q6_K ? ORA_Q6_K : w_dtype; }

static void ffn_one(int act, int w_dtype, const void* Wg, const void* Wu, const void* Wd, int64_t row0, int64_t drow0,
                    int64_t F, int64_t Hin, int64_t Hout, const double* xt, double* a, double* row, double* y) {
  const int gf = gu_format(w_dtype), df = down_format(w_dtype);
  for (int64_t i = 0; i < F; ++i) {
    load_row(Wg, gf, row0 + i, Hin, row);
    double g = dot(row, xt, Hin);
    load_row(Wu, gf, row0 + i, Hin, row);
    double u = dot(row, xt, Hin);
    a[i] = ora_act(act, g) * u;
  }
  for (int64_t j = 0; j < Hout; ++j) {
    load_row(Wd, df, drow0 + j, F, row);
    y[j] = dot(row, a, F);
  }
}

/* Expert e applied to token t: y[H]. */
void ora_expert(const ora_desc* d, const ora_tensors* w, int64_t t, int64_t e, double* y) {
  int64_t H = d->H, I = d->I, big = H > I ? H : I;
  double* xt = (double*)malloc(sizeof(double) * H);
  double* a = (double*)malloc(sizeof(double) * I);
  double* row = (double*)malloc(sizeof(double) * big);
  load_row(w->x, d->act_dtype, t, H, xt);
  ffn_one(d->act, d->w_dtype, w->gate, w->up, w->down, e * I, e * H, I, H, H, xt, a, row, y);
  free(xt);
  free(a);
  free(row);
}

double ora_sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/*
 * The whole layer on a list of tokens (tokens == NULL: tokens 0..n-1).
 * out[n,H] f64.  Optional outputs: logits[n,E], ids[n,K], w[n,K], gate_s[n]
 * (the shared-expert scale), absmax[n] (max_e sum_h |x W_r| + |b|, the scale of
 * the logits' rounding error).  force_ids[n,K], when given, replaces the
 * selection (weights are then those of the forced set under the oracle's own
 * logits).
 */
void ora_layer(const ora_desc* d, const ora_tensors* w, const int64_t* tokens, int64_t n, const int32_t* force_ids,
               double* out, double* logits_out, int32_t* ids_out, double* w_out, double* gate_s_out,
               double* absmax_out) {
  const int64_t H = d->H, E = d->E, I = d->I, K = d->K, Is = d->shared_I;
  const ora_route rt = route_of(d);
  int64_t big = H;
  if (I > big) big = I;
  if (Is > big) big = Is;
#pragma omp parallel
  {
    double* xt = (double*)malloc(sizeof(double) * H);
    double* row = (double*)malloc(sizeof(double) * big);
    double* a = (double*)malloc(sizeof(double) * (I > Is ? I : Is) + 8);
    double* y = (double*)malloc(sizeof(double) * H);
    double* l = (double*)malloc(sizeof(double) * E);
    double* p = (double*)malloc(sizeof(double) * E);
    ora_key* keys = (ora_key*)malloc(sizeof(ora_key) * E);
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * K);
    double* wk = (double*)malloc(sizeof(double) * K);
#pragma omp for schedule(dynamic, 1)
    for (int64_t i = 0; i < n; ++i) {
      int64_t t = tokens ? tokens[i] : i;
      load_row(w->x, d->act_dtype, t, H, xt);
      double am = 0.0;
      logits_one(d, w, xt, row, l, &am);
      if (force_ids) {
        for (int64_t k = 0; k < K; ++k) ids[k] = force_ids[i * K + k];
        gate_all(l, E, d->gating, p);
        weights_of(p, ids, K, d->renormalize, wk);
      } else {
        select_one(l, &rt, keys, p, ids, wk);
      }
      double* o = out + i * H;
      for (int64_t j = 0; j < H; ++j) o[j] = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        int64_t e = ids[k];
        ffn_one(d->act, d->w_dtype, w->gate, w->up, w->down, e * I, e * H, I, H, H, xt, a, row, y);
        for (int64_t j = 0; j < H; ++j) o[j] += wk[k] * y[j];
      }
      double s = 1.0;
      if (Is > 0) {
        if (d->has_shared_gate) {
          load_row(w->sh_gate_w, d->router_dtype, 0, H, row);
          s = ora_sigmoid(dot(row, xt, H));
        }
        ffn_one(d->act, d->w_dtype, w->sh_gate, w->sh_up, w->sh_down, 0, 0, Is, H, H, xt, a, row, y);
        for (int64_t j = 0; j < H; ++j) o[j] += s * y[j];
      }
      if (logits_out)
        for (int64_t e = 0; e < E; ++e) logits_out[i * E + e] = l[e];
      if (ids_out)
        for (int64_t k = 0; k < K; ++k) ids_out[i * K + k] = ids[k];
      if (w_out)
        for (int64_t k = 0; k < K; ++k) w_out[i * K + k] = wk[k];
      if (gate_s_out) gate_s_out[i] = s;
      if (absmax_out) absmax_out[i] = am;
    }
    free(xt);
    free(row);
    free(a);
    free(y);
    free(l);
    free(p);
    free(keys);
    free(ids);
    free(wk);
  }
}

/* Router logits only (step 1) for a token list; absmax as in ora_layer. */
void ora_logits(const ora_desc* d, const ora_tensors* w, const int64_t* tokens, int64_t n, double* logits,
                double* absmax) {
  const int64_t H = d->H, E = d->E;
#pragma omp parallel
  {
    double* xt = (double*)malloc(sizeof(double) * H);
    double* row = (double*)malloc(sizeof(double) * H);
#pragma omp for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
      int64_t t = tokens ? tokens[i] : i;
      load_row(w->x, d->act_dtype, t, H, xt);
      logits_one(d, w, xt, row, logits + i * E, absmax ? absmax + i : NULL);
    }
    free(xt);
    free(row);
  }
}

/* Shared expert alone for a token list: y[n,H] = s * FFN_shared(x), s as in step 6; gate_s[n] optional. */
void ora_shared(const ora_desc* d, const ora_tensors* w, const int64_t* tokens, int64_t n, double* y_out,
                double* gate_s_out) {
  const int64_t H = d->H, Is = d->shared_I;
  int64_t big = H > Is ? H : Is;
#pragma omp parallel
  {
    double* xt = (double*)malloc(sizeof(double) * H);
    double* row = (double*)malloc(sizeof(double) * big);
    double* a = (double*)malloc(sizeof(double) * Is + 8);
#pragma omp for schedule(dynamic, 1)
    for (int64_t i = 0; i < n; ++i) {
      int64_t t = tokens ? tokens[i] : i;
      load_row(w->x, d->act_dtype, t, H, xt);
      double s = 1.0;
      if (d->has_shared_gate) {
        load_row(w->sh_gate_w, d->router_dtype, 0, H, row);
        s = ora_sigmoid(dot(row, xt, H));
      }
      double* y = y_out + i * H;
      ffn_one(d->act, d->w_dtype, w->sh_gate, w->sh_up, w->sh_down, 0, 0, Is, H, H, xt, a, row, y);
      for (int64_t j = 0; j < H; ++j) y[j] *= s;
      if (gate_s_out) gate_s_out[i] = s;
    }
    free(xt);
    free(row);
    free(a);
  }
}

/* Derivative of the activation (step "act * up" of the backward, header). */
double ora_act_grad(int act, double g) {
  if (act == ORA_SILU) {
    const double s = 1.0 / (1.0 + exp(-g));
    return s * (1.0 + g * (1.0 - s));
  }
  const double c = sqrt(2.0 / M_PI), a = 0.044715;
  const double th = tanh(c * (g + a * g * g * g));
  return 0.5 * (1.0 + th) + 0.5 * g * (1.0 - th * th) * c * (1.0 + 3.0 * a * g * g);
}

/* Backward of the combine: y[T,K,H], w[T,K], d_out[T,H] (f32, as stored) ->
 * d_y[T,K,H], d_w[T,K] in f64. */
void ora_combine_backward(const float* y, const float* w, const float* d_out, int64_t T, int64_t K, int64_t H,
                          double* d_y, double* d_w) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t k = 0; k < K; ++k) {
      const int64_t p = t * K + k;
      double s = 0.0;
      for (int64_t d = 0; d < H; ++d) {
        d_y[p * H + d] = (double)w[p] * (double)d_out[t * H + d];
        s += (double)y[p * H + d] * (double)d_out[t * H + d];
      }
      d_w[p] = s;
    }
  }
}

/* Backward of act(gate) * up: gate_up[P, 2I] (gate in columns [0, I), up in
 * [I, 2I)), d_h[P, I] (f32) -> d_gate_up[P, 2I] in f64, same layout. */
void ora_act_up_backward(int act, const float* gate_up, const float* d_h, int64_t P, int64_t I,
                         double* d_gate_up) {
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < P; ++p) {
    for (int64_t i = 0; i < I; ++i) {
      const double g = gate_up[p * 2 * I + i], u = gate_up[p * 2 * I + I + i], dh = d_h[p * I + i];
      d_gate_up[p * 2 * I + i] = dh * u * ora_act_grad(act, g);
      d_gate_up[p * 2 * I + I + i] = dh * ora_act(act, g);
    }
  }
}

/* Dequantise n rows of a Q8_0 (or f32/bf16) matrix with `cols` columns to f64. */
void ora_load_rows(const void* base, int dtype, int64_t r0, int64_t n, int64_t cols, double* out) {
  for (int64_t r = 0; r < n; ++r) load_row(base, dtype, r0 + r, cols, out + r * cols);
}

void ora_act_array(int act, const double* g, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = ora_act(act, g[i]);
}

int ora_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void ora_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
