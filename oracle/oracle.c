/*
 * oracle.c -- float64 CPU definition of causal sliding-window RoPE attention
 * with parameter-free QK RMSNorm, grouped-query attention (GQA) and the
 * value-embedding residual, forward and backward.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark load this file. The CUDA library never calls it, and
 * the two share no code, headers, tables or constants.
 *
 * What it follows. Page "5만원으로 나만의 ChatGPT 훈련하는 방법" (apidog.com):
 *   - section "1. GPT 모델 (nanochat/gpt.py)", architecture list: rotary
 *     embeddings (RoPE) instead of learned positions, QK normalisation, GQA
 *     (fewer KV heads than query heads) and sliding-window attention with a
 *     per-layer pattern such as "SSSL";
 *   - same section, "값 임베딩 (Value Embeddings, ResFormer)": the value
 *     embedding, viewed per KV head, is mixed in as v + 3*sigmoid(gate)*ve
 *     with one gate per (token, KV head) broadcast over head_dim;
 *   - section "5. 플래시 어텐션 통합 (nanochat/flash_attention.py)": the
 *     attention itself is a causal call with a window size on (B, T, H, D)
 *     tensors.
 * The pages do not write the attention arithmetic out. This file takes the
 * plain reading, one step per function:
 *   r(x) = (sum_d x_d^2 / D + eps)^(-1/2),  n(x) = r(x) x          (RMSNorm)
 *   RoPE: pairs (i, i + D/2), angle a = pos * base^(-2i/D),
 *         y_i = x_i cos a - x_{i+D/2} sin a, y_{i+D/2} = x_i sin a + x_{i+D/2} cos a
 *   q~ = RoPE(n(q)), k~ = RoPE(n(k)), v_eff = v + 3 sigmoid(gate) ve
 *   s_ij = c q~_i . k~_j for i - W < j <= i (W keys, the query itself included)
 *   lse_i = log sum_j exp(s_ij),  p_ij = exp(s_ij - lse_i),  O_i = sum_j p_ij v_eff_j
 * and the backward is the chain rule of the same steps, written out.
 * Query head h reads KV head h / (H / Hk).
 *
 * Layouts (row-major, D contiguous): q, O, dO (B,T,H,D); k, v, ve (B,T,Hk,D);
 * gate (B,T,Hk); lse (B,H,T); rstd (B,T,heads).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_NO_NORM 1 /* test switch: skip the RMSNorm (n(x) = x) */
#define ORACLE_NO_ROPE 2 /* test switch: skip the rotation */

typedef struct {
  int B, T, H, Hk, D, W;
  int has_ve;
  int flags;      /* ORACLE_NO_NORM | ORACLE_NO_ROPE, test switches only */
  int pos_offset; /* position of token 0; 0 in normal use (test hook) */
  double rope_base, eps, scale;
} oracle_layer;

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

static size_t idx4(int b, int t, int h, int d, int T, int Hn, int D) {
  return (((size_t)b * T + t) * Hn + h) * (size_t)D + d;
}

/* RMSNorm of one row: writes n = r x, returns r. Architecture list, "QK
 * normalization"; parameter-free, eps inside the square root. */
static double rms_norm_row(const double *x, double *n, int D, double eps,
                           int skip) {
  if (skip) {
    memcpy(n, x, sizeof(double) * D);
    return 1.0;
  }
  double ss = 0.0;
  for (int d = 0; d < D; ++d) ss += x[d] * x[d];
  double r = 1.0 / sqrt(ss / D + eps);
  for (int d = 0; d < D; ++d) n[d] = x[d] * r;
  return r;
}

/* Rotation of one row at position pos. Architecture list, "Rotary
 * embeddings (RoPE)"; half-split pairs, positive angle. inverse=1 applies the
 * transpose (the inverse rotation), used by the backward. */
static void rope_row(const double *x, double *y, int D, double pos,
                     double base, int inverse, int skip) {
  int half = D / 2;
  if (skip) {
    memcpy(y, x, sizeof(double) * D);
    return;
  }
  for (int i = 0; i < half; ++i) {
    double w = pow(base, -2.0 * i / (double)D);
    double a = pos * w;
    double c = cos(a), s = sin(a);
    double x0 = x[i], x1 = x[i + half];
    if (!inverse) {
      y[i] = x0 * c - x1 * s;
      y[i + half] = x0 * s + x1 * c;
    } else {
      y[i] = x0 * c + x1 * s;
      y[i + half] = -x0 * s + x1 * c;
    }
  }
}

/* Prologue: q~ = RoPE(n(q)), k~ = RoPE(n(k)), v_eff = v + 3 sigmoid(gate) ve.
 * rq, rk receive the RMSNorm factors r (1 when the norm is switched off).
 * ve and gate are read only when has_ve. */
void oracle_prologue(const oracle_layer *L, const double *q, const double *k,
                     const double *v, const double *ve, const double *gate,
                     double *qt, double *kt, double *veff, double *rq,
                     double *rk) {
  const int B = L->B, T = L->T, H = L->H, Hk = L->Hk, D = L->D;
  const int no_norm = (L->flags & ORACLE_NO_NORM) != 0;
  const int no_rope = (L->flags & ORACLE_NO_ROPE) != 0;
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < T; ++t) {
      double n[1024];
      double pos = (double)(t + L->pos_offset);
      for (int h = 0; h < H; ++h) {
        size_t o = idx4(b, t, h, 0, T, H, D);
        rq[((size_t)b * T + t) * H + h] =
            rms_norm_row(q + o, n, D, L->eps, no_norm);
        rope_row(n, qt + o, D, pos, L->rope_base, 0, no_rope);
      }
      for (int h = 0; h < Hk; ++h) {
        size_t o = idx4(b, t, h, 0, T, Hk, D);
        rk[((size_t)b * T + t) * Hk + h] =
            rms_norm_row(k + o, n, D, L->eps, no_norm);
        rope_row(n, kt + o, D, pos, L->rope_base, 0, no_rope);
        /* Value residual ("값 임베딩"): one gate per (token, KV head). */
        double coef = L->has_ve ? 3.0 * sigmoid(gate[((size_t)b * T + t) * Hk + h]) : 0.0;
        for (int d = 0; d < D; ++d)
          veff[o + d] = v[o + d] + (L->has_ve ? coef * ve[o + d] : 0.0);
      }
    }
}

static int kv_head(const oracle_layer *L, int h) { return h / (L->H / L->Hk); }

/* First visible key of query i: W keys including the query itself. */
static int first_key(const oracle_layer *L, int i) {
  long lo = (long)i - (long)L->W + 1;
  return lo < 0 ? 0 : (int)lo;
}

static double score(const oracle_layer *L, const double *qt, const double *kt,
                    int b, int h, int i, int j) {
  const double *qi = qt + idx4(b, i, h, 0, L->T, L->H, L->D);
  const double *kj = kt + idx4(b, j, kv_head(L, h), 0, L->T, L->Hk, L->D);
  double s = 0.0;
  for (int d = 0; d < L->D; ++d) s += qi[d] * kj[d];
  return L->scale * s;
}

/* Softmax probabilities of one query row: p[j] for j = 0..T-1 (0 where the
 * causal window masks the key). Returns lse_i. */
double oracle_probs_row(const oracle_layer *L, const double *qt,
                        const double *kt, int b, int h, int i, double *p) {
  int lo = first_key(L, i);
  double m = -INFINITY;
  for (int j = 0; j < L->T; ++j) p[j] = 0.0;
  for (int j = lo; j <= i; ++j) {
    p[j] = score(L, qt, kt, b, h, i, j);
    if (p[j] > m) m = p[j];
  }
  double sum = 0.0;
  for (int j = lo; j <= i; ++j) sum += exp(p[j] - m);
  double lse = m + log(sum);
  for (int j = lo; j <= i; ++j) p[j] = exp(p[j] - lse);
  return lse;
}

/* Forward of one query row: O_i = sum_j p_ij v_eff_j and lse_i. */
static double fwd_row(const oracle_layer *L, const double *qt,
                      const double *kt, const double *veff, int b, int h,
                      int i, double *o, double *p) {
  const int D = L->D, hk = kv_head(L, h);
  double lse = oracle_probs_row(L, qt, kt, b, h, i, p);
  for (int d = 0; d < D; ++d) o[d] = 0.0;
  for (int j = first_key(L, i); j <= i; ++j) {
    const double *vj = veff + idx4(b, j, hk, 0, L->T, L->Hk, D);
    for (int d = 0; d < D; ++d) o[d] += p[j] * vj[d];
  }
  return lse;
}

/* Forward over the whole layer: O (B,T,H,D), lse (B,H,T), natural log. */
void oracle_attn_fwd(const oracle_layer *L, const double *qt, const double *kt,
                     const double *veff, double *O, double *lse) {
  const int B = L->B, T = L->T, H = L->H, D = L->D;
#pragma omp parallel
  {
    double *p = (double *)malloc(sizeof(double) * (size_t)T);
#pragma omp for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
      for (int h = 0; h < H; ++h)
        for (int i = 0; i < T; ++i)
          lse[((size_t)b * H + h) * T + i] =
              fwd_row(L, qt, kt, veff, b, h, i, O + idx4(b, i, h, 0, T, H, D), p);
    free(p);
  }
}

/* Forward of selected rows only. rows holds n triples (b, h, i). */
void oracle_fwd_rows(const oracle_layer *L, const double *qt, const double *kt,
                     const double *veff, int n, const int *rows, double *O,
                     double *lse) {
#pragma omp parallel
  {
    double *p = (double *)malloc(sizeof(double) * (size_t)L->T);
#pragma omp for schedule(dynamic, 1)
    for (int r = 0; r < n; ++r)
      lse[r] = fwd_row(L, qt, kt, veff, rows[3 * r], rows[3 * r + 1],
                       rows[3 * r + 2], O + (size_t)r * L->D, p);
    free(p);
  }
}

/* Backward of the attention core, given dO and the forward's O and lse:
 *   Delta_i = dO_i . O_i,  dp_ij = dO_i . v_eff_j,  ds_ij = p_ij (dp_ij - Delta_i)
 *   dq~_i = c sum_j ds_ij k~_j
 *   dk~_j = c sum_{h in group} sum_i ds_ij q~_i
 *   dv_eff_j = sum_{h in group} sum_i p_ij dO_i
 * Outputs dqt (B,T,H,D), dkt and dveff (B,T,Hk,D), overwritten. */
void oracle_attn_bwd(const oracle_layer *L, const double *qt, const double *kt,
                     const double *veff, const double *O, const double *lse,
                     const double *dO, double *dqt, double *dkt,
                     double *dveff) {
  const int B = L->B, T = L->T, H = L->H, Hk = L->Hk, D = L->D;
  const int g = H / Hk;
  memset(dqt, 0, sizeof(double) * (size_t)B * T * H * D);
  memset(dkt, 0, sizeof(double) * (size_t)B * T * Hk * D);
  memset(dveff, 0, sizeof(double) * (size_t)B * T * Hk * D);
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int b = 0; b < B; ++b)
    for (int hk = 0; hk < Hk; ++hk)
      for (int h = hk * g; h < (hk + 1) * g; ++h)
        for (int i = 0; i < T; ++i) {
          const double *dOi = dO + idx4(b, i, h, 0, T, H, D);
          const double *Oi = O + idx4(b, i, h, 0, T, H, D);
          const double *qi = qt + idx4(b, i, h, 0, T, H, D);
          double *dqi = dqt + idx4(b, i, h, 0, T, H, D);
          double li = lse[((size_t)b * H + h) * T + i];
          double delta = 0.0;
          for (int d = 0; d < D; ++d) delta += dOi[d] * Oi[d];
          for (int j = first_key(L, i); j <= i; ++j) {
            const double *kj = kt + idx4(b, j, hk, 0, T, Hk, D);
            const double *vj = veff + idx4(b, j, hk, 0, T, Hk, D);
            double p = exp(score(L, qt, kt, b, h, i, j) - li);
            double dp = 0.0;
            for (int d = 0; d < D; ++d) dp += dOi[d] * vj[d];
            double ds = p * (dp - delta);
            double *dkj = dkt + idx4(b, j, hk, 0, T, Hk, D);
            double *dvj = dveff + idx4(b, j, hk, 0, T, Hk, D);
            for (int d = 0; d < D; ++d) {
              dqi[d] += L->scale * ds * kj[d];
              dkj[d] += L->scale * ds * qi[d];
              dvj[d] += p * dOi[d];
            }
          }
        }
}

/* dq~ of selected query rows (b, h, i), from scratch: the row's own lse, O
 * and Delta are recomputed here from the definition. */
void oracle_dq_rows(const oracle_layer *L, const double *qt, const double *kt,
                    const double *veff, const double *dO, int n,
                    const int *rows, double *dqt) {
  const int D = L->D, T = L->T;
#pragma omp parallel
  {
    double *p = (double *)malloc(sizeof(double) * (size_t)T);
    double *o = (double *)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
    for (int r = 0; r < n; ++r) {
      int b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
      int hk = kv_head(L, h);
      fwd_row(L, qt, kt, veff, b, h, i, o, p);
      const double *dOi = dO + idx4(b, i, h, 0, T, L->H, D);
      double delta = 0.0;
      for (int d = 0; d < D; ++d) delta += dOi[d] * o[d];
      double *out = dqt + (size_t)r * D;
      for (int d = 0; d < D; ++d) out[d] = 0.0;
      for (int j = first_key(L, i); j <= i; ++j) {
        const double *vj = veff + idx4(b, j, hk, 0, T, L->Hk, D);
        const double *kj = kt + idx4(b, j, hk, 0, T, L->Hk, D);
        double dp = 0.0;
        for (int d = 0; d < D; ++d) dp += dOi[d] * vj[d];
        double ds = p[j] * (dp - delta);
        for (int d = 0; d < D; ++d) out[d] += L->scale * ds * kj[d];
      }
    }
    free(o);
    free(p);
  }
}

/* dk~ and dv_eff of selected key rows (b, hk, j), from scratch: every query
 * of the group that sees key j gets its lse, O and Delta recomputed. */
void oracle_dkv_rows(const oracle_layer *L, const double *qt, const double *kt,
                     const double *veff, const double *dO, int n,
                     const int *rows, double *dkt, double *dveff) {
  const int D = L->D, T = L->T, H = L->H, g = L->H / L->Hk;
#pragma omp parallel
  {
    double *p = (double *)malloc(sizeof(double) * (size_t)T);
    double *o = (double *)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
    for (int r = 0; r < n; ++r) {
      int b = rows[3 * r], hk = rows[3 * r + 1], j = rows[3 * r + 2];
      const double *vj = veff + idx4(b, j, hk, 0, T, L->Hk, D);
      double *dk = dkt + (size_t)r * D, *dv = dveff + (size_t)r * D;
      for (int d = 0; d < D; ++d) dk[d] = dv[d] = 0.0;
      long last = (long)j + (long)L->W - 1;
      if (last > T - 1) last = T - 1;
      for (int h = hk * g; h < (hk + 1) * g; ++h)
        for (int i = j; i <= (int)last; ++i) {
          fwd_row(L, qt, kt, veff, b, h, i, o, p);
          const double *dOi = dO + idx4(b, i, h, 0, T, H, D);
          const double *qi = qt + idx4(b, i, h, 0, T, H, D);
          double delta = 0.0, dp = 0.0;
          for (int d = 0; d < D; ++d) {
            delta += dOi[d] * o[d];
            dp += dOi[d] * vj[d];
          }
          double ds = p[j] * (dp - delta);
          for (int d = 0; d < D; ++d) {
            dk[d] += L->scale * ds * qi[d];
            dv[d] += p[j] * dOi[d];
          }
        }
    }
    free(o);
    free(p);
  }
}

/* Chain rule back through the prologue, row-wise:
 *   RoPE^-1: the transpose rotation of dq~, dk~;
 *   RMSNorm: dx = r (dn - n mean_d(dn * n)) with n = r x;
 *   dv = dv_eff, dve = 3 sigmoid(g) dv_eff,
 *   dgate = 3 sigmoid(g) (1 - sigmoid(g)) sum_d dv_eff * ve.
 * dve and dgate are written only when has_ve. */
void oracle_prologue_bwd(const oracle_layer *L, const double *q,
                         const double *k, const double *ve, const double *gate,
                         const double *dqt, const double *dkt,
                         const double *dveff, double *dq, double *dk,
                         double *dv, double *dve, double *dgate) {
  const int B = L->B, T = L->T, H = L->H, Hk = L->Hk, D = L->D;
  const int no_norm = (L->flags & ORACLE_NO_NORM) != 0;
  const int no_rope = (L->flags & ORACLE_NO_ROPE) != 0;
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < T; ++t) {
      double n[1024], dn[1024];
      double pos = (double)(t + L->pos_offset);
      for (int pass = 0; pass < 2; ++pass) {
        int Hn = pass == 0 ? H : Hk;
        const double *x = pass == 0 ? q : k;
        const double *dy = pass == 0 ? dqt : dkt;
        double *dx = pass == 0 ? dq : dk;
        for (int h = 0; h < Hn; ++h) {
          size_t o = idx4(b, t, h, 0, T, Hn, D);
          rope_row(dy + o, dn, D, pos, L->rope_base, 1, no_rope);
          if (no_norm) {
            for (int d = 0; d < D; ++d) dx[o + d] = dn[d];
            continue;
          }
          double r = rms_norm_row(x + o, n, D, L->eps, 0);
          double dot = 0.0;
          for (int d = 0; d < D; ++d) dot += dn[d] * n[d];
          dot /= D;
          for (int d = 0; d < D; ++d) dx[o + d] = r * (dn[d] - n[d] * dot);
        }
      }
      for (int h = 0; h < Hk; ++h) {
        size_t o = idx4(b, t, h, 0, T, Hk, D);
        for (int d = 0; d < D; ++d) dv[o + d] = dveff[o + d];
        if (!L->has_ve) continue;
        double s = sigmoid(gate[((size_t)b * T + t) * Hk + h]);
        double acc = 0.0;
        for (int d = 0; d < D; ++d) {
          dve[o + d] = 3.0 * s * dveff[o + d];
          acc += dveff[o + d] * ve[o + d];
        }
        dgate[((size_t)b * T + t) * Hk + h] = 3.0 * s * (1.0 - s) * acc;
      }
    }
}

/* Decode step with a key/value cache: page section "6. 추론 엔진
 * (nanochat/engine.py)", generation with a pre-filled KV cache
 * (flash_attn_with_kvcache). L->T is the cache capacity. Sequence b already
 * holds len[b] tokens: rows 0..len[b]-1 of kc (k~) and vc (v_eff), layout
 * (B, T, Hk, D). Its new token sits at position p = len[b] (< T): the
 * prologue is applied to it at position p, its k~ and v_eff rows are written
 * to the caches at row p, and its query rows attend over cache rows
 * (p - W, p]. q (B, H, D); k, v, ve (B, Hk, D); gate (B, Hk). Outputs
 * O (B, H, D) and lse (B, H), natural log. */
void oracle_decode(const oracle_layer *L, const double *q, const double *k,
                   const double *v, const double *ve, const double *gate,
                   const int *len, double *kc, double *vc, double *O,
                   double *lse) {
  const int B = L->B, T = L->T, H = L->H, Hk = L->Hk, D = L->D;
  const int no_norm = (L->flags & ORACLE_NO_NORM) != 0;
  const int no_rope = (L->flags & ORACLE_NO_ROPE) != 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int b = 0; b < B; ++b) {
    const int p = len[b];
    const double pos = (double)(p + L->pos_offset);
    double n[1024];
    double *qt = (double *)malloc(sizeof(double) * (size_t)H * D);
    double *s = (double *)malloc(sizeof(double) * (size_t)T);
    for (int h = 0; h < H; ++h) {
      rms_norm_row(q + ((size_t)b * H + h) * D, n, D, L->eps, no_norm);
      rope_row(n, qt + (size_t)h * D, D, pos, L->rope_base, 0, no_rope);
    }
    for (int h = 0; h < Hk; ++h) {
      const size_t o = ((size_t)b * Hk + h) * D;
      const size_t c = idx4(b, p, h, 0, T, Hk, D);
      rms_norm_row(k + o, n, D, L->eps, no_norm);
      rope_row(n, kc + c, D, pos, L->rope_base, 0, no_rope);
      double coef = L->has_ve ? 3.0 * sigmoid(gate[(size_t)b * Hk + h]) : 0.0;
      for (int d = 0; d < D; ++d) vc[c + d] = v[o + d] + (L->has_ve ? coef * ve[o + d] : 0.0);
    }
    const int lo = first_key(L, p);
    for (int h = 0; h < H; ++h) {
      const int hk = kv_head(L, h);
      const double *qh = qt + (size_t)h * D;
      double m = -INFINITY;
      for (int j = lo; j <= p; ++j) {
        const double *kj = kc + idx4(b, j, hk, 0, T, Hk, D);
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += qh[d] * kj[d];
        s[j] = L->scale * dot;
        if (s[j] > m) m = s[j];
      }
      double sum = 0.0;
      for (int j = lo; j <= p; ++j) sum += exp(s[j] - m);
      const double l = m + log(sum);
      double *o = O + ((size_t)b * H + h) * D;
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      for (int j = lo; j <= p; ++j) {
        const double pj = exp(s[j] - l);
        const double *vj = vc + idx4(b, j, hk, 0, T, Hk, D);
        for (int d = 0; d < D; ++d) o[d] += pj * vj[d];
      }
      lse[(size_t)b * H + h] = l;
    }
    free(s);
    free(qt);
  }
}

/* The value-embedding gate's projection: page "5만원으로 나만의 ChatGPT
 * 훈련하는 방법", section "1. GPT 모델", value-embedding code: the gate is a
 * linear map (no bias: the page shows none) of the first C channels of the
 * block input x, one output per KV head, before 3*sigmoid(.):
 *   gate[b,t,h] = sum_{c<C} x[b,t,c] w[h,c].
 * x (B, T, ldx) with ldx >= C (only the first C entries of a row are read);
 * w (Hk, C); gate (B, T, Hk). */
void oracle_gate_logits(int B, int T, int Hk, int C, int ldx, const double *x,
                        const double *w, double *gate) {
  for (long n = 0; n < (long)B * T; ++n)
    for (int h = 0; h < Hk; ++h) {
      double s = 0.0;
      for (int c = 0; c < C; ++c) s += x[n * ldx + c] * w[(long)h * C + c];
      gate[n * Hk + h] = s;
    }
}

/* Its backward, given dgate = dL/dgate (B, T, Hk):
 *   dx[b,t,c] = sum_h dgate[b,t,h] w[h,c]   (dx (B, T, C): the first C
 *                                            channels of x; the rest get 0)
 *   dw[h,c]   = sum_{b,t} dgate[b,t,h] x[b,t,c]. */
void oracle_gate_bwd(int B, int T, int Hk, int C, int ldx, const double *x,
                     const double *w, const double *dgate, double *dx,
                     double *dw) {
  for (long n = 0; n < (long)B * T; ++n)
    for (int c = 0; c < C; ++c) {
      double s = 0.0;
      for (int h = 0; h < Hk; ++h) s += dgate[n * Hk + h] * w[(long)h * C + c];
      dx[n * C + c] = s;
    }
  for (int h = 0; h < Hk; ++h)
    for (int c = 0; c < C; ++c) {
      double s = 0.0;
      for (long n = 0; n < (long)B * T; ++n) s += dgate[n * Hk + h] * x[n * ldx + c];
      dw[(long)h * C + c] = s;
    }
}
