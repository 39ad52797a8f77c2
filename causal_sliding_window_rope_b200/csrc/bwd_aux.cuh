// bwd_aux.cuh -- the backward's HBM-bound helpers.
//
// preprocess: Delta_i = dO_i . O_i per (b, h, t), the row term of the
//   softmax backward (ds_ij = p_ij (dp_ij - Delta_i)).
// epilogue: the chain rule back through the prologue (page section
//   "1. GPT 모델": RoPE, QK normalisation, value-embedding code):
//   dq = RMSNorm'(RoPE^-1(dq~)), dk likewise, dv = dv_eff,
//   dve = 3 s dv_eff, dgate = 3 s (1 - s) sum_d dv_eff ve with s = sigmoid(gate).
// Both use the prologue's row layout: a row of D elements is owned by
// D / VEC lanes holding one 16-byte vector each; reductions are shuffles.
#pragma once
#include "prologue.cuh"

namespace cswattn {

// Row terms of the backward, in the padded layout (B, H, Tpad) with Tpad a
// multiple of 64: delta = dO.O and lse2 = lse * log2(e); past T, delta = 0
// and lse2 = +inf (so exp2(s - lse2) = 0 for padding queries).
struct PreParams {
  long long rows;  // B * T * H
  int T, H, Tpad;
  const void *O, *dO;
  const float* lse;  // (B, H, T)
  float* delta;      // (B, H, Tpad)
  float* lse2;       // (B, H, Tpad)
};

template <typename T, int D>
__global__ void __launch_bounds__(256) preprocess_kernel(const PreParams p) {
  using V = Vec16<T>;
  constexpr int VEC = V::N;
  constexpr int LPR = D / VEC;
  constexpr int RPW = 32 / LPR;           // rows per warp per slot
  constexpr int U = kRowsInFlight;        // slots per pass
  const int sub = threadIdx.x % LPR;
  const int lrow = (threadIdx.x % 32) / LPR;
  const long long warp_global = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) / 32;
  const long long n_warps = static_cast<long long>(gridDim.x) * 8;
  // Uniform trip count across the warp; U rows' loads in flight per lane.
  for (long long base = warp_global * RPW * U; base < p.rows; base += n_warps * RPW * U) {
    float o[U][VEC], g[U][VEC];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long row = base + u * RPW + lrow;
      if (row < p.rows) {
        V::load(static_cast<const T*>(p.O) + row * D + sub * VEC, o[u]);
        V::load(static_cast<const T*>(p.dO) + row * D + sub * VEC, g[u]);
      } else {
#pragma unroll
        for (int i = 0; i < VEC; ++i) o[u][i] = g[u][i] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long row = base + u * RPW + lrow;
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc = fmaf(o[u][i], g[u][i], acc);
#pragma unroll
      for (int off = LPR / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off, LPR);
      if (row < p.rows && sub == 0) {
        // row = (b*T + t)*H + h  ->  (b*H + h)*Tpad + t
        const long long h = row % p.H;
        const long long bt = row / p.H;
        const long long t = bt % p.T, b = bt / p.T;
        const long long o = (b * p.H + h) * p.Tpad;
        p.delta[o + t] = acc;
        p.lse2[o + t] = p.lse[(b * p.H + h) * p.T + t] * 1.4426950408889634f;
        if (t == p.T - 1) {
          for (long long tp = p.T; tp < p.Tpad; ++tp) {
            p.delta[o + tp] = 0.f;
            p.lse2[o + tp] = INFINITY;
          }
        }
      }
    }
  }
}

struct EpiParams {
  int B, T, H, Hk;
  int has_ve;
  float omega[kMaxHalfD];
  const void *q, *k, *ve, *gate;        // prologue inputs (layer dtype)
  const float *rstd_q, *rstd_k;
  const float* dq_acc;                  // (B,H,T,D) dq~ (scaled)
  const float *dk_acc, *dv_acc;         // (B,T,Hk,D) dk~ (scaled), dv_eff
  void *dq, *dk, *dv, *dve, *dgate;     // outputs (layer dtype)
};

template <int VEC>
__device__ __forceinline__ void load_f32(const float* src, float (&x)[VEC]) {
#pragma unroll
  for (int i = 0; i < VEC; i += 4) {
    float4 u = *reinterpret_cast<const float4*>(src + i);
    x[i] = u.x;
    x[i + 1] = u.y;
    x[i + 2] = u.z;
    x[i + 3] = u.w;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kPrologueThreads) epilogue_kernel(const EpiParams p) {
  using V = Vec16<T>;
  constexpr int VEC = V::N;
  constexpr int LPR = D / VEC;
  constexpr int HALF = D / 2;
  constexpr int ROWS_PER_PASS = kPrologueThreads / LPR;

  __shared__ float s_cos[kPrologueTok][HALF];
  __shared__ float s_sin[kPrologueTok][HALF];

  const long long n_tok = static_cast<long long>(p.B) * p.T;
  const long long tok0 = static_cast<long long>(blockIdx.x) * kPrologueTok;
  for (int e = threadIdx.x; e < kPrologueTok * HALF; e += kPrologueThreads) {
    const int tt = e / HALF, i = e % HALF;
    const long long tok = tok0 + tt;
    const int t = tok < n_tok ? static_cast<int>(tok % p.T) : 0;
    float s, c;
    sincosf(static_cast<float>(t) * p.omega[i], &s, &c);
    s_cos[tt][i] = c;
    s_sin[tt][i] = s;
  }
  __syncthreads();

  const int rows_per_tok = p.H + 2 * p.Hk;
  const int total_rows = kPrologueTok * rows_per_tok;
  const int sub = threadIdx.x % LPR;
  const int grp = threadIdx.x / LPR;

  // Like the prologue: U rows per lane per pass, loads first.
  constexpr int U = kRowsInFlight;
  for (int base = 0; base < total_rows; base += ROWS_PER_PASS * U) {
    float dy[U][VEC], x[U][VEC];
    float rs[U], gl[U];
    int kind[U], tt[U];
    bool valid[U];
    size_t row[U], off[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = base + u * ROWS_PER_PASS + grp;
      const bool in_range = r < total_rows;
      const int rr = in_range ? r : 0;
      tt[u] = rr / rows_per_tok;
      const int kind_row = rr % rows_per_tok;
      const long long tok = tok0 + tt[u];
      valid[u] = in_range && tok < n_tok;
      const long long tk = valid[u] ? tok : 0;
      const int t = static_cast<int>(tk % p.T);
      const long long b = tk / p.T;
      int head, nheads;
      if (kind_row < p.H) {
        kind[u] = 0; head = kind_row; nheads = p.H;
      } else if (kind_row < p.H + p.Hk) {
        kind[u] = 1; head = kind_row - p.H; nheads = p.Hk;
      } else {
        kind[u] = 2; head = kind_row - p.H - p.Hk; nheads = p.Hk;
      }
      row[u] = static_cast<size_t>(tk) * nheads + head;  // (b,t,head)
      off[u] = row[u] * D + static_cast<size_t>(sub) * VEC;
      rs[u] = 0.f;
      gl[u] = 0.f;
      if (valid[u]) {
        // Gradient w.r.t. the rotated, normalised row (or dv_eff for kind 2).
        const float* src;
        if (kind[u] == 0)
          src = p.dq_acc + ((static_cast<size_t>(b) * p.H + head) * p.T + t) * D + sub * VEC;
        else
          src = (kind[u] == 1 ? p.dk_acc : p.dv_acc) + off[u];
        load_f32<VEC>(src, dy[u]);
        if (kind[u] != 2) {
          V::load(static_cast<const T*>(kind[u] == 0 ? p.q : p.k) + off[u], x[u]);
          rs[u] = (kind[u] == 0 ? p.rstd_q : p.rstd_k)[row[u]];
        } else if (p.has_ve) {
          V::load(static_cast<const T*>(p.ve) + off[u], x[u]);  // ve for the value rows
          gl[u] = V::scalar(p.gate, row[u]);
        } else {
#pragma unroll
          for (int i = 0; i < VEC; ++i) x[u][i] = 0.f;
        }
      } else {
#pragma unroll
        for (int i = 0; i < VEC; ++i) dy[u][i] = x[u][i] = 0.f;
      }
    }

#pragma unroll
    for (int u = 0; u < U; ++u) {
      // RoPE^-1 (the transpose rotation).
      float dn[VEC];
      if constexpr (LPR >= 2) {
        float partner[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i)
          partner[i] = __shfl_xor_sync(0xffffffffu, dy[u][i], LPR / 2, LPR);
        const bool lower = sub < LPR / 2;
        const int pair0 = (lower ? sub : sub - LPR / 2) * VEC;
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
          const float c = s_cos[tt[u]][pair0 + i], s = s_sin[tt[u]][pair0 + i];
          // lower: dy_i c + dy_{i+D/2} s ; upper: -dy_{i-D/2} s + dy_i c
          dn[i] = lower ? fmaf(dy[u][i], c, partner[i] * s) : fmaf(-partner[i], s, dy[u][i] * c);
        }
      } else {
#pragma unroll
        for (int i = 0; i < HALF; ++i) {
          const float c = s_cos[tt[u]][i], s = s_sin[tt[u]][i];
          dn[i] = fmaf(dy[u][i], c, dy[u][i + HALF] * s);
          dn[i + HALF] = fmaf(-dy[u][i], s, dy[u][i + HALF] * c);
        }
      }
      // One shuffle reduction serves both row kinds: for q/k rows the
      // RMSNorm term sum_d dn*n (n = r x); for value rows sum_d dv_eff*ve.
      const bool vrow = kind[u] == 2;
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < VEC; ++i)
        dot = vrow ? fmaf(dy[u][i], x[u][i], dot) : fmaf(dn[i], x[u][i] * rs[u], dot);
#pragma unroll
      for (int o = LPR / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o, LPR);
      if (!valid[u]) continue;
      if (vrow) {
        V::store(static_cast<T*>(p.dv) + off[u], dy[u]);
        if (p.has_ve) {
          const float sg = 1.0f / (1.0f + expf(-gl[u]));
          const float coef = 3.0f * sg;
          float o[VEC];
#pragma unroll
          for (int i = 0; i < VEC; ++i) o[i] = coef * dy[u][i];
          V::store(static_cast<T*>(p.dve) + off[u], o);
          if (sub == 0) {
            const float dg = dot * coef * (1.0f - sg);
            if constexpr (sizeof(T) == 2)
              static_cast<__nv_bfloat16*>(p.dgate)[row[u]] = __float2bfloat16_rn(dg);
            else
              static_cast<float*>(p.dgate)[row[u]] = dg;
          }
        }
      } else {
        // RMSNorm backward: dx = r (dn - n mean(dn * n)), n = r x.
        const float mean = dot / static_cast<float>(D);
        float o[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i) o[i] = rs[u] * (dn[i] - x[u][i] * rs[u] * mean);
        V::store(static_cast<T*>(kind[u] == 0 ? p.dq : p.dk) + off[u], o);
      }
    }
  }
}

}  // namespace cswattn
