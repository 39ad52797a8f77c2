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

struct PreParams {
  long long rows;  // B * T * H
  int T, H;
  const void *O, *dO;
  float* delta;    // (B, H, T)
};

template <typename T, int D>
__global__ void __launch_bounds__(256) preprocess_kernel(const PreParams p) {
  using V = Vec16<T>;
  constexpr int VEC = V::N;
  constexpr int LPR = D / VEC;
  constexpr int RPB = 256 / LPR;  // rows per block pass
  const int sub = threadIdx.x % LPR;
  const long long stride = static_cast<long long>(gridDim.x) * RPB;
  const long long first = static_cast<long long>(blockIdx.x) * RPB + threadIdx.x / LPR;
  // Uniform trip count across the warp.
  const long long warp_first = first - (threadIdx.x % 32) / LPR;
  for (long long base = warp_first; base < p.rows; base += stride) {
    const long long row = base + (threadIdx.x % 32) / LPR;
    const bool valid = row < p.rows;
    float acc = 0.f;
    if (valid) {
      float o[VEC], g[VEC];
      V::load(static_cast<const T*>(p.O) + row * D + sub * VEC, o);
      V::load(static_cast<const T*>(p.dO) + row * D + sub * VEC, g);
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc = fmaf(o[i], g[i], acc);
    }
#pragma unroll
    for (int off = LPR / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off, LPR);
    if (valid && sub == 0) {
      // row = (b*T + t)*H + h  ->  delta[(b*H + h)*T + t]
      const long long h = row % p.H;
      const long long bt = row / p.H;
      const long long t = bt % p.T, b = bt / p.T;
      p.delta[(b * p.H + h) * p.T + t] = acc;
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

  for (int base = 0; base < total_rows; base += ROWS_PER_PASS) {
    const int r = base + grp;
    const bool in_range = r < total_rows;
    const int rr = in_range ? r : 0;
    const int tt = rr / rows_per_tok;
    const int kind_row = rr % rows_per_tok;
    const long long tok = tok0 + tt;
    const bool valid = in_range && tok < n_tok;
    const long long tk = valid ? tok : 0;
    const int t = static_cast<int>(tk % p.T);
    const long long b = tk / p.T;
    int kind, head, nheads;
    if (kind_row < p.H) {
      kind = 0; head = kind_row; nheads = p.H;
    } else if (kind_row < p.H + p.Hk) {
      kind = 1; head = kind_row - p.H; nheads = p.Hk;
    } else {
      kind = 2; head = kind_row - p.H - p.Hk; nheads = p.Hk;
    }
    const size_t row = static_cast<size_t>(tk) * nheads + head;  // (b,t,head)
    const size_t off = row * D + static_cast<size_t>(sub) * VEC;

    // Gradient w.r.t. the rotated, normalised row (or dv_eff for kind 2).
    float dy[VEC];
    if (valid) {
      const float* src;
      if (kind == 0)
        src = p.dq_acc + ((static_cast<size_t>(b) * p.H + head) * p.T + t) * D + sub * VEC;
      else
        src = (kind == 1 ? p.dk_acc : p.dv_acc) + off;
      load_f32<VEC>(src, dy);
    } else {
#pragma unroll
      for (int i = 0; i < VEC; ++i) dy[i] = 0.f;
    }

    // RoPE^-1 (the transpose rotation).
    float dn[VEC];
    if constexpr (LPR >= 2) {
      float partner[VEC];
#pragma unroll
      for (int i = 0; i < VEC; ++i) partner[i] = __shfl_xor_sync(0xffffffffu, dy[i], LPR / 2, LPR);
      const bool lower = sub < LPR / 2;
      const int pair0 = (lower ? sub : sub - LPR / 2) * VEC;
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        const float c = s_cos[tt][pair0 + i], s = s_sin[tt][pair0 + i];
        // lower: dy_i c + dy_{i+D/2} s ; upper: -dy_{i-D/2} s + dy_i c
        dn[i] = lower ? fmaf(dy[i], c, partner[i] * s) : fmaf(-partner[i], s, dy[i] * c);
      }
    } else {
#pragma unroll
      for (int i = 0; i < HALF; ++i) {
        const float c = s_cos[tt][i], s = s_sin[tt][i];
        dn[i] = fmaf(dy[i], c, dy[i + HALF] * s);
        dn[i + HALF] = fmaf(-dy[i], s, dy[i + HALF] * c);
      }
    }

    // RMSNorm backward: dx = r (dn - n mean(dn * n)), n = r x.
    float x[VEC];
    float rs = 0.f;
    if (valid && kind != 2) {
      V::load(static_cast<const T*>(kind == 0 ? p.q : p.k) + off, x);
      rs = (kind == 0 ? p.rstd_q : p.rstd_k)[row];
    } else {
#pragma unroll
      for (int i = 0; i < VEC; ++i) x[i] = 0.f;
    }
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < VEC; ++i) dot = fmaf(dn[i], x[i] * rs, dot);
#pragma unroll
    for (int o = LPR / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o, LPR);
    dot /= static_cast<float>(D);

    // Value side: dgate reduction (all lanes take part).
    float ve[VEC];
    float coef = 0.f, dg = 0.f;
    if (valid && kind == 2 && p.has_ve) {
      V::load(static_cast<const T*>(p.ve) + off, ve);
      const float s = 1.0f / (1.0f + expf(-V::scalar(p.gate, row)));
      coef = 3.0f * s;
#pragma unroll
      for (int i = 0; i < VEC; ++i) dg = fmaf(dy[i], ve[i], dg);
      dg *= coef * (1.0f - s);
    }
#pragma unroll
    for (int o = LPR / 2; o >= 1; o >>= 1) dg += __shfl_xor_sync(0xffffffffu, dg, o, LPR);

    if (!valid) continue;
    if (kind == 2) {
      V::store(static_cast<T*>(p.dv) + off, dy);
      if (p.has_ve) {
        float o[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i) o[i] = coef * dy[i];
        V::store(static_cast<T*>(p.dve) + off, o);
        if (sub == 0) {
          if constexpr (sizeof(T) == 2)
            static_cast<__nv_bfloat16*>(p.dgate)[row] = __float2bfloat16_rn(dg);
          else
            static_cast<float*>(p.dgate)[row] = dg;
        }
      }
    } else {
      float o[VEC];
#pragma unroll
      for (int i = 0; i < VEC; ++i) o[i] = rs * (dn[i] - x[i] * rs * dot);
      V::store(static_cast<T*>(kind == 0 ? p.dq : p.dk) + off, o);
    }
  }
}

}  // namespace cswattn
