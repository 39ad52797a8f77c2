// prologue.cuh -- fused QK RMSNorm + RoPE + value-embedding residual.
//
// Page "5만원으로 나만의 ChatGPT 훈련하는 방법", section "1. GPT 모델
// (nanochat/gpt.py)": the architecture list (RoPE, QK normalisation) and the
// value-embedding code (v + 3*sigmoid(gate)*ve, one gate per token and KV
// head, broadcast over head_dim).
//
// One CTA handles kTok consecutive tokens (b, t). It first computes
// cos/sin(t * omega_i) for its tokens into shared memory, then walks the
// H query rows, Hk key rows and Hk value rows of each token. A row of D
// elements is owned by LPR = D / VEC lanes, each holding one 16-byte vector,
// so every load and store is a coalesced 16-byte access. The RMS is a
// shuffle reduction over the row's lanes; the RoPE partner of element i
// (i +- D/2) sits in lane (lane ^ LPR/2) at the same vector slot.
#pragma once
#include "common.cuh"

namespace cswattn {

constexpr int kPrologueThreads = 256;
constexpr int kPrologueTok = 8;
constexpr int kMaxHalfD = 64;
#ifndef CSW_ROWS_IN_FLIGHT
#define CSW_ROWS_IN_FLIGHT 1
#endif
// Rows each lane loads before computing, in the HBM-bound row kernels.
constexpr int kRowsInFlight = CSW_ROWS_IN_FLIGHT;

struct PrologueParams {
  int B, T, H, Hk;
  int has_ve;
  float eps;
  float omega[kMaxHalfD];  // rope_base^(-2i/D), i < D/2, rounded from double
  const void *q, *k, *v, *ve, *gate;
  void *q_out, *k_out, *v_out;
  float *rstd_q, *rstd_k;
};

template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const void* p, float (&x)[N]) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
  __device__ static void store(void* p, const float (&x)[N]) {
    uint4 u;
    uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = u;
  }
  __device__ static float scalar(const void* p, size_t i) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  }
};
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ static void load(const void* p, float (&x)[N]) {
    float4 u = *reinterpret_cast<const float4*>(p);
    x[0] = u.x;
    x[1] = u.y;
    x[2] = u.z;
    x[3] = u.w;
  }
  __device__ static void store(void* p, const float (&x)[N]) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
  __device__ static float scalar(const void* p, size_t i) {
    return reinterpret_cast<const float*>(p)[i];
  }
};

template <typename T, int D>
__global__ void __launch_bounds__(kPrologueThreads)
    prologue_kernel(const PrologueParams p) {
  using V = Vec16<T>;
  constexpr int VEC = V::N;
  static_assert(D % VEC == 0, "head_dim must be a multiple of the vector width");
  constexpr int LPR = D / VEC;          // lanes per row
  static_assert(LPR >= 1 && LPR <= 32 && (LPR & (LPR - 1)) == 0, "lanes per row");
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
  const int sub = threadIdx.x % LPR;        // lane within the row group
  const int grp = threadIdx.x / LPR;        // row group within the CTA

  // kRowsInFlight rows per lane per pass: all loads of a pass are issued
  // before any arithmetic, so each lane keeps several 16-byte loads in
  // flight. Uniform trip count: every lane takes part in every shuffle.
  constexpr int U = kRowsInFlight;
  for (int base = 0; base < total_rows; base += ROWS_PER_PASS * U) {
    float x[U][VEC], e[U][VEC];
    float gl[U];
    int kind[U];
    bool valid[U];
    size_t row[U], off[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = base + u * ROWS_PER_PASS + grp;
      const bool in_range = r < total_rows;
      const int rr = in_range ? r : 0;
      const int tt = rr / rows_per_tok;
      const int kind_row = rr % rows_per_tok;
      const long long tok = tok0 + tt;
      valid[u] = in_range && tok < n_tok;
      // Row kinds: [0, H) query heads, [H, H+Hk) key heads, then value heads.
      int head, nheads;
      if (kind_row < p.H) {
        kind[u] = 0; head = kind_row; nheads = p.H;
      } else if (kind_row < p.H + p.Hk) {
        kind[u] = 1; head = kind_row - p.H; nheads = p.Hk;
      } else {
        kind[u] = 2; head = kind_row - p.H - p.Hk; nheads = p.Hk;
      }
      row[u] = static_cast<size_t>(valid[u] ? tok : 0) * nheads + head;
      off[u] = row[u] * D + static_cast<size_t>(sub) * VEC;
      const void* src = kind[u] == 0 ? p.q : (kind[u] == 1 ? p.k : p.v);
      if (valid[u]) {
        V::load(static_cast<const T*>(src) + off[u], x[u]);
      } else {
#pragma unroll
        for (int i = 0; i < VEC; ++i) x[u][i] = 0.f;
      }
      gl[u] = 0.f;
      if (valid[u] && kind[u] == 2 && p.has_ve) {
        V::load(static_cast<const T*>(p.ve) + off[u], e[u]);
        gl[u] = V::scalar(p.gate, row[u]);
      } else {
#pragma unroll
        for (int i = 0; i < VEC; ++i) e[u][i] = 0.f;
      }
    }

#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = base + u * ROWS_PER_PASS + grp;
      const int tt = (r < total_rows ? r : 0) / rows_per_tok;
      // RMSNorm: mean of squares over the row's LPR lanes (shuffle reduction).
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < VEC; ++i) ss = fmaf(x[u][i], x[u][i], ss);
#pragma unroll
      for (int o = LPR / 2; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o, LPR);
      const float rstd = rsqrtf(ss / static_cast<float>(D) + p.eps);
      float n[VEC];
#pragma unroll
      for (int i = 0; i < VEC; ++i) n[i] = x[u][i] * rstd;

      // RoPE on half-split pairs (i, i + D/2).
      float y[VEC];
      if constexpr (LPR >= 2) {
        float partner[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i)
          partner[i] = __shfl_xor_sync(0xffffffffu, n[i], LPR / 2, LPR);
        const bool lower = sub < LPR / 2;
        const int pair0 = (lower ? sub : sub - LPR / 2) * VEC;
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
          const float c = s_cos[tt][pair0 + i], s = s_sin[tt][pair0 + i];
          // lower half: x_i c - x_{i+D/2} s ; upper half: x_{i-D/2} s + x_i c
          y[i] = lower ? fmaf(n[i], c, -partner[i] * s) : fmaf(partner[i], s, n[i] * c);
        }
      } else {
#pragma unroll
        for (int i = 0; i < HALF; ++i) {
          const float c = s_cos[tt][i], s = s_sin[tt][i];
          y[i] = fmaf(n[i], c, -n[i + HALF] * s);
          y[i + HALF] = fmaf(n[i], s, n[i + HALF] * c);
        }
      }
      if (!valid[u]) continue;

      if (kind[u] == 2) {
        // Value residual: v + 3 sigmoid(gate) ve (e = 0 without ve).
        const float coef = p.has_ve ? 3.0f / (1.0f + expf(-gl[u])) : 0.f;
        float vv[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i) vv[i] = fmaf(coef, e[u][i], x[u][i]);
        V::store(static_cast<T*>(p.v_out) + off[u], vv);
      } else {
        V::store(static_cast<T*>(kind[u] == 0 ? p.q_out : p.k_out) + off[u], y);
        if (sub == 0) (kind[u] == 0 ? p.rstd_q : p.rstd_k)[row[u]] = rstd;
      }
    }
  }
}

}  // namespace cswattn
