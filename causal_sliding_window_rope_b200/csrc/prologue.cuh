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
// elements is owned by LPR = D / (2 HV) lanes; lane l holds the HV-element
// slices [l HV, (l+1) HV) of both halves of the row (elements i and
// i + D/2), so every RoPE pair is inside one lane and each lane keeps two
// vector loads in flight per row. Loads and stores are coalesced vector
// accesses; the RMS is a shuffle reduction over the row's LPR lanes.
#pragma once
#include "common.cuh"

namespace cswattn {

constexpr int kPrologueThreads = 256;
constexpr int kPrologueTok = 8;
constexpr int kMaxHalfD = 64;

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

// HV consecutive elements of type T <-> float[HV], as one vector access
// (16, 8 or 4 bytes).
template <typename T, int HV>
struct HalfVec;
template <>
struct HalfVec<__nv_bfloat16, 8> {
  __device__ static void load(const __nv_bfloat16* p, float (&x)[8]) { Vec16<__nv_bfloat16>::load(p, x); }
  __device__ static void store(__nv_bfloat16* p, const float (&x)[8]) { Vec16<__nv_bfloat16>::store(p, x); }
};
template <>
struct HalfVec<float, 4> {
  __device__ static void load(const float* p, float (&x)[4]) { Vec16<float>::load(p, x); }
  __device__ static void store(float* p, const float (&x)[4]) { Vec16<float>::store(p, x); }
};
template <>
struct HalfVec<float, 2> {
  __device__ static void load(const float* p, float (&x)[2]) {
    const float2 u = *reinterpret_cast<const float2*>(p);
    x[0] = u.x;
    x[1] = u.y;
  }
  __device__ static void store(float* p, const float (&x)[2]) {
    *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
  }
};

// Row geometry of the split-halves layout for element type T and width D.
template <typename T, int D>
struct RowLayout {
  static constexpr int HALF = D / 2;
  static constexpr int HV = (16 / static_cast<int>(sizeof(T))) < HALF ? 16 / static_cast<int>(sizeof(T)) : HALF;
  static constexpr int LPR = HALF / HV;  // lanes per row
  static_assert(HALF % HV == 0 && LPR >= 1 && LPR <= 32 && (LPR & (LPR - 1)) == 0, "row layout");
};

// Sum over the LPR lanes of a row (xor shuffles within the row's lane group).
template <int LPR>
__device__ __forceinline__ float row_sum(float v) {
#pragma unroll
  for (int o = LPR / 2; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o, LPR);
  return v;
}

// Per-CTA token table of the row kernels: the CTA's kPrologueTok consecutive
// tokens (b, t), and cos/sin(t * omega_i) for each of them.
template <int HALF>
struct TokenTable {
  float cos_[kPrologueTok][HALF];
  float sin_[kPrologueTok][HALF];
  int b[kPrologueTok], t[kPrologueTok];
  bool valid[kPrologueTok];

  __device__ void fill(long long tok0, long long n_tok, int T, const float* omega) {
    if (threadIdx.x < kPrologueTok) {
      const long long tok = tok0 + threadIdx.x;
      valid[threadIdx.x] = tok < n_tok;
      const long long tk = tok < n_tok ? tok : 0;
      b[threadIdx.x] = static_cast<int>(tk / T);
      t[threadIdx.x] = static_cast<int>(tk % T);
    }
    for (int e = threadIdx.x; e < kPrologueTok * HALF; e += blockDim.x) {
      const int tt = e / HALF, i = e % HALF;
      const long long tok = tok0 + tt;
      const int t_ = tok < n_tok ? static_cast<int>(tok % T) : 0;
      float sn, cs;
      sincosf(static_cast<float>(t_) * omega[i], &sn, &cs);
      cos_[tt][i] = cs;
      sin_[tt][i] = sn;
    }
  }
  // cos and sin of the VEC consecutive pairs starting at pair0 (16-byte loads).
  template <int VEC>
  __device__ void load(int tt, int pair0, float (&c)[VEC], float (&s)[VEC]) const {
    if constexpr (VEC % 4 == 0) {
#pragma unroll
      for (int i = 0; i < VEC; i += 4) {
        const float4 c4 = *reinterpret_cast<const float4*>(&cos_[tt][pair0 + i]);
        const float4 s4 = *reinterpret_cast<const float4*>(&sin_[tt][pair0 + i]);
        c[i] = c4.x; c[i + 1] = c4.y; c[i + 2] = c4.z; c[i + 3] = c4.w;
        s[i] = s4.x; s[i + 1] = s4.y; s[i + 2] = s4.z; s[i + 3] = s4.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        c[i] = cos_[tt][pair0 + i];
        s[i] = sin_[tt][pair0 + i];
      }
    }
  }
};

// Division-free walk over the rows (token tt, row kind_row) of a CTA: each
// lane group advances by a fixed stride per pass.
struct RowCursor {
  int tt, kind_row;
  __device__ void advance(int by, int rows_per_tok) {
    kind_row += by;
    while (kind_row >= rows_per_tok) {
      kind_row -= rows_per_tok;
      ++tt;
    }
  }
};

template <typename T, int D>
__global__ void __launch_bounds__(kPrologueThreads)
    prologue_kernel(const PrologueParams p) {
  using RL = RowLayout<T, D>;
  using HVec = HalfVec<T, RL::HV>;
  constexpr int HV = RL::HV, LPR = RL::LPR, HALF = RL::HALF;
  constexpr int ROWS_PER_PASS = kPrologueThreads / LPR;

  __shared__ __align__(16) TokenTable<HALF> tab;

  const long long n_tok = static_cast<long long>(p.B) * p.T;
  const long long tok0 = static_cast<long long>(blockIdx.x) * kPrologueTok;
  tab.fill(tok0, n_tok, p.T, p.omega);
  __syncthreads();

  const int rows_per_tok = p.H + 2 * p.Hk;
  const int total_rows = kPrologueTok * rows_per_tok;
  const int sub = threadIdx.x % LPR;  // lane within the row group
  const int grp = threadIdx.x / LPR;  // row group within the CTA
  RowCursor cur{0, 0};
  cur.advance(grp, rows_per_tok);

  // Uniform trip count: every lane takes part in every shuffle.
  for (int base = 0; base < total_rows; base += ROWS_PER_PASS) {
    const bool in_range = base + grp < total_rows;
    const int tt = in_range ? cur.tt : 0;
    const int kind_row = in_range ? cur.kind_row : 0;
    cur.advance(ROWS_PER_PASS, rows_per_tok);
    const bool valid = in_range && tab.valid[tt];
    // Row kinds: [0, H) query heads, [H, H+Hk) key heads, then value heads.
    int kind, head, nheads;
    if (kind_row < p.H) {
      kind = 0; head = kind_row; nheads = p.H;
    } else if (kind_row < p.H + p.Hk) {
      kind = 1; head = kind_row - p.H; nheads = p.Hk;
    } else {
      kind = 2; head = kind_row - p.H - p.Hk; nheads = p.Hk;
    }
    const size_t row = static_cast<size_t>(valid ? tok0 + tt : 0) * nheads + head;
    const size_t off_lo = row * D + static_cast<size_t>(sub) * HV;
    const size_t off_hi = off_lo + HALF;
    const T* src = static_cast<const T*>(kind == 0 ? p.q : (kind == 1 ? p.k : p.v));
    float xl[HV], xh[HV], el[HV], eh[HV];
    float gl = 0.f;
    if (valid) {
      HVec::load(src + off_lo, xl);
      HVec::load(src + off_hi, xh);
    } else {
#pragma unroll
      for (int i = 0; i < HV; ++i) xl[i] = xh[i] = 0.f;
    }
    const bool has_e = valid && kind == 2 && p.has_ve;
    if (has_e) {
      HVec::load(static_cast<const T*>(p.ve) + off_lo, el);
      HVec::load(static_cast<const T*>(p.ve) + off_hi, eh);
      gl = Vec16<T>::scalar(p.gate, row);
    } else {
#pragma unroll
      for (int i = 0; i < HV; ++i) el[i] = eh[i] = 0.f;
    }

    // RMSNorm: mean of squares over the row (shuffle reduction over its lanes).
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < HV; ++i) ss = fmaf(xl[i], xl[i], fmaf(xh[i], xh[i], ss));
    ss = row_sum<LPR>(ss);
    const float rstd = rsqrtf(ss / static_cast<float>(D) + p.eps);
    if (!valid) continue;

    if (kind == 2) {
      // Value residual: v + 3 sigmoid(gate) ve.
      const float coef = has_e ? 3.0f / (1.0f + expf(-gl)) : 0.f;
#pragma unroll
      for (int i = 0; i < HV; ++i) {
        xl[i] = fmaf(coef, el[i], xl[i]);
        xh[i] = fmaf(coef, eh[i], xh[i]);
      }
      HVec::store(static_cast<T*>(p.v_out) + off_lo, xl);
      HVec::store(static_cast<T*>(p.v_out) + off_hi, xh);
      continue;
    }
    // RoPE on the pairs (i, i + D/2) held by this lane.
    float cv[HV], sv[HV], yl[HV], yh[HV];
    tab.template load<HV>(tt, sub * HV, cv, sv);
#pragma unroll
    for (int i = 0; i < HV; ++i) {
      const float nl = xl[i] * rstd, nh = xh[i] * rstd;
      yl[i] = fmaf(nl, cv[i], -nh * sv[i]);
      yh[i] = fmaf(nl, sv[i], nh * cv[i]);
    }
    T* dst = static_cast<T*>(kind == 0 ? p.q_out : p.k_out);
    HVec::store(dst + off_lo, yl);
    HVec::store(dst + off_hi, yh);
    if (sub == 0) (kind == 0 ? p.rstd_q : p.rstd_k)[row] = rstd;
  }
}

}  // namespace cswattn
