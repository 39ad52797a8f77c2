// prologue.cuh -- fused QK RMSNorm + RoPE + value-embedding residual.
//
// Page "5만원으로 나만의 ChatGPT 훈련하는 방법", section "1. GPT 모델
// (nanochat/gpt.py)": the architecture list (RoPE, QK normalisation) and the
// value-embedding code (v + 3*sigmoid(gate)*ve, one gate per token and KV
// head, broadcast over head_dim).
//
// One CTA handles `tok` consecutive tokens (b, t). The row kernels are bound
// by HBM bandwidth and are short (tens of microseconds), so what matters is
// how many bytes are in flight from the start: the CTA computes
// cos/sin(t omega_i) for its tokens into shared memory (which needs no
// global memory, so it overlaps the previous kernel's tail under
// programmatic launch), then in the staged form thread 0 issues one bulk
// copy (cp.async.bulk) per input tensor for the whole token block and the
// rows are read from shared memory once they have landed. (The direct form
// reads global memory row by row; it serves layers whose token block does
// not fit in shared memory.)
//
// A row of D elements is owned by LPR = D / (2 HV) lanes; lane l holds the
// HV-element slices [l HV, (l+1) HV) of both halves of the row (elements i
// and i + D/2), so every RoPE pair is inside one lane. The RMS is a shuffle
// reduction over the row's LPR lanes; results go to global memory as
// coalesced vector stores.
#pragma once
#include "common.cuh"

namespace cswattn {

constexpr int kPrologueThreads = 256;
constexpr int kPrologueTok = 8;   // most tokens per CTA
constexpr int kMaxHalfD = 64;

struct PrologueParams {
  int B, T, H, Hk;
  int has_ve;
  int tok;                  // tokens per CTA (1..kPrologueTok)
  unsigned long long wait_ns;  // bound of the staging wait
  float eps;
  float omega[kMaxHalfD];  // rope_base^(-2i/D), i < D/2, rounded from double
  const void *q, *k, *v, *ve, *gate;
  void *q_out, *k_out, *v_out;
  float *rstd_q, *rstd_k;
  // Gate from the block input instead of given logits (xg non-null): the
  // logits are x[b,t,:gc] . w_gate[h,:], rounded to the layer dtype and
  // written to gate_out (B,T,Hk) for the backward.
  const void* xg;        // (B,T,x_stride) block input, layer dtype
  long long x_stride;    // elements between consecutive tokens of xg
  int gc;                // gate channels C (the first C entries of a row)
  const void* w_gate;    // (Hk, C), layer dtype
  void* gate_out;        // (B,T,Hk), layer dtype
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

// Per-CTA token table of the row kernels: the CTA's ntt (at most
// kPrologueTok) consecutive tokens (b, t), and cos/sin(t * omega_i) for each.
// A lane reads the HV pairs sub*HV .. sub*HV + HV - 1 as 16-byte chunks;
// with HV a multiple of 4 the pairs are stored chunk-major (chunk q of every
// lane, then chunk q + 1), so the lanes of a quarter warp read one
// contiguous 128-byte span (no bank conflicts).
template <int HALF, int HV>
struct TokenTable {
  static constexpr bool kChunked = HV % 4 == 0;
  float cos_[kPrologueTok][HALF];
  float sin_[kPrologueTok][HALF];
  int b[kPrologueTok], t[kPrologueTok];

  __device__ static int pos(int i) {
    if constexpr (kChunked) return (((i % HV) >> 2) * (HALF / HV) + i / HV) * 4 + (i & 3);
    else return i;
  }

  // Tokens tok0 .. tok0 + ntt - 1, all of them below B*T.
  __device__ void fill(long long tok0, int T, const float* omega, int ntt) {
    if (threadIdx.x < ntt) {
      const long long tok = tok0 + threadIdx.x;
      b[threadIdx.x] = static_cast<int>(tok / T);
      t[threadIdx.x] = static_cast<int>(tok % T);
    }
    for (int e = threadIdx.x; e < ntt * HALF; e += blockDim.x) {
      const int tt = e / HALF, i = e % HALF;
      const int t_ = static_cast<int>((tok0 + tt) % T);
      float sn, cs;
      sincosf(static_cast<float>(t_) * omega[i], &sn, &cs);
      cos_[tt][pos(i)] = cs;
      sin_[tt][pos(i)] = sn;
    }
  }
  // cos and sin of the HV consecutive pairs starting at pair0 = sub * HV.
  __device__ void load(int tt, int pair0, float (&c)[HV], float (&s)[HV]) const {
    if constexpr (kChunked) {
#pragma unroll
      for (int q = 0; q < HV / 4; ++q) {
        const int at = (q * (HALF / HV) + pair0 / HV) * 4;
        const float4 c4 = *reinterpret_cast<const float4*>(&cos_[tt][at]);
        const float4 s4 = *reinterpret_cast<const float4*>(&sin_[tt][at]);
        c[4 * q] = c4.x; c[4 * q + 1] = c4.y; c[4 * q + 2] = c4.z; c[4 * q + 3] = c4.w;
        s[4 * q] = s4.x; s[4 * q + 1] = s4.y; s[4 * q + 2] = s4.z; s[4 * q + 3] = s4.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < HV; ++i) {
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

// Staging of one CTA's token block into shared memory: thread 0 arms the
// barrier with the block's byte count and issues the bulk copies; every
// thread later waits for the bytes (bounded; a timeout is recorded in the
// status word and the CTA computes nothing).
struct Stage {
  uint64_t* bar;
  __device__ void arm(uint32_t bytes) const {
    mbar_init(bar, 1);
    fence_barrier_init();
    fence_proxy_async_smem();
    mbar_expect_tx(bar, bytes);
  }
  // bytes: a multiple of 16; both addresses 16-byte aligned.
  __device__ void copy(void* dst, const void* src, uint32_t bytes) const {
    bulk_load(dst, src, bytes, bar);
  }
  // On a timeout the copies may still be in flight: wait for them (with the
  // fixed drain bound) before the CTA returns, so that none lands in the
  // shared memory of a later CTA.
  __device__ bool wait(unsigned long long limit_ns) const {
    if (mbar_try_wait(bar, 0)) return true;
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, 0)) {
      if (globaltimer() - t0 > limit_ns) {
        atomicOr(&g_status, kStatusTimeout);
        drain_wait(bar, 0);
        return false;
      }
    }
    return true;
  }
};

// Shared-memory bytes of the staged prologue for `tok` tokens: q, k, v and
// ve rows, then the block's gate logits as float32 (with ve).
__host__ __device__ inline size_t prologue_stage_bytes(int tok, int H, int Hk, int D, int esize,
                                                       bool has_ve) {
  return static_cast<size_t>(tok) * (H + (has_ve ? 3 : 2) * Hk) * D * esize +
         (has_ve ? static_cast<size_t>(tok) * Hk * 4 : 0);
}

template <typename T, int D, bool STAGED>
__global__ void __launch_bounds__(kPrologueThreads)
    prologue_kernel(const PrologueParams p) {
  using RL = RowLayout<T, D>;
  using HVec = HalfVec<T, RL::HV>;
  constexpr int HV = RL::HV, LPR = RL::LPR, HALF = RL::HALF;
  constexpr int ROWS_PER_PASS = kPrologueThreads / LPR;

  __shared__ __align__(16) TokenTable<HALF, HV> tab;
  __shared__ uint64_t s_bar;
  extern __shared__ __align__(128) uint8_t stage_smem[];

  const long long n_tok = static_cast<long long>(p.B) * p.T;
  const long long tok0 = static_cast<long long>(blockIdx.x) * p.tok;
  const int ntt = static_cast<int>(n_tok - tok0 < p.tok ? n_tok - tok0 : p.tok);
  // Row bases of the block: token tt, head h of a tensor with n heads is
  // row tt * n + h from these.
  const size_t qrow = static_cast<size_t>(p.H) * D, kvrow = static_cast<size_t>(p.Hk) * D;
  const T *qb = static_cast<const T*>(p.q) + tok0 * qrow;
  const T *kb = static_cast<const T*>(p.k) + tok0 * kvrow;
  const T *vb = static_cast<const T*>(p.v) + tok0 * kvrow;
  const T *eb = p.has_ve ? static_cast<const T*>(p.ve) + tok0 * kvrow : nullptr;
  const Stage stage{&s_bar};
  // The block's gate logits (value rows), staged next to the rows so that no
  // row waits on a global load: float32 after the ve rows.
  float* s_gate = reinterpret_cast<float*>(stage_smem + static_cast<size_t>(p.tok) * (qrow + 3 * kvrow) * sizeof(T));
  pdl_launch_dependents();
  tab.fill(tok0, p.T, p.omega, ntt);
  pdl_wait();
  if constexpr (STAGED) {
    T* sq = reinterpret_cast<T*>(stage_smem);
    T* sk = sq + p.tok * qrow;
    T* sv = sk + p.tok * kvrow;
    T* se = sv + p.tok * kvrow;
    if (p.has_ve && !p.xg)
      for (int i = threadIdx.x; i < ntt * p.Hk; i += blockDim.x)
        s_gate[i] = Vec16<T>::scalar(p.gate, static_cast<size_t>(tok0) * p.Hk + i);
    if (threadIdx.x == 0) {
      const uint32_t qb_ = static_cast<uint32_t>(ntt * qrow * sizeof(T));
      const uint32_t kb_ = static_cast<uint32_t>(ntt * kvrow * sizeof(T));
      stage.arm(qb_ + (p.has_ve ? 3u : 2u) * kb_);
      stage.copy(sq, qb, qb_);
      stage.copy(sk, kb, kb_);
      stage.copy(sv, vb, kb_);
      if (p.has_ve) stage.copy(se, eb, kb_);
    }
    qb = sq;
    kb = sk;
    vb = sv;
    eb = se;
  }
  __syncthreads();
  if constexpr (STAGED) {
    if (!stage.wait(p.wait_ns)) return;
  }

  const int rows_per_tok = p.H + 2 * p.Hk;
  const int total_rows = ntt * rows_per_tok;
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
    const bool valid = in_range;  // every token of the block exists
    // Row kinds: [0, H) query heads, [H, H+Hk) key heads, then value heads.
    int kind, head, nheads;
    if (kind_row < p.H) {
      kind = 0; head = kind_row; nheads = p.H;
    } else if (kind_row < p.H + p.Hk) {
      kind = 1; head = kind_row - p.H; nheads = p.Hk;
    } else {
      kind = 2; head = kind_row - p.H - p.Hk; nheads = p.Hk;
    }
    // Row within the block (source) and within the tensor (destination).
    const size_t brow = static_cast<size_t>(tt) * nheads + head;
    const size_t row = static_cast<size_t>(valid ? tok0 + tt : 0) * nheads + head;
    const size_t off_lo = row * D + static_cast<size_t>(sub) * HV;
    const size_t off_hi = off_lo + HALF;
    const size_t boff = brow * D + static_cast<size_t>(sub) * HV;
    const T* src = kind == 0 ? qb : (kind == 1 ? kb : vb);
    if (valid && !check_bounds(row < static_cast<size_t>(n_tok) * nheads && tt < ntt && head < nheads))
      continue;  // checked build: a row outside the tensor is skipped
    float xl[HV], xh[HV], el[HV], eh[HV];
    float gl = 0.f;
    if (valid) {
      HVec::load(src + boff, xl);
      HVec::load(src + boff + HALF, xh);
    } else {
#pragma unroll
      for (int i = 0; i < HV; ++i) xl[i] = xh[i] = 0.f;
    }
    const bool has_e = valid && kind == 2 && p.has_ve;
    if (has_e) {
      HVec::load(eb + boff, el);
      HVec::load(eb + boff + HALF, eh);
      if (!p.xg) gl = STAGED ? s_gate[tt * p.Hk + head] : Vec16<T>::scalar(p.gate, row);
    } else {
#pragma unroll
      for (int i = 0; i < HV; ++i) el[i] = eh[i] = 0.f;
    }
    if (p.xg) {
      // Gate logit of value rows: the row's LPR lanes split the C channels
      // of x; the reduction runs on every lane (uniform shuffles).
      float gp = 0.f;
      if (has_e) {
        const T* xr = static_cast<const T*>(p.xg) + (tok0 + tt) * p.x_stride;
        const T* wr = static_cast<const T*>(p.w_gate) + static_cast<size_t>(head) * p.gc;
        for (int c = sub; c < p.gc; c += LPR) gp = fmaf(Vec16<T>::scalar(xr, c), Vec16<T>::scalar(wr, c), gp);
      }
      gp = row_sum<LPR>(gp);
      if (has_e) {
        // Rounded to the layer dtype: the backward reads the stored logit.
        if constexpr (sizeof(T) == 2) {
          const __nv_bfloat16 g16 = __float2bfloat16_rn(gp);
          gl = __bfloat162float(g16);
          if (sub == 0) static_cast<__nv_bfloat16*>(p.gate_out)[row] = g16;
        } else {
          gl = gp;
          if (sub == 0) static_cast<float*>(p.gate_out)[row] = gp;
        }
      }
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
    tab.load(tt, sub * HV, cv, sv);
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
