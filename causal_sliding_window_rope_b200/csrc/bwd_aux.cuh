// bwd_aux.cuh -- the backward's HBM-bound helpers.
//
// preprocess: Delta_i = dO_i . O_i per (b, h, t), the row term of the
//   softmax backward (ds_ij = p_ij (dp_ij - Delta_i)).
// epilogue: the chain rule back through the prologue (page section
//   "1. GPT 모델": RoPE, QK normalisation, value-embedding code):
//   dq = RMSNorm'(RoPE^-1(dq~)), dk likewise, dv = dv_eff,
//   dve = 3 s dv_eff, dgate = 3 s (1 - s) sum_d dv_eff ve with s = sigmoid(gate).
// Both stage their token block into shared memory with bulk copies issued at
// kernel start, like the prologue, and use its split-halves row layout (each
// lane holds matching slices of both halves of a row); reductions are
// shuffles over a row's lanes.
#pragma once
#include "prologue.cuh"

namespace cswattn {

// Row terms of the backward, in the padded layout (B, H, Tpad) with Tpad a
// multiple of 64: delta = dO.O and nlse2 = -lse * log2(e) (negated, so that
// the backward forms c2 s + nlse2 with one fused multiply-add); past T,
// delta = 0 and nlse2 = -inf (so exp2(c2 s + nlse2) = 0 for padding queries).
struct PreParams {
  long long rows;  // B * T * H
  int T, H, Tpad;
  int tok;                     // tokens per CTA (1..kPrologueTok)
  unsigned long long wait_ns;  // bound of the staging wait
  const void *O, *dO;
  const float* lse;  // (B, H, T)
  float* delta;      // (B, H, Tpad)
  float* nlse2;      // (B, H, Tpad)
  float* dq_zero;    // (B, T, H, D) accumulator to clear, or null
};

// Shared-memory bytes of the staged preprocess for `tok` tokens: O and dO
// rows, then the block's lse values (float32).
__host__ __device__ inline size_t preprocess_stage_bytes(int tok, int H, int D, int esize) {
  return 2 * static_cast<size_t>(tok) * H * D * esize + static_cast<size_t>(tok) * H * 4;
}

// One CTA per `tok` consecutive tokens, staged like the prologue (one bulk
// copy each for the block's O and dO rows); each row (token, head) is owned
// by LPR lanes in the split-halves layout, reduced with shuffles.
template <typename T, int D, bool STAGED>
__global__ void __launch_bounds__(kPrologueThreads) preprocess_kernel(const PreParams p) {
  using RL = RowLayout<T, D>;
  using HVec = HalfVec<T, RL::HV>;
  constexpr int HV = RL::HV, LPR = RL::LPR, HALF = RL::HALF;
  constexpr int ROWS_PER_PASS = kPrologueThreads / LPR;
  __shared__ int s_b[kPrologueTok], s_t[kPrologueTok];
  __shared__ uint64_t s_bar;
  extern __shared__ __align__(128) uint8_t stage_smem[];
  const long long n_tok = p.rows / p.H;
  const long long tok0 = static_cast<long long>(blockIdx.x) * p.tok;
  const int ntt = static_cast<int>(n_tok - tok0 < p.tok ? n_tok - tok0 : p.tok);
  const size_t orow = static_cast<size_t>(p.H) * D;
  const T* ob = static_cast<const T*>(p.O) + tok0 * orow;
  const T* gb = static_cast<const T*>(p.dO) + tok0 * orow;
  const Stage stage{&s_bar};
  pdl_launch_dependents();
  if (threadIdx.x < ntt) {
    const long long tok = tok0 + threadIdx.x;
    s_b[threadIdx.x] = static_cast<int>(tok / p.T);
    s_t[threadIdx.x] = static_cast<int>(tok % p.T);
  }
  pdl_wait();
  // The block's lse values, staged next to the rows so that no row waits on
  // a global load: float32 after the dO rows.
  float* s_lse = reinterpret_cast<float*>(stage_smem + 2 * static_cast<size_t>(p.tok) * orow * sizeof(T));
  if constexpr (STAGED) {
    T* so = reinterpret_cast<T*>(stage_smem);
    T* sg = so + p.tok * orow;
    if (threadIdx.x == 0) {
      const uint32_t nb = static_cast<uint32_t>(ntt * orow * sizeof(T));
      stage.arm(2 * nb);
      stage.copy(so, ob, nb);
      stage.copy(sg, gb, nb);
    }
    ob = so;
    gb = sg;
    for (int i = threadIdx.x; i < ntt * p.H; i += blockDim.x) {
      const long long tok = tok0 + i / p.H;
      const long long b = tok / p.T, t = tok % p.T;
      s_lse[i] = p.lse[(b * p.H + i % p.H) * p.T + t];
    }
  }
  if (p.dq_zero) {
    // The block's rows of the dq accumulator (contiguous in (B,T,H,D)).
    float4* z = reinterpret_cast<float4*>(p.dq_zero + tok0 * orow);
    const int n4 = static_cast<int>(ntt * orow / 4);
    for (int i = threadIdx.x; i < n4; i += blockDim.x) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();
  if constexpr (STAGED) {
    if (!stage.wait(p.wait_ns)) return;
  }
  const int sub = threadIdx.x % LPR;
  const int grp = threadIdx.x / LPR;
  const int total_rows = ntt * p.H;
  RowCursor cur{0, 0};
  cur.advance(grp, p.H);
  for (int base = 0; base < total_rows; base += ROWS_PER_PASS) {
    const bool valid = base + grp < total_rows;
    const int tt = valid ? cur.tt : 0, h = valid ? cur.kind_row : 0;
    cur.advance(ROWS_PER_PASS, p.H);
    float acc = 0.f;
    if (valid) {
      const size_t lo = (static_cast<size_t>(tt) * p.H + h) * D + sub * HV;
      float o0[HV], o1[HV], g0[HV], g1[HV];
      HVec::load(ob + lo, o0);
      HVec::load(ob + lo + HALF, o1);
      HVec::load(gb + lo, g0);
      HVec::load(gb + lo + HALF, g1);
#pragma unroll
      for (int i = 0; i < HV; ++i) acc = fmaf(o0[i], g0[i], fmaf(o1[i], g1[i], acc));
    }
    acc = row_sum<LPR>(acc);
    if (valid && sub == 0 && check_bounds(s_b[tt] < p.rows / p.H / p.T && s_t[tt] < p.T && h < p.H)) {
      const long long b = s_b[tt], t = s_t[tt];
      const long long o = (b * p.H + h) * p.Tpad;
      p.delta[o + t] = acc;
      p.nlse2[o + t] = (STAGED ? s_lse[tt * p.H + h] : p.lse[(b * p.H + h) * p.T + t]) * -1.4426950408889634f;
      if (t == p.T - 1) {
        for (long long tp = p.T; tp < p.Tpad; ++tp) {
          p.delta[o + tp] = 0.f;
          p.nlse2[o + tp] = -INFINITY;
        }
      }
    }
  }
}

struct EpiParams {
  int B, T, H, Hk;
  int has_ve;
  int tok;                              // tokens per CTA (1..kPrologueTok)
  unsigned long long wait_ns;           // bound of the staging wait
  float omega[kMaxHalfD];
  const void *q, *k, *ve, *gate;        // prologue inputs (layer dtype)
  const float *rstd_q, *rstd_k;
  const float* dq_acc;                  // (B,T,H,D) dq~ (scaled)
  const float *dk_acc, *dv_acc;         // [parts] x (B,T,Hk,D) partial dk~ (scaled), dv_eff
  int parts;                            // number of partial slots to sum
  long long kv_stride;                  // elements between partial slots
  void *dq, *dk, *dv, *dve, *dgate;     // outputs (layer dtype)
};

// Shared-memory bytes of the staged epilogue for `tok` tokens: dq~, the dk~
// and dv_eff partial slots (float32), then q, k and ve (layer dtype), then
// the block's rstd_q, rstd_k and gate values (float32).
__host__ __device__ inline size_t epilogue_stage_bytes(int tok, int H, int Hk, int D, int esize,
                                                       int parts, bool has_ve) {
  return static_cast<size_t>(tok) * D *
             ((static_cast<size_t>(H) + 2 * static_cast<size_t>(parts) * Hk) * 4 +
              (static_cast<size_t>(H) + (has_ve ? 2 : 1) * Hk) * esize) +
         static_cast<size_t>(tok) * (H + 2 * Hk) * 4;
}

template <int VEC>
__device__ __forceinline__ void load_f32(const float* src, float (&x)[VEC]) {
  if constexpr (VEC == 8) {
    // Two 16-byte chunks per lane, the lanes 32 bytes apart: a lane whose
    // chunk pair starts in the upper 128 bytes of a 256-byte span (address
    // bit 7) reads its second chunk first, so each load instruction of a
    // quarter warp covers 128 distinct bytes of banks (no conflicts).
    const int sw = static_cast<int>((reinterpret_cast<uintptr_t>(src) >> 7) & 1);
    const float4 a = *reinterpret_cast<const float4*>(src + 4 * sw);
    const float4 b = *reinterpret_cast<const float4*>(src + 4 - 4 * sw);
    const float4 lo = sw ? b : a, hi = sw ? a : b;
    x[0] = lo.x; x[1] = lo.y; x[2] = lo.z; x[3] = lo.w;
    x[4] = hi.x; x[5] = hi.y; x[6] = hi.z; x[7] = hi.w;
  } else if constexpr (VEC % 4 == 0) {
#pragma unroll
    for (int i = 0; i < VEC; i += 4) {
      float4 u = *reinterpret_cast<const float4*>(src + i);
      x[i] = u.x;
      x[i + 1] = u.y;
      x[i + 2] = u.z;
      x[i + 3] = u.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < VEC; i += 2) {
      float2 u = *reinterpret_cast<const float2*>(src + i);
      x[i] = u.x;
      x[i + 1] = u.y;
    }
  }
}

template <typename T, int D, bool STAGED>
__global__ void __launch_bounds__(kPrologueThreads) epilogue_kernel(const EpiParams p) {
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
  // Block bases: token tt, head h of a tensor with n heads is row tt * n + h.
  const size_t qrow = static_cast<size_t>(p.H) * D, kvrow = static_cast<size_t>(p.Hk) * D;
  // Element stride between partial slots as seen from the block bases.
  size_t slot = static_cast<size_t>(p.kv_stride);
  const float* dqb = p.dq_acc + tok0 * qrow;
  const float* dkb = p.dk_acc + tok0 * kvrow;
  const float* dvb = p.dv_acc + tok0 * kvrow;
  const T* qb = static_cast<const T*>(p.q) + tok0 * qrow;
  const T* kb = static_cast<const T*>(p.k) + tok0 * kvrow;
  const T* eb = p.has_ve ? static_cast<const T*>(p.ve) + tok0 * kvrow : nullptr;
  const Stage stage{&s_bar};
  // Staged row terms (float32): rstd_q [tok][H], rstd_k [tok][Hk], gate
  // [tok][Hk], after the staged rows.
  float* s_rterm = reinterpret_cast<float*>(
      stage_smem + static_cast<size_t>(p.tok) * D *
                       ((static_cast<size_t>(p.H) + 2 * static_cast<size_t>(p.parts) * p.Hk) * 4 +
                        (static_cast<size_t>(p.H) + (p.has_ve ? 2 : 1) * p.Hk) * sizeof(T)));
  pdl_launch_dependents();
  tab.fill(tok0, p.T, p.omega, ntt);
  pdl_wait();
  if constexpr (STAGED) {
    float* sdq = reinterpret_cast<float*>(stage_smem);
    float* sdk = sdq + p.tok * qrow;
    float* sdv = sdk + p.parts * p.tok * kvrow;
    T* sq = reinterpret_cast<T*>(sdv + p.parts * p.tok * kvrow);
    T* sk = sq + p.tok * qrow;
    T* se = sk + p.tok * kvrow;
    if (threadIdx.x == 0) {
      const uint32_t qf = static_cast<uint32_t>(ntt * qrow * 4);
      const uint32_t kf = static_cast<uint32_t>(ntt * kvrow * 4);
      const uint32_t qh = static_cast<uint32_t>(ntt * qrow * sizeof(T));
      const uint32_t kh = static_cast<uint32_t>(ntt * kvrow * sizeof(T));
      stage.arm(qf + 2 * p.parts * kf + qh + (p.has_ve ? 2u : 1u) * kh);
      stage.copy(sdq, dqb, qf);
      for (int pi = 0; pi < p.parts; ++pi) {
        stage.copy(sdk + pi * p.tok * kvrow, dkb + pi * slot, kf);
        stage.copy(sdv + pi * p.tok * kvrow, dvb + pi * slot, kf);
      }
      stage.copy(sq, qb, qh);
      stage.copy(sk, kb, kh);
      if (p.has_ve) stage.copy(se, eb, kh);
    }
    // rstd_q, rstd_k and the gate logits of the block, after the rows.
    for (int i = threadIdx.x; i < ntt * p.H; i += blockDim.x) s_rterm[i] = p.rstd_q[tok0 * p.H + i];
    for (int i = threadIdx.x; i < ntt * p.Hk; i += blockDim.x) {
      s_rterm[p.tok * p.H + i] = p.rstd_k[tok0 * p.Hk + i];
      if (p.has_ve)
        s_rterm[p.tok * (p.H + p.Hk) + i] = Vec16<T>::scalar(p.gate, static_cast<size_t>(tok0) * p.Hk + i);
    }
    dqb = sdq;
    dkb = sdk;
    dvb = sdv;
    slot = p.tok * kvrow;
    qb = sq;
    kb = sk;
    eb = se;
  }
  __syncthreads();
  if constexpr (STAGED) {
    if (!stage.wait(p.wait_ns)) return;
  }

  const int rows_per_tok = p.H + 2 * p.Hk;
  const int total_rows = ntt * rows_per_tok;
  const int sub = threadIdx.x % LPR;
  const int grp = threadIdx.x / LPR;
  RowCursor cur{0, 0};
  cur.advance(grp, rows_per_tok);

  for (int base = 0; base < total_rows; base += ROWS_PER_PASS) {
    const bool valid = base + grp < total_rows;
    const int tt = valid ? cur.tt : 0;
    const int kind_row = valid ? cur.kind_row : 0;
    cur.advance(ROWS_PER_PASS, rows_per_tok);
    int kind, head, nheads;
    if (kind_row < p.H) {
      kind = 0; head = kind_row; nheads = p.H;
    } else if (kind_row < p.H + p.Hk) {
      kind = 1; head = kind_row - p.H; nheads = p.Hk;
    } else {
      kind = 2; head = kind_row - p.H - p.Hk; nheads = p.Hk;
    }
    // Row within the block (sources) and within the tensor (destinations).
    const size_t brow = static_cast<size_t>(tt) * nheads + head;
    const size_t row = static_cast<size_t>(tok0 + tt) * nheads + head;  // (b,t,head)
    if (valid && !check_bounds(row < static_cast<size_t>(n_tok) * nheads && tt < ntt)) continue;
    const size_t off_lo = row * D + static_cast<size_t>(sub) * HV;
    const size_t off_hi = off_lo + HALF;
    const size_t boff = brow * D + static_cast<size_t>(sub) * HV;

    // Gradient w.r.t. the rotated, normalised row (or dv_eff for value rows),
    // and the row's input (q or k) or ve.
    float dl[HV], dh[HV], xl[HV], xh[HV];
    float rs = 0.f, gl = 0.f;
    if (valid) {
      const float* src = kind == 0 ? dqb : (kind == 1 ? dkb : dvb);
      load_f32<HV>(src + boff, dl);
      load_f32<HV>(src + boff + HALF, dh);
      if (kind != 0) {
        // dK / dV arrive as partial sums from the backward's parts.
        for (int pi = 1; pi < p.parts; ++pi) {
          float el[HV], eh[HV];
          load_f32<HV>(src + pi * slot + boff, el);
          load_f32<HV>(src + pi * slot + boff + HALF, eh);
#pragma unroll
          for (int i = 0; i < HV; ++i) {
            dl[i] += el[i];
            dh[i] += eh[i];
          }
        }
      }
      if (kind != 2) {
        HVec::load((kind == 0 ? qb : kb) + boff, xl);
        HVec::load((kind == 0 ? qb : kb) + boff + HALF, xh);
        if constexpr (STAGED)
          rs = kind == 0 ? s_rterm[tt * p.H + head] : s_rterm[p.tok * p.H + tt * p.Hk + head];
        else
          rs = (kind == 0 ? p.rstd_q : p.rstd_k)[row];
      } else if (p.has_ve) {
        HVec::load(eb + boff, xl);
        HVec::load(eb + boff + HALF, xh);
        if constexpr (STAGED)
          gl = s_rterm[p.tok * (p.H + p.Hk) + tt * p.Hk + head];
        else
          gl = Vec16<T>::scalar(p.gate, row);
      } else {
#pragma unroll
        for (int i = 0; i < HV; ++i) xl[i] = xh[i] = 0.f;
      }
    } else {
#pragma unroll
      for (int i = 0; i < HV; ++i) dl[i] = dh[i] = xl[i] = xh[i] = 0.f;
    }

    // RoPE^-1 on this lane's pairs (kind 2 rows skip it below).
    float cv[HV], sv[HV], nl[HV], nh[HV];
    tab.load(tt, sub * HV, cv, sv);
#pragma unroll
    for (int i = 0; i < HV; ++i) {
      nl[i] = fmaf(dl[i], cv[i], dh[i] * sv[i]);
      nh[i] = fmaf(-dl[i], sv[i], dh[i] * cv[i]);
    }
    // One reduction serves both row kinds: for q/k rows sum_d dn*n with
    // n = r x (the RMSNorm term); for value rows sum_d dv_eff*ve.
    const bool vrow = kind == 2;
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < HV; ++i)
      dot = vrow ? fmaf(dl[i], xl[i], fmaf(dh[i], xh[i], dot))
                 : fmaf(nl[i], xl[i] * rs, fmaf(nh[i], xh[i] * rs, dot));
    dot = row_sum<LPR>(dot);
    if (!valid) continue;
    if (vrow) {
      HVec::store(static_cast<T*>(p.dv) + off_lo, dl);
      HVec::store(static_cast<T*>(p.dv) + off_hi, dh);
      if (p.has_ve) {
        const float sg = 1.0f / (1.0f + expf(-gl));
        const float coef = 3.0f * sg;
        float ol[HV], oh[HV];
#pragma unroll
        for (int i = 0; i < HV; ++i) {
          ol[i] = coef * dl[i];
          oh[i] = coef * dh[i];
        }
        HVec::store(static_cast<T*>(p.dve) + off_lo, ol);
        HVec::store(static_cast<T*>(p.dve) + off_hi, oh);
        if (sub == 0) {
          const float dg = dot * coef * (1.0f - sg);
          if constexpr (sizeof(T) == 2)
            static_cast<__nv_bfloat16*>(p.dgate)[row] = __float2bfloat16_rn(dg);
          else
            static_cast<float*>(p.dgate)[row] = dg;
        }
      }
    } else {
      // RMSNorm backward: dx = r (dn - n mean(dn * n)), n = r x.
      const float mean = dot / static_cast<float>(D);
      float ol[HV], oh[HV];
#pragma unroll
      for (int i = 0; i < HV; ++i) {
        ol[i] = rs * (nl[i] - xl[i] * rs * mean);
        oh[i] = rs * (nh[i] - xh[i] * rs * mean);
      }
      T* dst = static_cast<T*>(kind == 0 ? p.dq : p.dk);
      HVec::store(dst + off_lo, ol);
      HVec::store(dst + off_hi, oh);
    }
  }
}

}  // namespace cswattn
