// simt_f32.cuh -- float32 attention on CUDA cores for small head_dim.
//
// The microgpt-sized layer (T=16, head_dim=4) is far below one tensor-core
// tile and its tolerance (max-abs 1e-4) rules out TF32, so it runs in plain
// fp32 FMA: one thread per query row in the forward, one thread per query
// row (dq) and per key row (dk, dv) in the backward. Same arithmetic as the
// page's causal windowed attention call (section "5. 플래시 어텐션 통합"),
// online softmax in the forward, recomputed probabilities from the row
// log-sum-exp in the backward.
#pragma once
#include "common.cuh"

namespace cswattn {

struct SimtParams {
  int B, T, H, Hk, W;
  int Tpad;                    // row stride of delta (B,H,Tpad)
  float scale;
  const float *q, *k, *v;      // q_out (B,T,H,D), k_out, v_out (B,T,Hk,D)
  const float *O, *dO, *lse;   // backward inputs
  const float* delta;          // (B,H,Tpad) dO.O
  float *out_O, *out_lse;      // forward outputs
  float *dq_acc;               // (B,T,H,D) dq~ (scaled)
  float *dk_acc, *dv_acc;      // (B,T,Hk,D) dk~ (scaled), dv_eff
};

template <int D>
__global__ void __launch_bounds__(128) simt_fwd_kernel(const SimtParams p) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rows = static_cast<long long>(p.B) * p.H * p.T;
  if (idx >= rows) return;
  const int i = static_cast<int>(idx % p.T);
  const int h = static_cast<int>((idx / p.T) % p.H);
  const int b = static_cast<int>(idx / (static_cast<long long>(p.T) * p.H));
  const int hk = h / (p.H / p.Hk);
  const float* qi = p.q + ((static_cast<size_t>(b) * p.T + i) * p.H + h) * D;
  float qv[D], acc[D];
#pragma unroll
  for (int d = 0; d < D; ++d) {
    qv[d] = qi[d];
    acc[d] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int lo = max(0, i - p.W + 1);
  for (int j = lo; j <= i; ++j) {
    const size_t kv = ((static_cast<size_t>(b) * p.T + j) * p.Hk + hk) * D;
    float s = 0.f;
#pragma unroll
    for (int d = 0; d < D; ++d) s = fmaf(qv[d], p.k[kv + d], s);
    s *= p.scale;
    const float m_new = fmaxf(m, s);
    const float alpha = expf(m - m_new);  // 0 on the first key (m = -inf)
    const float pj = expf(s - m_new);
    l = l * alpha + pj;
#pragma unroll
    for (int d = 0; d < D; ++d) acc[d] = fmaf(pj, p.v[kv + d], acc[d] * alpha);
    m = m_new;
  }
  const float inv = 1.f / l;
  float* o = p.out_O + ((static_cast<size_t>(b) * p.T + i) * p.H + h) * D;
#pragma unroll
  for (int d = 0; d < D; ++d) o[d] = acc[d] * inv;
  p.out_lse[(static_cast<size_t>(b) * p.H + h) * p.T + i] = m + logf(l);
}

// dq~_i = c * sum_j p_ij (dp_ij - Delta_i) k~_j, written to dq_acc (B,T,H,D).
template <int D>
__global__ void __launch_bounds__(128) simt_bwd_dq_kernel(const SimtParams p) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rows = static_cast<long long>(p.B) * p.H * p.T;
  if (idx >= rows) return;
  const int i = static_cast<int>(idx % p.T);
  const int h = static_cast<int>((idx / p.T) % p.H);
  const int b = static_cast<int>(idx / (static_cast<long long>(p.T) * p.H));
  const int hk = h / (p.H / p.Hk);
  const size_t qo = ((static_cast<size_t>(b) * p.T + i) * p.H + h) * D;
  float qv[D], dov[D], acc[D];
#pragma unroll
  for (int d = 0; d < D; ++d) {
    qv[d] = p.q[qo + d];
    dov[d] = p.dO[qo + d];
    acc[d] = 0.f;
  }
  const size_t row = (static_cast<size_t>(b) * p.H + h) * p.T + i;
  const float li = p.lse[row];
  const float di = p.delta[(static_cast<size_t>(b) * p.H + h) * p.Tpad + i];
  const int lo = max(0, i - p.W + 1);
  for (int j = lo; j <= i; ++j) {
    const size_t kv = ((static_cast<size_t>(b) * p.T + j) * p.Hk + hk) * D;
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int d = 0; d < D; ++d) {
      s = fmaf(qv[d], p.k[kv + d], s);
      dp = fmaf(dov[d], p.v[kv + d], dp);
    }
    const float pij = expf(s * p.scale - li);
    const float ds = pij * (dp - di);
#pragma unroll
    for (int d = 0; d < D; ++d) acc[d] = fmaf(ds, p.k[kv + d], acc[d]);
  }
  float* out = p.dq_acc + qo;
#pragma unroll
  for (int d = 0; d < D; ++d) out[d] = acc[d] * p.scale;
}

// dk~_j = c * sum_{h in group} sum_i ds_ij q~_i and dv_j = sum p_ij dO_i.
template <int D>
__global__ void __launch_bounds__(128) simt_bwd_dkv_kernel(const SimtParams p) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rows = static_cast<long long>(p.B) * p.Hk * p.T;
  if (idx >= rows) return;
  const int j = static_cast<int>(idx % p.T);
  const int hk = static_cast<int>((idx / p.T) % p.Hk);
  const int b = static_cast<int>(idx / (static_cast<long long>(p.T) * p.Hk));
  const int g = p.H / p.Hk;
  const size_t kvo = ((static_cast<size_t>(b) * p.T + j) * p.Hk + hk) * D;
  float kv[D], vv[D], dk[D], dv[D];
#pragma unroll
  for (int d = 0; d < D; ++d) {
    kv[d] = p.k[kvo + d];
    vv[d] = p.v[kvo + d];
    dk[d] = 0.f;
    dv[d] = 0.f;
  }
  const int last = static_cast<int>(min(static_cast<long long>(p.T) - 1,
                                        static_cast<long long>(j) + p.W - 1));
  for (int h = hk * g; h < (hk + 1) * g; ++h) {
    for (int i = j; i <= last; ++i) {
      const size_t qo = ((static_cast<size_t>(b) * p.T + i) * p.H + h) * D;
      const size_t row = (static_cast<size_t>(b) * p.H + h) * p.T + i;
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int d = 0; d < D; ++d) {
        s = fmaf(p.q[qo + d], kv[d], s);
        dp = fmaf(p.dO[qo + d], vv[d], dp);
      }
      const float pij = expf(s * p.scale - p.lse[row]);
      const float ds = pij * (dp - p.delta[(static_cast<size_t>(b) * p.H + h) * p.Tpad + i]);
#pragma unroll
      for (int d = 0; d < D; ++d) {
        dk[d] = fmaf(ds, p.q[qo + d], dk[d]);
        dv[d] = fmaf(pij, p.dO[qo + d], dv[d]);
      }
    }
  }
#pragma unroll
  for (int d = 0; d < D; ++d) {
    p.dk_acc[kvo + d] = dk[d] * p.scale;
    p.dv_acc[kvo + d] = dv[d];
  }
}

}  // namespace cswattn
