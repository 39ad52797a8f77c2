// gate.cuh -- backward of the value-embedding gate's projection.
//
// Page "5만원으로 나만의 ChatGPT 훈련하는 방법", section "1. GPT 모델",
// value-embedding code: the gate logits are a bias-free linear map of the
// first C channels of the block input x, one logit per KV head:
//   gate[b,t,h] = sum_{c<C} x[b,t,c] w[h,c].
// Given dgate = dL/dgate (the attention backward's dgate output):
//   dx[b,t,c] = sum_h dgate[b,t,h] w[h,c]          (B, T, C)
//   dw[h,c]   = sum_{b,t} dgate[b,t,h] x[b,t,c]    (Hk, C), float32
// One launch does both. The dw blocks each own 32 channels of one head and
// sum over all tokens in a fixed order (32 token lanes, then a tree over the
// lanes), so dw is deterministic; the dx blocks take 1024 (token, channel)
// entries each.
#pragma once
#include "prologue.cuh"

namespace cswattn {

constexpr int kGateDwThreads = 1024;  // 32 channels x 32 token lanes (dx: 1024 entries)

struct GateBwdParams {
  long long ntok;      // B * T
  long long x_stride;  // elements between consecutive tokens of x
  int Hk, C;
  int dw_blocks;       // Hk * ceil(C / 32)
  const void* x;       // (B, T, x_stride), layer dtype
  const void* w;       // (Hk, C), layer dtype
  const void* dgate;   // (B, T, Hk), layer dtype
  void* dx;            // (B, T, C), layer dtype
  float* dw;           // (Hk, C)
};

template <typename T>
__global__ void __launch_bounds__(kGateDwThreads) gate_bwd_kernel(const GateBwdParams p) {
  __shared__ float red[32][33];
  pdl_launch_dependents();
  pdl_wait();
  const int blk = static_cast<int>(blockIdx.x);
  if (blk < p.dw_blocks) {
    // ---- dw[h, c0 + lane]: token lane `tl` sums tokens tl, tl + 32, ...
    const int cblocks = (p.C + 31) / 32;
    const int h = blk / cblocks, c0 = (blk % cblocks) * 32;
    const int lane = threadIdx.x & 31, tl = threadIdx.x >> 5;
    const int c = c0 + lane;
    float acc = 0.f;
    if (c < p.C) {
      const T* x = static_cast<const T*>(p.x);
      const T* dg = static_cast<const T*>(p.dgate);
#pragma unroll 4
      for (long long n = tl; n < p.ntok; n += 32)
        acc = fmaf(Vec16<T>::scalar(dg, n * p.Hk + h), Vec16<T>::scalar(x, n * p.x_stride + c), acc);
    }
    red[tl][lane] = acc;
    __syncthreads();
    for (int s = 16; s >= 1; s >>= 1) {
      if (tl < s) red[tl][lane] += red[tl + s][lane];
      __syncthreads();
    }
    if (tl == 0 && c < p.C) p.dw[static_cast<size_t>(h) * p.C + c] = red[0][lane];
  } else {
    // ---- dx: one (token, channel) entry per thread
    const long long e = static_cast<long long>(blk - p.dw_blocks) * kGateDwThreads + threadIdx.x;
    if (e >= p.ntok * p.C) return;
    const long long n = e / p.C;
    const int c = static_cast<int>(e % p.C);
    const T* dg = static_cast<const T*>(p.dgate);
    const T* w = static_cast<const T*>(p.w);
    float s = 0.f;
    for (int h = 0; h < p.Hk; ++h)
      s = fmaf(Vec16<T>::scalar(dg, n * p.Hk + h), Vec16<T>::scalar(w, static_cast<size_t>(h) * p.C + c), s);
    if constexpr (sizeof(T) == 2)
      static_cast<__nv_bfloat16*>(p.dx)[e] = __float2bfloat16_rn(s);
    else
      static_cast<float*>(p.dx)[e] = s;
  }
}

}  // namespace cswattn
