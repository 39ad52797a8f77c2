// gate.cuh -- backward of the value-embedding gate's projection.
//
// Page "5만원으로 나만의 ChatGPT 훈련하는 방법", section "1. GPT 모델",
// value-embedding code: the gate logits are a bias-free linear map of the
// first C channels of the block input x, one logit per KV head:
//   gate[b,t,h] = sum_{c<C} x[b,t,c] w[h,c].
// Given dgate = dL/dgate (the attention backward's dgate output):
//   dx[b,t,c] = sum_h dgate[b,t,h] w[h,c]          (B, T, C)
//   dw[h,c]   = sum_{b,t} dgate[b,t,h] x[b,t,c]    (Hk, C), float32
// One launch does both. A cluster of kGateCluster dw blocks owns 32
// channels of one head: block r of the cluster sums tokens r*32 + lane + 256 i
// over its 32 token lanes (a tree over the lanes), and the cluster's block 0
// adds the blocks' partials from their shared memory in rank order, so dw is
// deterministic and needs no scratch memory; the dx blocks take 1024
// (token, channel) entries each.
#pragma once
#include <cooperative_groups.h>

#include "prologue.cuh"

namespace cswattn {

constexpr int kGateDwThreads = 1024;  // 32 channels x 32 token lanes (dx: 1024 entries)
constexpr int kGateCluster = 8;       // dw blocks per (head, 32 channels), one cluster

struct GateBwdParams {
  long long ntok;      // B * T
  long long x_stride;  // elements between consecutive tokens of x
  int Hk, C;
  int dw_blocks;       // Hk * ceil(C / 32) * kGateCluster
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
    // ---- dw[h, c0 + lane]: token lane `tl` of cluster block `rank` sums
    // tokens rank*32 + tl, + 32*kGateCluster, ...
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = static_cast<int>(cluster.block_rank());
    const int cblocks = (p.C + 31) / 32;
    const int grp = blk / kGateCluster;
    const int h = grp / cblocks, c0 = (grp % cblocks) * 32;
    const int lane = threadIdx.x & 31, tl = threadIdx.x >> 5;
    const int c = c0 + lane;
    float acc = 0.f;
    if (c < p.C) {
      const T* x = static_cast<const T*>(p.x);
      const T* dg = static_cast<const T*>(p.dgate);
#pragma unroll 4
      for (long long n = rank * 32 + tl; n < p.ntok; n += 32 * kGateCluster)
        acc = fmaf(Vec16<T>::scalar(dg, n * p.Hk + h), Vec16<T>::scalar(x, n * p.x_stride + c), acc);
    }
    red[tl][lane] = acc;
    __syncthreads();
    for (int s = 16; s >= 1; s >>= 1) {
      if (tl < s) red[tl][lane] += red[tl + s][lane];
      __syncthreads();
    }
    cluster.sync();  // every block's partial in its red[0]
    if (rank == 0 && tl == 0 && c < p.C) {
      float sum = 0.f;
      for (int r = 0; r < kGateCluster; ++r) sum += cluster.map_shared_rank(&red[0][0], r)[lane];
      p.dw[static_cast<size_t>(h) * p.C + c] = sum;
    }
    cluster.sync();  // the partials stay until block 0 has read them
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
