// fp8.cuh -- tensor-wise E4M3 quantization of the projection's operands.
//
// Page "5만원으로 나만의 ChatGPT 훈련하는 방법", section "3. 정밀도 관리
// (nanochat/common.py)": with --fp8 the Linear layers become Float8Linear
// with tensor-wise scaling. For a tensor t: scale = amax(|t|) / 448 (1 for
// an all-zero tensor) and its FP8 E4M3 codes are round-to-nearest-even of
// t / scale (float32 division), saturated to the largest finite value.
// Two grid-stride kernels over 8-element (16-byte) vectors of both
// operands: fp8_amax folds |t| into two float bit patterns (atomicMax on the
// bits of non-negative floats orders them as the floats); fp8_quant writes
// the codes (8 bytes per vector) and the two scales.
#pragma once
#include <cuda_fp8.h>

#include "common.cuh"

namespace cswattn {

constexpr int kFp8Threads = 256;
constexpr float kE4M3Max = 448.0f;

struct Fp8QuantParams {
  const __nv_bfloat16* a;  // rows_a x cols, row stride lda (elements)
  long long rows_a, lda;
  const __nv_bfloat16* b;  // rows_b x cols, contiguous
  long long rows_b;
  int cols;                 // multiple of 8; lda multiple of 8; a, b 16-byte aligned
  unsigned int* amax_bits;  // [2], zero on entry of fp8_amax
  uint8_t* a8;              // rows_a x cols codes, contiguous, 8-byte aligned
  uint8_t* b8;              // rows_b x cols codes, contiguous, 8-byte aligned
  float* scales;            // [2]: scale of a, scale of b
};

// Both operands as one sequence of 8-element vectors: a's rows first (cols/8
// vectors each), then b's. Returns the vector's source address and its
// index among the codes of its operand (in vectors), and which operand.
struct Fp8Vec {
  const uint4* src;
  long long dst;  // vector index into a8 or b8
  bool is_b;
};

__device__ __forceinline__ Fp8Vec fp8_vec(const Fp8QuantParams& p, long long v, long long na8, int cpr) {
  Fp8Vec r;
  r.is_b = v >= na8;
  if (!r.is_b) {
    const long long row = v / cpr, c = v - row * cpr;
    r.src = reinterpret_cast<const uint4*>(p.a + row * p.lda + c * 8);
    r.dst = v;
  } else {
    r.src = reinterpret_cast<const uint4*>(p.b) + (v - na8);
    r.dst = v - na8;
  }
  return r;
}

__global__ void __launch_bounds__(kFp8Threads) fp8_amax_kernel(const Fp8QuantParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int cpr = p.cols / 8;
  const long long na8 = p.rows_a * cpr, n8 = na8 + p.rows_b * cpr;
  float ma = 0.f, mb = 0.f;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long v = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; v < n8; v += stride) {
    const Fp8Vec e = fp8_vec(p, v, na8, cpr);
    const uint4 u = __ldg(e.src);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(h2[j]);
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    if (e.is_b) mb = fmaxf(mb, m);
    else ma = fmaxf(ma, m);
  }
  for (int o = 16; o >= 1; o >>= 1) {
    ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, o));
    mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
  }
  if ((threadIdx.x & 31) == 0) {
    atomicMax(&p.amax_bits[0], __float_as_uint(ma));
    atomicMax(&p.amax_bits[1], __float_as_uint(mb));
  }
}

__device__ __forceinline__ float fp8_scale(unsigned int amax_bits) {
  const float amax = __uint_as_float(amax_bits);
  return amax > 0.f ? amax / kE4M3Max : 1.f;
}

__global__ void __launch_bounds__(kFp8Threads) fp8_quant_kernel(const Fp8QuantParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const float sa = fp8_scale(p.amax_bits[0]), sb = fp8_scale(p.amax_bits[1]);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    p.scales[0] = sa;
    p.scales[1] = sb;
  }
  const int cpr = p.cols / 8;
  const long long na8 = p.rows_a * cpr, n8 = na8 + p.rows_b * cpr;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long v = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; v < n8; v += stride) {
    const Fp8Vec e = fp8_vec(p, v, na8, cpr);
    const float s = e.is_b ? sb : sa;
    const uint4 u = __ldg(e.src);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(h2[j]);
      // t / s in float32 (a true division), then E4M3 round-to-nearest-even, saturating
      const uint32_t c0 = __nv_cvt_float_to_fp8(f.x / s, __NV_SATFINITE, __NV_E4M3);
      const uint32_t c1 = __nv_cvt_float_to_fp8(f.y / s, __NV_SATFINITE, __NV_E4M3);
      w[j >> 1] |= (c0 | (c1 << 8)) << ((j & 1) * 16);  // element 2j at byte 2j (little-endian)
    }
    uint2* dst = reinterpret_cast<uint2*>(e.is_b ? p.b8 : p.a8) + e.dst;
    *dst = make_uint2(w[0], w[1]);
  }
}

}  // namespace cswattn
