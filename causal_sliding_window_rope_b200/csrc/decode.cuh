// decode.cuh -- one generation step with a key/value cache (bf16).
//
// Page "5만원으로 나만의 ChatGPT 훈련하는 방법", section "6. 추론 엔진
// (nanochat/engine.py)": generation attends over a pre-filled KV cache
// (flash_attn_with_kvcache). Same layer as the training path (section
// "1. GPT 모델": RoPE, QK normalisation, GQA, sliding window, value
// embedding), with one new token per sequence:
//   p = len[b] (tokens already cached), the new token's position;
//   q~ = RoPE_p(n(q)), k~ = RoPE_p(n(k)), v_eff = v + 3 sigmoid(gate) ve;
//   k~, v_eff are written to the caches at row p;
//   O_h = sum_j softmax_j(c q~_h . k~_j) v_eff_j over cache rows (p - W, p].
//
// The step reads the window of the K/V cache once: it is bound by HBM
// bandwidth, not by the tensor cores (one query row per head). Two kernels:
//   decode_attn: split-KV. CTA = (64-key chunk of the window, KV head,
//     sequence), small enough that several CTAs per SM keep their copies in
//     flight: TMA brings the chunk's K and V rows (128B-swizzled panels)
//     into shared memory while the CTA computes the new token's prologue
//     (its query rows of this KV head; the chunk holding row p also its key
//     and value rows, which it writes to the caches and over the staged
//     row); two threads per key score it against the g query
//     heads of the group (half of head_dim each), the CTA reduces the chunk's
//     max and sum per head, and each thread accumulates two columns of P V
//     over half of the keys; the partial (max, sum, O) goes to the workspace;
//   decode_combine: one CTA per (sequence, query head) merges the chunks'
//     partials (rescaled by exp(m_s - M)) into O and lse.
// A cache length outside [0, T) is reported through the status word
// (CSWATTN_ERR_INVALID_ARG at the next status check) and that sequence is
// left untouched.
#pragma once
#include "prologue.cuh"

namespace cswattn {

constexpr unsigned int kStatusRange = 8u;

namespace dec {

constexpr int kChunk = 64;      // keys per split
constexpr int kThreads = 128;
constexpr int kMaxGroup = 16;   // query heads per KV head handled by one CTA
constexpr int kPanel = kChunk * 128;  // kChunk rows x 128 bytes

// Number of kChunk-key chunks a window of W keys (in a cache of T rows) can
// straddle: the chunks are aligned to absolute positions.
__host__ __device__ inline int decode_splits(int T, int W) {
  const int w = W < T ? W : T;
  const int n = (w + kChunk - 1) / kChunk + 1;
  const int cap = (T + kChunk - 1) / kChunk;
  return n < cap ? n : cap;
}

struct AttnParams {
  int B, T, H, Hk, W, g, nsplit, has_ve;
  float scale_log2;  // softmax scale * log2(e)
  float eps;
  float omega[kMaxHalfD];                      // rope_base^(-2i/D)
  const int* len;                              // (B) tokens already cached
  const __nv_bfloat16 *q, *k, *v, *ve, *gate;  // (B,H,D), (B,Hk,D), (B,Hk)
  __nv_bfloat16 *kc, *vc;                      // (B,T,Hk,D) caches
  float* part_ml;     // (B,H,nsplit,2): running max (log2 units), sum
  float* part_o;      // (B,H,nsplit,D): unnormalised partial O
  unsigned long long wait_ns;
};

// Prologue of one row of the new token (page section "1. GPT 모델": QK
// RMSNorm, RoPE at the token's position, value residual), in the row
// kernels' split-halves layout: lane `sub` of the row's LPR lanes holds
// elements [sub HV, (sub+1) HV) of both halves. kind 0: query head (scaled
// by c log2(e) into shared fp32), 1: key (RMSNorm + RoPE), 2: value
// (v + 3 sigmoid(gate) ve); kinds 1 and 2 return their bf16 halves.
template <int D>
struct NewToken {
  using RL = RowLayout<__nv_bfloat16, D>;
  using HVec = HalfVec<__nv_bfloat16, RL::HV>;
  static constexpr int HV = RL::HV, LPR = RL::LPR, HALF = RL::HALF;

  __device__ static void row(const AttnParams& p, int b, int kind, int head, int sub, bool valid,
                             const float* cs, const float* sn, float (&yl)[HV], float (&yh)[HV]) {
    const int nh = kind == 0 ? p.H : p.Hk;
    const size_t src = (static_cast<size_t>(b) * nh + head) * D + sub * HV;
    const __nv_bfloat16* x = kind == 0 ? p.q : (kind == 1 ? p.k : p.v);
    float xl[HV], xh[HV];
    if (valid) {
      HVec::load(x + src, xl);
      HVec::load(x + src + HALF, xh);
    } else {
#pragma unroll
      for (int i = 0; i < HV; ++i) xl[i] = xh[i] = 0.f;
    }
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < HV; ++i) ss = fmaf(xl[i], xl[i], fmaf(xh[i], xh[i], ss));
    ss = row_sum<LPR>(ss);
    if (kind == 2) {
      float coef = 0.f;
      if (valid && p.has_ve) {
        coef = 3.0f / (1.0f + expf(-__bfloat162float(p.gate[static_cast<size_t>(b) * p.Hk + head])));
        float el[HV], eh[HV];
        HVec::load(p.ve + src, el);
        HVec::load(p.ve + src + HALF, eh);
#pragma unroll
        for (int i = 0; i < HV; ++i) {
          xl[i] = fmaf(coef, el[i], xl[i]);
          xh[i] = fmaf(coef, eh[i], xh[i]);
        }
      }
#pragma unroll
      for (int i = 0; i < HV; ++i) {
        yl[i] = xl[i];
        yh[i] = xh[i];
      }
      return;
    }
    const float rstd = rsqrtf(ss / static_cast<float>(D) + p.eps);
#pragma unroll
    for (int i = 0; i < HV; ++i) {
      const float c = cs[sub * HV + i], s = sn[sub * HV + i];
      const float nl = xl[i] * rstd, nh2 = xh[i] * rstd;
      yl[i] = fmaf(nl, c, -nh2 * s);
      yh[i] = fmaf(nl, s, nh2 * c);
    }
  }
};

// Shared memory of decode_attn_kernel<D> (dynamic, with 1 KB of alignment slack).
template <int D>
constexpr int decode_attn_smem() {
  return 4 * kPanel + (kMaxGroup * D + kMaxGroup * kChunk + kMaxGroup * D + kMaxGroup * 6 + D) * 4 + 1024;
}

template <int D>
__global__ void __launch_bounds__(kThreads) decode_attn_kernel(const __grid_constant__ CUtensorMap tmK,
                                                               const __grid_constant__ CUtensorMap tmV,
                                                               const AttnParams p) {
  static_assert(kThreads == 2 * kChunk && kThreads == D || kThreads == 2 * D, "thread mapping");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint8_t* sK = smem;                   // 2 panels
  uint8_t* sV = smem + 2 * kPanel;      // 2 panels
  float* sq = reinterpret_cast<float*>(smem + 4 * kPanel);  // [g][D], scaled by c log2(e)
  float* sp = sq + kMaxGroup * D;                            // [g][kChunk] scores -> probabilities
  float* so = sp + kMaxGroup * kChunk;                       // [g][D] second half of P V
  float* red = so + kMaxGroup * D;                           // [g][4] warp partials
  float* stat = red + kMaxGroup * 4;                         // [g][2] max, sum
  float* cs = stat + kMaxGroup * 2;                          // [D/2] cos(p omega_i)
  float* sn = cs + D / 2;                                    // [D/2] sin(p omega_i)
  __shared__ uint64_t bar;

  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = p.g;
  pdl_launch_dependents();
  pdl_wait();
  const int pos = p.len[b];
  const bool in_range = pos >= 0 && pos < p.T;
  if (!in_range && split == 0 && hk == 0 && tid == 0) atomicOr(&g_status, kStatusRange);
  const int lo = in_range ? max(0, pos - p.W + 1) : 0;
  const int c0 = (lo / kChunk) * kChunk + split * kChunk;
  const bool work = in_range && c0 <= pos;
  const bool owns_new = work && pos < c0 + kChunk;  // this chunk holds the new token's row
  auto part = [&](int h) { return (static_cast<size_t>(b) * p.H + h) * p.nsplit + split; };
  if (!check_bounds(b < p.B && hk < p.Hk && split < p.nsplit && (hk + 1) * g <= p.H)) return;
  if (!work) {
    // Empty chunk: a partial that the combine step ignores.
    for (int i = tid; i < g * D; i += blockDim.x) p.part_o[part(hk * g + i / D) * D + i % D] = 0.f;
    if (tid < g) {
      p.part_ml[part(hk * g + tid) * 2] = -INFINITY;
      p.part_ml[part(hk * g + tid) * 2 + 1] = 0.f;
    }
    return;
  }
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    fence_proxy_async_smem();
    mbar_expect_tx(&bar, 4 * kPanel);
    // Rows past T read as zero; rows past pos are masked below.
    tma_load_4d(&tmK, &bar, sK, 0, hk, c0, b);
    tma_load_4d(&tmK, &bar, sK + kPanel, 64, hk, c0, b);
    tma_load_4d(&tmV, &bar, sV, 0, hk, c0, b);
    tma_load_4d(&tmV, &bar, sV + kPanel, 64, hk, c0, b);
  }
  // The new token's prologue at position pos: its g query rows of this KV
  // head (into sq, scaled by c log2(e)), and, in the chunk that holds row
  // pos, its key and value rows (written to the caches and, after the chunk
  // has landed, over row pos - c0 of the staged tiles).
  using NT = NewToken<D>;
  for (int i = tid; i < D / 2; i += blockDim.x) {
    float sv_, cv_;
    sincosf(static_cast<float>(pos) * p.omega[i], &sv_, &cv_);
    cs[i] = cv_;
    sn[i] = sv_;
  }
  __syncthreads();
  const int sub = tid % NT::LPR, grp = tid / NT::LPR;
  constexpr int kRowsPerPass = kThreads / NT::LPR;
  float kl[NT::HV], kh2[NT::HV];
  bool have_k = false, have_v = false;
  for (int base = 0; base < g + 2; base += kRowsPerPass) {
    const int rr = base + grp;
    const int kind = rr < g ? 0 : (rr == g ? 1 : 2);
    const bool valid = rr < g || (owns_new && rr < g + 2);
    float yl[NT::HV], yh[NT::HV];
    NT::row(p, b, kind, kind == 0 ? hk * g + rr : hk, sub, valid, cs, sn, yl, yh);
    if (!valid) continue;
    if (kind == 0) {
#pragma unroll
      for (int i = 0; i < NT::HV; ++i) {
        sq[rr * D + sub * NT::HV + i] = yl[i] * p.scale_log2;
        sq[rr * D + NT::HALF + sub * NT::HV + i] = yh[i] * p.scale_log2;
      }
    } else {
      const size_t crow = ((static_cast<size_t>(b) * p.T + pos) * p.Hk + hk) * D + sub * NT::HV;
      __nv_bfloat16* cache = kind == 1 ? p.kc : p.vc;
      NT::HVec::store(cache + crow, yl);
      NT::HVec::store(cache + crow + NT::HALF, yh);
#pragma unroll
      for (int i = 0; i < NT::HV; ++i) {
        kl[i] = yl[i];
        kh2[i] = yh[i];
      }
      have_k = kind == 1;
      have_v = kind == 2;
    }
  }
  __syncthreads();
  {
    bool ok = mbar_try_wait(&bar, 0);
    const uint64_t t0 = globaltimer();
    while (!ok) {
      ok = mbar_try_wait(&bar, 0);
      if (!ok && globaltimer() - t0 > p.wait_ns) {
        atomicOr(&g_status, kStatusTimeout);
        drain_wait(&bar, 0);  // the tile copies land before the CTA exits
        break;
      }
    }
    if (!__syncthreads_and(ok)) return;
  }
  if (have_k || have_v) {
    // Row pos of the staged tile (bf16, 128B-swizzled panels) gets the new
    // token's values: the copy brought in whatever the cache held there.
    const int rr = pos - c0;
    uint8_t* tile = have_k ? sK : sV;
    auto put = [&](int d0, const float (&x)[NT::HV]) {
      uint4 u;
      uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) w[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
      *reinterpret_cast<uint4*>(tile + (d0 >> 6) * kPanel + rr * 128 + ((((d0 & 63) >> 3) ^ (rr & 7)) << 4)) = u;
    };
    static_assert(NT::HV == 8, "one 16-byte chunk per half");
    put(sub * NT::HV, kl);
    put(NT::HALF + sub * NT::HV, kh2);
  }
  __syncthreads();

  // Scores (log2 units): threads 2r and 2r+1 take key r = tid / 2, each half
  // of its columns (one 128-byte panel of D = 128, half a panel of D = 64).
  const int r = tid >> 1, half = tid & 1;
  const int j = c0 + r;
  const bool key_ok = j >= lo && j <= pos;
  {
    constexpr int kChunks = D / 16;  // 16-byte chunks per half row
    float acc[kMaxGroup];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) acc[h] = 0.f;
#pragma unroll
    for (int cc = 0; cc < kChunks; ++cc) {
      const int c = half * kChunks + cc;  // 16-byte chunk of the row
      const uint8_t* row = sK + (c >> 3) * kPanel + r * 128;
      const uint4 u = *reinterpret_cast<const uint4*>(row + (((c & 7) ^ (r & 7)) << 4));
      const __nv_bfloat162* kv = reinterpret_cast<const __nv_bfloat162*>(&u);
      float kf[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(kv[e]);
        kf[2 * e] = f.x;
        kf[2 * e + 1] = f.y;
      }
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) {
        if (h >= g) break;
        const float4 qa = *reinterpret_cast<const float4*>(sq + h * D + c * 8);
        const float4 qb = *reinterpret_cast<const float4*>(sq + h * D + c * 8 + 4);
        acc[h] = fmaf(qa.x, kf[0], fmaf(qa.y, kf[1], fmaf(qa.z, kf[2], fmaf(qa.w, kf[3], acc[h]))));
        acc[h] = fmaf(qb.x, kf[4], fmaf(qb.y, kf[5], fmaf(qb.z, kf[6], fmaf(qb.w, kf[7], acc[h]))));
      }
    }
    // Whole-row scores, then the chunk max per head.
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
      if (h >= g) break;
      float s = acc[h] + __shfl_xor_sync(0xffffffffu, acc[h], 1);
      s = key_ok ? s : -INFINITY;
      if (half == 0) sp[h * kChunk + r] = s;
      float m = s;
#pragma unroll
      for (int o = 16; o >= 2; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) red[h * 4 + warp] = m;
    }
  }
  __syncthreads();
  if (tid < g) stat[tid * 2] = fmaxf(fmaxf(red[tid * 4], red[tid * 4 + 1]), fmaxf(red[tid * 4 + 2], red[tid * 4 + 3]));
  __syncthreads();
  // Probabilities relative to the chunk max (thread tid < kChunk: key tid),
  // and their sum per head.
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    if (h >= g) break;
    const float m = stat[h * 2];
    float e = 0.f;
    if (tid < kChunk) {
      const int jj = c0 + tid;
      e = (jj >= lo && jj <= pos) ? exp2f(sp[h * kChunk + tid] - m) : 0.f;
      sp[h * kChunk + tid] = e;
    }
    float s = e;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) red[h * 4 + warp] = s;
  }
  __syncthreads();
  if (tid < g) {
    stat[tid * 2 + 1] = (red[tid * 4] + red[tid * 4 + 1]) + (red[tid * 4 + 2] + red[tid * 4 + 3]);
    p.part_ml[part(hk * g + tid) * 2] = stat[tid * 2];
    p.part_ml[part(hk * g + tid) * 2 + 1] = stat[tid * 2 + 1];
  }
  // P V: thread (column pair cp, key part kh) sums its part of the keys for
  // columns 2cp, 2cp+1. Rows past pos are never read (they may hold anything);
  // rows before the window start are earlier tokens' rows, weighted by 0.
  {
    constexpr int kPairs = D / 2;
    constexpr int kKeyParts = kThreads / kPairs;  // 2 (D = 128) or 4 (D = 64)
    constexpr int kKeys = kChunk / kKeyParts;
    const int cp = tid % kPairs, kh = tid / kPairs;
    const int d = 2 * cp, pan = d >> 6, ch = (d & 63) >> 3, el = d & 7;
    float o0[kMaxGroup], o1[kMaxGroup];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) o0[h] = o1[h] = 0.f;
#pragma unroll 8
    for (int rr = 0; rr < kKeys; ++rr) {
      const int row = kh * kKeys + rr;
      if (c0 + row > pos) break;
      const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(
          sV + pan * kPanel + row * 128 + ((ch ^ (row & 7)) << 4) + el * 2));
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) {
        if (h >= g) break;
        const float pr = sp[h * kChunk + row];
        o0[h] = fmaf(pr, v.x, o0[h]);
        o1[h] = fmaf(pr, v.y, o1[h]);
      }
    }
    // Sum the key parts through shared memory (part 0 collects).
    for (int q = 1; q < kKeyParts; ++q) {
      if (kh == q) {
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
          if (h >= g) break;
          so[h * D + d] = o0[h];
          so[h * D + d + 1] = o1[h];
        }
      }
      __syncthreads();
      if (kh == 0) {
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
          if (h >= g) break;
          o0[h] += so[h * D + d];
          o1[h] += so[h * D + d + 1];
        }
      }
      __syncthreads();
    }
    if (kh == 0) {
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) {
        if (h >= g) break;
        *reinterpret_cast<float2*>(p.part_o + part(hk * g + h) * D + d) = make_float2(o0[h], o1[h]);
      }
    }
  }
}

struct CombineParams {
  int B, H, nsplit;
  const int* len;
  int T;
  const float* part_ml;
  const float* part_o;
  __nv_bfloat16* O;  // (B,H,D)
  float* lse;        // (B,H) natural log
};

template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const CombineParams p) {
  const int bh = blockIdx.x, b = bh / p.H, d = threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  const int pos = p.len[b];
  if (pos < 0 || pos >= p.T) return;
  const float* ml = p.part_ml + static_cast<size_t>(bh) * p.nsplit * 2;
  float M = -INFINITY;
#pragma unroll 8
  for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, ml[2 * s]);
  float L = 0.f, o = 0.f;
#pragma unroll 8
  for (int s = 0; s < p.nsplit; ++s) {
    if (ml[2 * s] == -INFINITY) continue;
    const float w = exp2f(ml[2 * s] - M);
    L = fmaf(ml[2 * s + 1], w, L);
    o = fmaf(p.part_o[(static_cast<size_t>(bh) * p.nsplit + s) * D + d], w, o);
  }
  p.O[static_cast<size_t>(bh) * D + d] = __float2bfloat16_rn(o / L);
  if (d == 0) p.lse[bh] = (M + log2f(L)) * 0.69314718055994531f;
}

}  // namespace dec
}  // namespace cswattn
