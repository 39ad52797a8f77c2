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
//   decode_attn: split-KV. CTA = (128-key chunk of the window, KV head,
//     sequence), 128 threads. TMA brings the chunk's K and V rows
//     (128B-swizzled panels, 32 KB each at head_dim 128) into shared memory
//     while the CTA computes the new token's prologue (the group's query
//     rows, in bf16 as the prologue stores them, into a 16-slot operand tile;
//     the chunk holding row p also its key and value rows, which it writes
//     to the caches and over the staged row). Both products run on the
//     tensor cores with the 16 head slots as N: S^T = K Q^T (M = 128 keys)
//     into TMEM; one thread per key reads its scores, masks, and the CTA
//     reduces the chunk's max and sum per head; the probabilities go to
//     shared memory as the bf16 operand P^T; O^T = V^T P^T (M = head_dim,
//     V read MN-major) into TMEM; one thread per column of O writes the
//     partial (max, sum, O) to the workspace. Three CTAs per SM keep their
//     tile copies in flight.
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

constexpr int kKeys = 128;      // keys per split (one CTA)
constexpr int kThreads = 128;   // one thread per key, then one per column of O
constexpr int kMaxGroup = 16;   // query heads per KV head handled by one CTA
constexpr int kSlots = 16;      // head slots: N of both tensor-core products
constexpr int kPanel = kKeys * 128;  // kKeys rows x 128 bytes

// Number of kKeys-key chunks a window of W keys (in a cache of T rows) can
// straddle: the chunks are aligned to absolute positions.
__host__ __device__ inline int decode_splits(int T, int W) {
  const int w = W < T ? W : T;
  const int n = (w + kKeys - 1) / kKeys + 1;
  const int cap = (T + kKeys - 1) / kKeys;
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

// Shared memory of decode_attn_kernel<D> (dynamic, 1 KB alignment slack).
// The two products' B operands are 16-row, K-major, 128B-swizzled tiles of
// 2 KB panels: Q (head slot x D) and P^T (head slot x 128 keys).
template <int D>
struct DecSmem {
  static constexpr int kTile = (D / 64) * kPanel;     // K or V: kKeys rows, D/64 swizzled panels
  static constexpr int kSPanel = kSlots * 128;        // 2 KB: 16 rows x 128 bytes
  static constexpr int kOffV = kTile;
  // V always spans two panels: the second product reads 128 rows of V^T
  // (at D = 64 the second panel is never loaded and its rows are unused).
  static constexpr int kOffQ = kOffV + 2 * kPanel;    // bf16 q~ rows, D/64 panels
  static constexpr int kOffP = kOffQ + (D / 64) * kSPanel;  // bf16 P^T, 2 panels (keys 0-63, 64-127)
  static constexpr int kOffRed = kOffP + 2 * kSPanel;  // float [16][4] warp partials
  static constexpr int kOffStat = kOffRed + kSlots * 4 * 4;  // float [16] chunk max
  static constexpr int kOffCS = kOffStat + kSlots * 4;       // float [D/2] cos, [D/2] sin
  static constexpr int kOffBar = kOffCS + D * 4;             // 4 mbarriers, TMEM slot, abort flag
  static constexpr int kBytes = kOffBar + 64 + 1024;
  static_assert(kOffQ % 1024 == 0 && kOffP % 1024 == 0, "operand tiles need 1024-byte alignment");
};

// Byte offset of element (row, col) of a 128B-swizzled K-major tile of
// 16-row panels (64 bf16 columns per panel).
__device__ __forceinline__ int slot_tile_ofs(int row, int col) {
  return (col >> 6) * (kSlots * 128) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2;
}

template <int D>
__global__ void __launch_bounds__(kThreads) decode_attn_kernel(const __grid_constant__ CUtensorMap tmK,
                                                               const __grid_constant__ CUtensorMap tmV,
                                                               const AttnParams p) {
  using SM = DecSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint8_t* sK = smem;
  uint8_t* sV = smem + SM::kOffV;
  uint8_t* sQ = smem + SM::kOffQ;
  uint8_t* sP = smem + SM::kOffP;
  float* red = reinterpret_cast<float*>(smem + SM::kOffRed);
  float* stat = reinterpret_cast<float*>(smem + SM::kOffStat);
  float* cs = reinterpret_cast<float*>(smem + SM::kOffCS);
  float* sn = cs + D / 2;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kOffBar);
  uint64_t* bar_k = bars;      // K tile landed
  uint64_t* bar_v = bars + 1;  // V tile landed
  uint64_t* bar_s = bars + 2;  // S^T = K Q^T done
  uint64_t* bar_o = bars + 3;  // O^T = V^T P^T done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 5);

  // KV head fastest: the CTAs reading the same cache rows run side by side.
  const int hk = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int g = p.g;
  pdl_launch_dependents();
  pdl_wait();
  const int pos = p.len[b];
  const bool in_range = pos >= 0 && pos < p.T;
  if (!in_range && split == 0 && hk == 0 && tid == 0) atomicOr(&g_status, kStatusRange);
  const int lo = in_range ? max(0, pos - p.W + 1) : 0;
  const int c0 = (lo / kKeys) * kKeys + split * kKeys;
  // A chunk with c0 <= pos holds at least one key of [lo, pos] (c0 <= lo + kKeys - 1).
  const bool work = in_range && c0 <= pos;
  const bool owns_new = work && pos < c0 + kKeys;  // this chunk holds the new token's row
  auto part = [&](int h) { return (static_cast<size_t>(b) * p.H + h) * p.nsplit + split; };
  if (!check_bounds(b < p.B && hk < p.Hk && split < p.nsplit && (hk + 1) * g <= p.H && g <= kSlots)) return;
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
    for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
    // Rows past T read as zero. Rows outside [lo, pos] may hold anything:
    // their scores are masked, and their V rows are zeroed before P V.
    mbar_expect_tx(bar_k, SM::kTile);
#pragma unroll
    for (int pn = 0; pn < D / 64; ++pn) tma_load_4d(&tmK, bar_k, sK + pn * kPanel, 64 * pn, hk, c0, b);
    mbar_expect_tx(bar_v, SM::kTile);
#pragma unroll
    for (int pn = 0; pn < D / 64; ++pn) tma_load_4d(&tmV, bar_v, sV + pn * kPanel, 64 * pn, hk, c0, b);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 32);  // columns 0-15: S^T (lane = key), 16-31: O^T (lane = column of O)
    tmem_relinquish();
  }
  // The new token's prologue at position pos while the tiles land.
  for (int i = tid; i < D / 2; i += blockDim.x) {
    float sv_, cv_;
    sincosf(static_cast<float>(pos) * p.omega[i], &sv_, &cv_);
    cs[i] = cv_;
    sn[i] = sv_;
  }
  for (int i = tid; i < (kSlots - g) * (D / 8); i += blockDim.x) {  // unused head slots: zero rows
    const int row = g + i / (D / 8), col = (i % (D / 8)) * 8;
    *reinterpret_cast<uint4*>(sQ + slot_tile_ofs(row, col)) = make_uint4(0u, 0u, 0u, 0u);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.wait_ns};

  // q~ rows of the group (bf16, as the prologue stores them) into the Q
  // tile; in the chunk holding row pos, k~ and v_eff to the caches (and,
  // once the tiles have landed, over row pos - c0 of the staged tiles).
  using NT = NewToken<D>;
  const int sub = tid % NT::LPR, grp = tid / NT::LPR;
  constexpr int kRowsPerPass = kThreads / NT::LPR;
  static_assert(NT::HV == 8, "one 16-byte chunk per half");
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
      uint4 u;
      u = make_uint4(pack_bf16x2(yl[0], yl[1]), pack_bf16x2(yl[2], yl[3]), pack_bf16x2(yl[4], yl[5]),
                     pack_bf16x2(yl[6], yl[7]));
      *reinterpret_cast<uint4*>(sQ + slot_tile_ofs(rr, sub * 8)) = u;
      u = make_uint4(pack_bf16x2(yh[0], yh[1]), pack_bf16x2(yh[2], yh[3]), pack_bf16x2(yh[4], yh[5]),
                     pack_bf16x2(yh[6], yh[7]));
      *reinterpret_cast<uint4*>(sQ + slot_tile_ofs(rr, NT::HALF + sub * 8)) = u;
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
  // Row pos of a staged tile (bf16, 128B-swizzled panels) takes the new
  // token's values: the copy brought in whatever the cache held there.
  auto put_row = [&](uint8_t* tile) {
    const int rr = pos - c0;
    auto put = [&](int d0, const float (&x)[NT::HV]) {
      const uint4 u = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                                 pack_bf16x2(x[6], x[7]));
      *reinterpret_cast<uint4*>(tile + (d0 >> 6) * kPanel + rr * 128 + ((((d0 & 63) >> 3) ^ (rr & 7)) << 4)) = u;
    };
    put(sub * NT::HV, kl);
    put(NT::HALF + sub * NT::HV, kh2);
  };

  bool issued_s = false, issued_o = false;
  bool ok = mbar_wait(bar_k, 0, wc);
  if (ok && have_k) put_row(sK);
  fence_proxy_async_smem();  // Q tile and the new K row, to the tensor cores' proxy
  ok = __syncthreads_and(ok);
  if (ok && tid == 0) {
    // S^T (128 keys x 16 slots) = K Q^T, K = D in steps of 16.
    tc_fence_after();
    constexpr uint32_t id = idesc_bf16(128, kSlots, 0, 0);
    const uint32_t k0 = smem_u32(sK), q0 = smem_u32(sQ);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t da = sdesc_sw128(k0 + (kk >> 2) * kPanel, 16, 1024) + static_cast<uint64_t>((kk & 3) * 2);
      const uint64_t db = sdesc_sw128(q0 + (kk >> 2) * SM::kSPanel, 16, 1024) + static_cast<uint64_t>((kk & 3) * 2);
      mma_ss(tmem, da, db, id, kk > 0 ? 1u : 0u);
    }
    mma_commit(bar_s);
    issued_s = true;
  }
  ok = ok && mbar_wait(bar_v, 0, wc);
  if (ok) {
    // Thread t owns row t of the V tile: rows outside [lo, pos] become zero
    // (probability 0 times a NaN would still be NaN in the product).
    const int j = c0 + tid;
    if (j < lo || j > pos) {
#pragma unroll
      for (int pn = 0; pn < D / 64; ++pn)
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(sV + pn * kPanel + tid * 128 + ((c ^ (tid & 7)) << 4)) =
              make_uint4(0u, 0u, 0u, 0u);  // chunk order rotated per row: no bank conflicts
    }
    if (have_v) put_row(sV);
  }
  ok = ok && mbar_wait(bar_s, 0, wc);
  ok = __syncthreads_and(ok);
  if (ok) {
    // Thread = key (TMEM lane): its scores in log2 units, masked by a select
    // (rows outside (pos - W, pos] may hold anything, NaN included).
    tc_fence_after();
    uint32_t sr[kSlots];
    tmem_ld16(tmem + (static_cast<uint32_t>(warp * 32) << 16), sr);
    tmem_ld_wait();
    const int r = tid, j = c0 + r;
    const bool key_ok = j >= lo && j <= pos;
    float sc[kSlots];
#pragma unroll
    for (int h = 0; h < kSlots; ++h) {
      sc[h] = key_ok ? __uint_as_float(sr[h]) * p.scale_log2 : -INFINITY;
      if (h < g) {
        float m = sc[h];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((tid & 31) == 0) red[h * 4 + warp] = m;
      }
    }
    __syncthreads();
    if (tid < g) stat[tid] = fmaxf(fmaxf(red[tid * 4], red[tid * 4 + 1]), fmaxf(red[tid * 4 + 2], red[tid * 4 + 3]));
    __syncthreads();
#pragma unroll
    for (int h = 0; h < kSlots; ++h) {
      // Probabilities (masked keys: exp2(-inf) = 0; unused slots: 0) as the
      // bf16 B operand P^T of the second product.
      const float e = h < g ? exp2f(sc[h] - stat[h]) : 0.f;
      *reinterpret_cast<__nv_bfloat16*>(sP + slot_tile_ofs(h, r)) = __float2bfloat16_rn(e);
      if (h < g) {
        float sum = e;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if ((tid & 31) == 0) red[h * 4 + warp] = sum;
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid < g) {
      p.part_ml[part(hk * g + tid) * 2] = stat[tid];
      p.part_ml[part(hk * g + tid) * 2 + 1] = (red[tid * 4] + red[tid * 4 + 1]) + (red[tid * 4 + 2] + red[tid * 4 + 3]);
    }
    if (tid == 0) {
      // O^T (D x 16 slots) = V^T P^T, K = 128 keys in steps of 16. V^T is
      // the V tile read MN-major (64-column panels kPanel apart); at D = 64
      // the second 64 rows of the product read other shared memory and are
      // never loaded back.
      tc_fence_after();
      constexpr uint32_t id = idesc_bf16(128, kSlots, 1, 0);
      const uint32_t v0 = smem_u32(sV), p0 = smem_u32(sP);
      const uint64_t dv = sdesc_sw128(v0, kPanel, 1024);
#pragma unroll
      for (int kk = 0; kk < kKeys / 16; ++kk) {
        const uint64_t db = sdesc_sw128(p0 + (kk >> 2) * SM::kSPanel, 16, 1024) + static_cast<uint64_t>((kk & 3) * 2);
        mma_ss(tmem + kSlots, dv + static_cast<uint64_t>((kk * 16 * 128) >> 4), db, id, kk > 0 ? 1u : 0u);
      }
      mma_commit(bar_o);
      issued_o = true;
    }
    ok = __syncthreads_and(mbar_wait(bar_o, 0, wc));
    if (ok) {
      // Thread = column d of O (TMEM lane): the group's partial outputs.
      tc_fence_after();
      uint32_t orr[kSlots];
      tmem_ld16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + kSlots, orr);
      tmem_ld_wait();
      const int d = tid;
      if (d < D) {
#pragma unroll
        for (int h = 0; h < kSlots; ++h)
          if (h < g) p.part_o[part(hk * g + h) * D + d] = __uint_as_float(orr[h]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (!ok && tid == 0) {
    // A wait ran out: the copies and products in flight land before the
    // CTA exits and frees its TMEM.
    drain_wait(bar_k, 0);
    drain_wait(bar_v, 0);
    if (issued_s) drain_wait(bar_s, 0);
    if (issued_o) drain_wait(bar_o, 0);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
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
