// qkv_sm100.cuh -- the QKV projection fused with the attention prologue, on
// tcgen05 tensor cores (bf16).
//
// Page "5만원으로 나만의 ChatGPT 훈련하는 방법", section "1. GPT 모델
// (nanochat/gpt.py)": the block input x is projected to the query, key and
// value heads (bias-free linear maps, the model's Linear layers), then the
// prologue of the attention applies QK RMSNorm and RoPE (architecture list)
// and the value residual v + 3 sigmoid(gate) ve (value-embedding code):
//   y = x W^T with W = [W_q; W_k; W_v] ((H + 2 Hk) D x C), per head
//   q (raw, bf16) and q~ = RoPE(RMSNorm(q)), likewise k; v_eff = v + 3 s ve.
//
// FP8 variant (section "3. 정밀도 관리": Float8Linear with tensor-wise
// scaling): x and W arrive as E4M3 codes with one scale each, the products
// are tcgen05.mma kind::f8f6f4 (K = 32 per instruction, 128-element chunks),
// and the accumulator is multiplied by the two scales before the epilogue.
//
// One CTA per (128-token tile, pair of stacked heads): the heads' 2 D output
// columns are one N = 2 D tile of the product (two heads per tile halve the
// operand bytes per product, which bound a one-head tile), and each epilogue
// thread holds whole head rows (RMSNorm and the RoPE pairs (i, i + D/2) are
// in-thread). Warp 0 loads 64-wide chunks of x (128 tokens) and of the
// heads' 2 D rows of W by TMA into a 3-stage ring; warp 1 issues tcgen05.mma
// (M = 128, N = 2 D, K = 16) into a TMEM accumulator; warps 2-5 fill a
// cos/sin table of the tile's positions while the products run, then, head
// by head, read the accumulator (thread = token row), round the projection
// to bf16 (the value the backward sees as q or k), normalise and rotate it
// (or form v_eff) and stage the rows in shared memory (the ring, free after
// the products) for TMA stores over the flattened (B*T) token dimension.
#pragma once
#include "common.cuh"

namespace cswattn {
namespace qkv {

constexpr int kBM = 128, kBK = 64;
constexpr int kNH = 2;  // stacked heads per CTA
constexpr int kThreads = 192;
constexpr int kStages = 3;
constexpr int kXBytes = kBM * kBK * 2;        // 16 KB: 128 tokens x 64 channels (128 bytes a row)
constexpr int kWBytes = kNH * 128 * kBK * 2;  // 32 KB: up to 2 x 128 weight rows x 128 bytes
constexpr int kStageBytes = kXBytes + kWBytes;
constexpr int kHeadStage = 4 * kBM * 128;     // output staging of one head: raw and final rows, 2 panels each
static_assert(kNH * kHeadStage <= kStages * kStageBytes, "output staging fits in the ring");
constexpr int kOffTab = kStages * kStageBytes;         // cos/sin table [64][128] x 2, float32
constexpr int kOffBar = kOffTab + 2 * kBM * 64 * 4;
constexpr int kSmemBytes = kOffBar + 256 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per block");

struct Params {
  int BT, T, H, Hk, C;
  int has_ve;
  float eps;
  float omega[64];               // rope_base^(-2i/D), i < D/2
  const __nv_bfloat16* ve;       // (B*T, Hk, D)
  const __nv_bfloat16* gate;     // (B*T, Hk) logits
  float* rstd_q;                 // (B*T, H)
  float* rstd_k;                 // (B*T, Hk)
  const float* scales;           // FP8 variant: scale of x, scale of W
  unsigned long long wait_ns;
};

// Stages a row's D values (bf16) as D/64 swizzled 128-byte panels of a
// 128-row staging tile (the layout of the output tensor maps).
template <int HD>
__device__ __forceinline__ void stage_row(uint8_t* tile, int r, const float* v) {
#pragma unroll
  for (int k = 0; k < HD / 8; ++k) {  // 16-byte chunk k of the row
    uint4 w;
    w.x = pack_bf16x2(v[8 * k + 0], v[8 * k + 1]);
    w.y = pack_bf16x2(v[8 * k + 2], v[8 * k + 3]);
    w.z = pack_bf16x2(v[8 * k + 4], v[8 * k + 5]);
    w.w = pack_bf16x2(v[8 * k + 6], v[8 * k + 7]);
    *reinterpret_cast<uint4*>(tile + (k >> 3) * (kBM * 128) + r * 128 + (((k & 7) ^ (r & 7)) << 4)) = w;
  }
}

// tmX: x as (C, B*T), 128-byte x 128-row boxes. tmW: W as (C, (H+2Hk) D),
// 128-byte x 2 HD-row boxes (64 bf16 or 128 E4M3 channels per box).
// tmQ/tmK/tmQo/tmKo/tmVo: the outputs as (D, heads, B*T), 64 x 1 x 128
// boxes.
template <int HD, bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    qkv_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
               const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmQo, const __grid_constant__ CUtensorMap tmKo,
               const __grid_constant__ CUtensorMap tmVo, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  pdl_launch_dependents();
  uint8_t* smem = smem_align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full = bars;             // [kStages]
  uint64_t* empty = bars + kStages;  // [kStages]
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* staged = bars + 2 * kStages + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * kStages + 3);
  float* tcos = reinterpret_cast<float*>(smem + kOffTab);  // [64 frequencies][128 rows]: a warp's rows in distinct banks
  float* tsin = tcos + kBM * 64;
  const int warp = warp_id(), lane = lane_id();
  const int nh = p.H + 2 * p.Hk;
  const int hh0 = static_cast<int>(blockIdx.x) * kNH;  // first stacked head: q heads, then k, then v
  const int m0 = static_cast<int>(blockIdx.y) * kBM;
  constexpr int kChunk = FP8 ? 2 * kBK : kBK;  // channels per stage (128 bytes per row)
  constexpr int kNCols = kNH * HD;             // N of the product, TMEM columns
  const int nk = (p.C + kChunk - 1) / kChunk;
  if (!check_bounds(m0 < p.BT && hh0 < nh && nk >= 1)) return;  // checked build

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(staged, 128);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kNCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  const WaitCtx wc{abort_flag, p.wait_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      prefetch_tmap(&tmX);
      prefetch_tmap(&tmW);
      int issued[kStages] = {};
      for (int kc = 0; kc < nk; ++kc) {
        const int s = kc % kStages, use = kc / kStages;
        if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1, wc)) break;
        uint8_t* st = smem + s * kStageBytes;
        mbar_expect_tx(&full[s], kXBytes + kNCols * 128);  // rows past the last head read as zero
        tma_load_2d(&tmX, &full[s], st, kc * kChunk, m0);
        tma_load_2d(&tmW, &full[s], st + kXBytes, kc * kChunk, hh0 * HD);
        ++issued[s];
      }
      for (int s = 0; s < kStages; ++s)
        if (issued[s] > 0) drain_wait(&full[s], (issued[s] - 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t id = FP8 ? idesc_e4m3(128, kNCols, 0, 0) : idesc_bf16(128, kNCols, 0, 0);  // x W^T
      const uint32_t s0 = smem_u32(smem);
      for (int kc = 0; kc < nk; ++kc) {
        const int s = kc % kStages, use = kc / kStages;
        if (!mbar_wait(&full[s], use & 1, wc)) break;
        tc_fence_after();
        const uint64_t da = sdesc_sw128(s0 + s * kStageBytes, 16, 1024);
        const uint64_t db = sdesc_sw128(s0 + s * kStageBytes + kXBytes, 16, 1024);
        // Four K-steps of 32 bytes per 128-byte row: 16 bf16 or 32 E4M3 channels each.
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          if constexpr (FP8)
            mma_ss_f8(tmem, da + static_cast<uint64_t>(kk * 2), db + static_cast<uint64_t>(kk * 2), id,
                      (kc > 0 || kk > 0) ? 1u : 0u);
          else
            mma_ss(tmem, da + static_cast<uint64_t>(kk * 2), db + static_cast<uint64_t>(kk * 2), id,
                   (kc > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
      }
      mma_commit(acc_full);  // also the drain: every issued product completes before it fires
      drain_wait(acc_full, 0);
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2-5)
    const int quad = warp & 3;  // TMEM lanes 32 quad .. 32 quad + 31
    const int r = quad * 32 + lane;
    const int m = m0 + r;       // flattened token (b T + t)
    const bool row_ok = m < p.BT;
    constexpr int HALF = HD / 2;
    auto kind_of = [&](int hh) { return hh < p.H ? 0 : (hh < p.H + p.Hk ? 1 : 2); };
    auto head_of = [&](int hh) { return hh < p.H ? hh : (hh < p.H + p.Hk ? hh - p.H : hh - p.H - p.Hk); };
    if (kind_of(hh0) != 2) {
      // cos/sin of this row's position, while the products run
      const float t = static_cast<float>(row_ok ? m % p.T : 0);
      for (int i = 0; i < HALF; ++i) {
        float sn, cs;
        sincosf(t * p.omega[i], &sn, &cs);
        tcos[i * kBM + r] = cs;
        tsin[i * kBM + r] = sn;
      }
    }
    const bool got = mbar_wait(acc_full, 0, wc);
    if (__all_sync(0xffffffffu, got)) {
      tc_fence_after();
      const float sxw = FP8 ? p.scales[0] * p.scales[1] : 1.f;
#pragma unroll 1
      for (int hi = 0; hi < kNH; ++hi) {
        const int hh = hh0 + hi;
        if (hh >= nh) break;  // an odd head count: the last pair has one head
        const int kind = kind_of(hh), head = head_of(hh);
        float y[HD];
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t a[32];
          tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + hi * HD + c * 32, a);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i)  // the projection as stored (bf16)
            y[32 * c + i] = __bfloat162float(__float2bfloat16_rn(__uint_as_float(a[i]) * sxw));
        }
        uint8_t* raw_tile = smem + hi * kHeadStage;                 // raw q or k rows (HD / 64 panels)
        uint8_t* out_tile = smem + hi * kHeadStage + 2 * kBM * 128;  // q~, k~ or v_eff rows
        if (kind == 2) {
          float coef = 0.f;
          if (p.has_ve && row_ok) {
            coef = 3.0f / (1.0f + expf(-__bfloat162float(p.gate[static_cast<size_t>(m) * p.Hk + head])));
            const uint4* ep = reinterpret_cast<const uint4*>(p.ve + (static_cast<size_t>(m) * p.Hk + head) * HD);
#pragma unroll
            for (int q = 0; q < HD / 8; ++q) {
              const uint4 u = __ldg(ep + q);
              const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                y[8 * q + 2 * e] = fmaf(coef, f.x, y[8 * q + 2 * e]);
                y[8 * q + 2 * e + 1] = fmaf(coef, f.y, y[8 * q + 2 * e + 1]);
              }
            }
          }
          stage_row<HD>(out_tile, r, y);
        } else {
          stage_row<HD>(raw_tile, r, y);
          float ss = 0.f;
#pragma unroll
          for (int i = 0; i < HD; ++i) ss = fmaf(y[i], y[i], ss);
          const float rstd = rsqrtf(ss / static_cast<float>(HD) + p.eps);
#pragma unroll
          for (int i = 0; i < HALF; ++i) {
            const float cs = tcos[i * kBM + r], sn = tsin[i * kBM + r];
            const float nl = y[i] * rstd, nh2 = y[i + HALF] * rstd;
            y[i] = fmaf(nl, cs, -nh2 * sn);
            y[i + HALF] = fmaf(nl, sn, nh2 * cs);
          }
          stage_row<HD>(out_tile, r, y);
          if (row_ok) (kind == 0 ? p.rstd_q[static_cast<size_t>(m) * p.H + head]
                                 : p.rstd_k[static_cast<size_t>(m) * p.Hk + head]) = rstd;
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(staged);
      if (r == 0 && mbar_wait(staged, 0, wc)) {
        for (int hi = 0; hi < kNH && hh0 + hi < nh; ++hi) {
          const int kind = kind_of(hh0 + hi), head = head_of(hh0 + hi);
          const uint8_t* raw_tile = smem + hi * kHeadStage;
          const uint8_t* out_tile = smem + hi * kHeadStage + 2 * kBM * 128;
#pragma unroll
          for (int pn = 0; pn < HD / 64; ++pn) {
            const int col = 64 * pn;
            if (kind == 0) {
              tma_store_3d(&tmQ, raw_tile + pn * (kBM * 128), col, head, m0);
              tma_store_3d(&tmQo, out_tile + pn * (kBM * 128), col, head, m0);
            } else if (kind == 1) {
              tma_store_3d(&tmK, raw_tile + pn * (kBM * 128), col, head, m0);
              tma_store_3d(&tmKo, out_tile + pn * (kBM * 128), col, head, m0);
            } else {
              tma_store_3d(&tmVo, out_tile + pn * (kBM * 128), col, head, m0);
            }
          }
        }
        bulk_commit();
        bulk_wait_read0();  // shared source read; the writes finish on their own
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kNCols);
  }
}

}  // namespace qkv
}  // namespace cswattn
