// fwd_sm100.cuh -- attention forward on tcgen05 tensor cores (bf16, D = 128 or 64).
//
// Computes O_i = sum_j softmax_j(c q~_i . k~_j) v_eff_j over the causal
// sliding window (i - W < j <= i) and the row log-sum-exp, the attention
// call of the page "5만원으로 나만의 ChatGPT 훈련하는 방법", section
// "5. 플래시 어텐션 통합 (nanochat/flash_attention.py)", with the window of
// the architecture list's "sliding window attention" and its GQA.
//
// Work unit (one CTA): two 128-row query tiles of the same (batch, KV head)
// that share every K/V tile staged in shared memory. Tiles of a (b, KV head)
// are ordered (query block, head within the group) and paired in that order,
// so for group size >= 2 a unit holds two heads of the group at the same
// query block (identical KV range) and for group size 1 two consecutive
// query blocks (the union of their ranges; each tile skips the KV tiles
// outside its own range). Only KV tiles inside [first window key, diagonal]
// are loaded and multiplied; masks are applied on the diagonal and
// window-edge tiles only.
//
// Roles (12 warps):
//   warp 0      TMA producer: Q tiles once, then K_j, V_j through one 5-slot ring
//   warp 1      TMEM owner + single-thread MMA issuer
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1: thread r
//               owns TMEM lane r = query row r, so the row max and sum are
//               in-thread; P goes back to TMEM as bf16 over the S columns.
//               At the end each warpgroup stages its O tile (bf16) in its
//               Q buffer and writes it with two TMA stores.
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each.
// Per KV tile: S_X = Q_X K_j^T (SS MMA, K-major both), softmax -> P_X,
// O_X += P_X V_j (TS MMA: P from TMEM, V MN-major from shared memory).
// The MMA order PV_0(j), S_0(j+1), PV_1(j), S_1(j+1) lets one tile's softmax
// overlap the other tile's matrix products. O is rescaled lazily: only when
// a row's max grows by more than 2^8 (in exp2 units).
#pragma once
#include "common.cuh"

namespace cswattn {
namespace fwd {

constexpr int kBM = 128;
constexpr int kD = 128;
constexpr int kThreads = 384;
constexpr int kTileBytes = kBM * kD * 2;     // 32 KB: 128 rows x 128 bf16
constexpr int kPanelBytes = kTileBytes / 2;  // 16 KB: 128 rows x 64 bf16 (one swizzle panel)
constexpr int kSlots = 5;                    // K/V ring: K_j, V_j, K_j+1, ... (2.5 KV steps)
constexpr int kOffQ = 0;                     // 2 tiles
constexpr int kOffKV = 2 * kTileBytes;       // kSlots tiles
constexpr int kOffBar = kOffKV + kSlots * kTileBytes;
constexpr int kSmemBytes = kOffBar + 256 + 1024;  // + barriers + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory per block");
constexpr float kRescaleThreshold = 8.0f;          // log2 units
// Register budgets after setmaxnreg; the sum may not exceed the launch
// allocation (384 threads x 168 registers).
constexpr int kRegLo = 80;   // producer / MMA warpgroup
constexpr int kRegHi = 208;  // each softmax warpgroup
static_assert(128 * kRegLo + 256 * kRegHi <= kThreads * 168, "register budget");

// Pairs of exponentials (of the 16 per 32-column chunk) taken on the FMA
// pipe instead of the MUFU unit: pair i when bit i is set.
constexpr unsigned kPolyPairs = 0x8080u;

// 2^x for a pair on the FMA pipe (Cody-Waite range reduction and a
// polynomial): x = n + f with n = rint(x) (the 1.5 * 2^23 rounding trick)
// and f in [-1/2, 1/2]; 2^f is a degree-3 polynomial whose coefficients were
// fitted to the relative error on that interval (max 7.5e-5, below half an
// ulp of bf16), and n is added to the exponent field. x is clamped to -125,
// so -inf gives 2^-125 (a normal number) rather than 0: far below anything
// that reaches a row sum beside its maximum's 1.
__device__ __forceinline__ void exp2_fma_x2(uint64_t x2, float& p0, float& p1) {
  float x0, x1;
  f2_unpack(x2, x0, x1);
  x2 = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t t2 = f2_add(x2, f2_pack(12582912.f, 12582912.f));
  const uint64_t n2 = f2_add(t2, f2_pack(-12582912.f, -12582912.f));
  const uint64_t f2 = f2_fma(n2, f2_pack(-1.f, -1.f), x2);
  uint64_t q2 = f2_fma(f2_pack(0.05517132f, 0.05517132f), f2, f2_pack(0.24261054f, 0.24261054f));
  q2 = f2_fma(q2, f2, f2_pack(0.69326099f, 0.69326099f));
  q2 = f2_fma(q2, f2, f2_pack(0.99992811f, 0.99992811f));
  float q0, q1, t0, t1;
  f2_unpack(q2, q0, q1);
  f2_unpack(t2, t0, t1);
  p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

struct Params {
  int B, T, H, Hk, W, g, nq, npairs;
  float scale_log2;  // softmax scale * log2(e)
  __nv_bfloat16* O;
  float* lse;
  unsigned long long wait_ns;
};

// HD: head_dim, 128 or 64 (a 64-wide head leaves the second column panel
// zero: its loads are filled with zeros, its products skipped, its stores
// not issued).
template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
               const Params p) {
  extern __shared__ uint8_t smem_raw[];
  pdl_launch_dependents();
  uint8_t* smem = smem_align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;   // [kSlots]
  uint64_t* kv_empty = bars + 6;  // [kSlots]
  uint64_t* s_full = bars + 11;   // [2] per tile
  uint64_t* p_full = bars + 13;   // [2] per tile
  uint64_t* o_full = bars + 15;   // [2] per tile
  uint64_t* mma_done = bars + 17;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 19);
  uint64_t* o_staged = bars + 20;  // [2] per tile: O rows written to shared memory

  const int warp = warp_id(), lane = lane_id();

  // ---- work unit: heavy (late query blocks) first
  const int BHk = p.B * p.Hk;
  const int pr = p.npairs - 1 - static_cast<int>(blockIdx.x) / BHk;
  const int bh = static_cast<int>(blockIdx.x) % BHk;
  const int b = bh / p.Hk, hk = bh % p.Hk;
  const int ntiles = p.nq * p.g;
  int qblk[2], head[2], lo_t[2], hi_t[2];
  bool valid[2];
#pragma unroll
  for (int X = 0; X < 2; ++X) {
    int t = 2 * pr + X;
    valid[X] = t < ntiles;
    if (!valid[X]) t = 2 * pr;
    qblk[X] = t / p.g;
    head[X] = hk * p.g + t % p.g;
    const int q0 = qblk[X] * kBM;
    lo_t[X] = max(0, q0 - p.W + 1) / kBM;
    hi_t[X] = qblk[X];
  }
  const int lo = valid[1] ? min(lo_t[0], lo_t[1]) : lo_t[0];
  const int hi = valid[1] ? max(hi_t[0], hi_t[1]) : hi_t[0];
  // Checked build: the unit lies inside the tensors (uniform over the CTA,
  // before any barrier or TMEM is set up).
  if (!check_bounds(pr >= 0 && b < p.B && hk < p.Hk && lo >= 0 && hi < p.nq && head[0] < p.H &&
                    head[1] < p.H && qblk[1] < p.nq))
    return;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&o_full[s], 1);
      mbar_init(&o_staged[s], 128);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // inputs of the previous kernel in the stream are complete from here on
  const WaitCtx wc{abort_flag, p.wait_ns};

  const uint32_t colS[2] = {0u, 128u};
  const uint32_t colO[2] = {256u, 384u};

  // Registers move from the producer/MMA warpgroup to the softmax
  // warpgroups, which hold a full 128-column S row per thread. Each role's
  // code sits inside its warpgroup's branch so ptxas compiles it under that
  // warpgroup's budget.
  if (warp < 4) {
    regs_dec<kRegLo>();
  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      // Ring slot of tile i (K_j at i = 2(j-lo), V_j at i+1): i % kSlots,
      // use i / kSlots; slots are consumed in the order they are filled.
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmO);
      int filled[kSlots] = {0, 0, 0, 0, 0};
      mbar_expect_tx(q_full, (valid[1] ? 2 : 1) * kTileBytes);
      for (int X = 0; X < 2; ++X) {
        if (!valid[X]) continue;
        uint8_t* dst = smem + kOffQ + X * kTileBytes;
        tma_load_4d(&tmQ, q_full, dst, 0, head[X], qblk[X] * kBM, b);
        tma_load_4d(&tmQ, q_full, dst + kPanelBytes, 64, head[X], qblk[X] * kBM, b);
      }
      int slot = 0, use = 0;
      for (int i = 0; i < 2 * (hi - lo + 1); ++i) {
        if (use > 0 && !mbar_wait(&kv_empty[slot], (use - 1) & 1, wc)) break;
        const int j = lo + (i >> 1);
        const CUtensorMap* tm = (i & 1) ? &tmV : &tmK;
        mbar_expect_tx(&kv_full[slot], kTileBytes);
        uint8_t* dst = smem + kOffKV + slot * kTileBytes;
        tma_load_4d(tm, &kv_full[slot], dst, 0, hk, j * kBM, b);
        tma_load_4d(tm, &kv_full[slot], dst + kPanelBytes, 64, hk, j * kBM, b);
        ++filled[slot];
        if (++slot == kSlots) {
          slot = 0;
          ++use;
        }
      }
      // Drain: every issued copy has landed before the CTA may exit.
      drain_wait(q_full, 0);
      for (int s2 = 0; s2 < kSlots; ++s2)
        if (filled[s2] > 0) drain_wait(&kv_full[s2], (filled[s2] - 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);   // Q K^T: both K-major
      constexpr uint32_t idPV = idesc_bf16(128, 128, 0, 1);  // P V: V MN-major
      const uint32_t sQa = smem_u32(smem + kOffQ);
      const uint32_t sKVa = smem_u32(smem + kOffKV);
      bool ok = mbar_wait(q_full, 0, wc);
      tc_fence_after();

      // Descriptors: a base per buffer plus a compile-time offset per k-step
      // (the start-address field holds address >> 4).
      const uint64_t dQ0 = sdesc_sw128(sQa, 16, 1024);
      const uint64_t dK0 = sdesc_sw128(sKVa, 16, 1024);           // K: K-major
      const uint64_t dV0 = sdesc_sw128(sKVa, kPanelBytes, 1024);  // V: MN-major
      // Ring position of K_j (kind 0) or V_j (kind 1).
      auto ring = [&](int j, int kind, int& slot, int& use) {
        const int i = 2 * (j - lo) + kind;
        slot = i % kSlots;
        use = i / kSlots;
      };

      auto issue_S = [&](int X, int j) -> bool {
        int s, use;
        ring(j, 0, s, use);
        if (!mbar_wait(&kv_full[s], use & 1, wc)) return false;
        tc_fence_after();
        const uint64_t qd = dQ0 + static_cast<uint64_t>((X * kTileBytes) >> 4);
        const uint64_t kd = dK0 + static_cast<uint64_t>((s * kTileBytes) >> 4);
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(X) * 128u;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          if (kk * 16 >= HD) break;  // zero columns of a 64-wide head
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kPanelBytes + (kk & 3) * 32) >> 4);
          mma_ss(d_tmem, qd + off, kd + off, idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[X]);
        return true;
      };
      auto issue_PV = [&](int X, int j) -> bool {
        int s, use;
        ring(j, 1, s, use);
        const int n = j - lo_t[X];
        if (!mbar_wait(&kv_full[s], use & 1, wc)) return false;
        const uint64_t vd = dV0 + static_cast<uint64_t>((s * kTileBytes) >> 4);
        const uint32_t o_tmem = tmem + 256u + static_cast<uint32_t>(X) * 128u;
        const uint32_t p_tmem = tmem + static_cast<uint32_t>(X) * 128u;
        if (!mbar_wait(&p_full[X], n & 1, wc)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(o_tmem, p_tmem + kk * 8, vd + static_cast<uint64_t>((kk * 2048) >> 4), idPV,
                 (n > 0 || kk > 0) ? 1u : 0u);
        return true;
      };

      int rs, ru;
      if (ok) {
        for (int X = 0; X < 2 && ok; ++X)
          if (valid[X] && lo_t[X] == lo) ok = issue_S(X, lo);
        ring(lo, 0, rs, ru);
        if (ok) mma_commit(&kv_empty[rs]);
      }
      for (int j = lo; ok && j <= hi; ++j) {
        for (int X = 0; X < 2 && ok; ++X) {
          if (!valid[X]) continue;
          if (j >= lo_t[X] && j <= hi_t[X]) {
            ok = issue_PV(X, j);
            if (ok && j == hi_t[X]) mma_commit(&o_full[X]);
          }
          if (ok && j + 1 >= lo_t[X] && j + 1 <= hi_t[X]) ok = issue_S(X, j + 1);
        }
        if (!ok) break;
        ring(j, 1, rs, ru);
        mma_commit(&kv_empty[rs]);  // V_j consumed
        if (j + 1 <= hi) {
          ring(j + 1, 0, rs, ru);
          mma_commit(&kv_empty[rs]);  // K_j+1 consumed
        }
      }
      // Drain: all issued MMAs complete before TMEM is released.
      mma_commit(mma_done);
      drain_wait(mma_done, 0);
    }
  }
  } else {
    regs_inc<kRegHi>();
    // -------------------------------------------------- softmax + epilogue
    const int X = (warp - 4) >> 2;
    if (valid[X]) {
      const int r = (warp & 3) * 32 + lane;  // TMEM lane = query row in the tile
      const int q0 = qblk[X] * kBM;
      const int qi = q0 + r;
      const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
      const uint32_t tS = tmem + lane_off + colS[X];
      const uint32_t tO = tmem + lane_off + colO[X];
      const float c2 = p.scale_log2;
      float m2 = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = lo_t[X]; j <= hi_t[X]; ++j) {
        const int n = j - lo_t[X];
        const bool got = mbar_wait(&s_full[X], n & 1, wc);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sv[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sv[c]);
        tmem_ld_wait();
        const int k0 = j * kBM;
        if (k0 + kBM - 1 > q0 || q0 + kBM - 1 - k0 >= p.W) {
          // Row r keeps the keys k0 + e with a <= e <= b (causal: kj <= qi;
          // window: qi - kj < W); an empty range keeps none. Chunks that
          // every lane of the warp keeps whole are skipped.
          int a = max(qi - p.W + 1 - k0, 0);
          const int b = min(qi - k0, kBM - 1);
          unsigned span = static_cast<unsigned>(b - a);
          if (b < a) {
            a = 1 << 20;
            span = 0u;
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (__all_sync(0xffffffffu, a <= 32 * c && 32 * c + 31 <= b)) continue;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (static_cast<unsigned>(32 * c + i - a) > span) sv[c][i] = __float_as_uint(-INFINITY);
          }
        }
        // Row max: a tree of three-input maxima per 32-column chunk.
        float mp[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float t[11];
#pragma unroll
          for (int k = 0; k < 10; ++k)
            t[k] = fmax3(__uint_as_float(sv[c][3 * k]), __uint_as_float(sv[c][3 * k + 1]),
                         __uint_as_float(sv[c][3 * k + 2]));
          t[10] = fmaxf(__uint_as_float(sv[c][30]), __uint_as_float(sv[c][31]));
          mp[c] = fmax3(fmax3(t[0], t[1], t[2]), fmax3(t[3], t[4], t[5]),
                        fmaxf(fmax3(t[6], t[7], t[8]), fmaxf(t[9], t[10])));
        }
        float mx = fmax3(mp[0], mp[1], fmaxf(mp[2], mp[3])) * c2;
        float alpha = 1.f;
        bool rescale = false;
        if (n == 0) {
          m2 = mx;
        } else if (mx > m2 + kRescaleThreshold) {
          alpha = ex2(m2 - mx);
          m2 = mx;
          rescale = true;
        }
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + c * 32, o);
          }
          tmem_st_wait();
        }
        const float mu = (m2 == -INFINITY) ? 0.f : m2;
        // x = c S - mu and the partial row sums, a pair of elements per
        // f32x2 instruction; four independent accumulator pairs.
        const uint64_t c2x2 = f2_pack(c2, c2), nmu2 = f2_pack(-mu, -mu);
        uint64_t ls2[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) ls2[a] = f2_pack(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint64_t x2 =
                f2_fma(f2_pack(__uint_as_float(sv[c][2 * i]), __uint_as_float(sv[c][2 * i + 1])), c2x2, nmu2);
            float p0, p1;
            if ((kPolyPairs >> i) & 1u) {
              exp2_fma_x2(x2, p0, p1);
            } else {
              float x0, x1;
              f2_unpack(x2, x0, x1);
              p0 = ex2(x0);
              p1 = ex2(x1);
            }
            ls2[i & 3] = f2_add(ls2[i & 3], f2_pack(p0, p1));
            pk[i] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tS + c * 16, pk);
        }
        float la, lb, lc, ld;
        f2_unpack(f2_add(ls2[0], ls2[1]), la, lb);
        f2_unpack(f2_add(ls2[2], ls2[3]), lc, ld);
        l = l * alpha + ((la + lb) + (lc + ld));
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[X]);
      }
      const bool o_ok = ok && mbar_wait(&o_full[X], 0, wc);
      if (__all_sync(0xffffffffu, o_ok)) {
        tc_fence_after();
        const float inv_l = 1.f / l;
        // Row r of O as bf16 into this tile's Q buffer, which is free once
        // o_full has fired (every product of the tile is complete), in the
        // 128B-swizzled two-panel layout of the tensor map; then one TMA
        // store per panel writes the tile (rows past T are not written).
        uint8_t* ot = smem + kOffQ + X * kTileBytes;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            const int k = c * 4 + v4;  // 16-byte chunk of the 256-byte row
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * v4 + 0]) * inv_l, __uint_as_float(o[8 * v4 + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(o[8 * v4 + 2]) * inv_l, __uint_as_float(o[8 * v4 + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(o[8 * v4 + 4]) * inv_l, __uint_as_float(o[8 * v4 + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(o[8 * v4 + 6]) * inv_l, __uint_as_float(o[8 * v4 + 7]) * inv_l);
            *reinterpret_cast<uint4*>(ot + (k >> 3) * kPanelBytes + r * 128 + (((k & 7) ^ (r & 7)) << 4)) = w;
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&o_staged[X]);
        if (r == 0 && mbar_wait(&o_staged[X], 0, wc)) {
          tma_store_4d(&tmO, ot, 0, head[X], q0, b);
          if (HD > 64) tma_store_4d(&tmO, ot + kPanelBytes, 64, head[X], q0, b);
          bulk_commit();
          bulk_wait_read0();  // shared source read; the writes finish on their own
        }
        if (qi < p.T)
          p.lse[(static_cast<size_t>(b) * p.H + head[X]) * p.T + qi] =
              (m2 + log2f(l)) * 0.69314718055994531f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fwd
}  // namespace cswattn
