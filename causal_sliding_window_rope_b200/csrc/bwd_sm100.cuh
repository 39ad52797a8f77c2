// bwd_sm100.cuh -- attention backward on tcgen05 tensor cores (bf16, D = 128 or 64).
//
// Gradient of the causal sliding-window attention of the page
// "5만원으로 나만의 ChatGPT 훈련하는 방법" (section "5. 플래시 어텐션 통합",
// with the architecture list's sliding window and GQA), written out:
//   p_ij = exp(c q~_i.k~_j - lse_i),  dp_ij = dO_i . v_j,
//   ds_ij = p_ij (dp_ij - Delta_i),   Delta_i = dO_i . O_i,
//   dv_j  = sum_{h in group} sum_i p_ij dO_i,
//   dk~_j = c sum_{h in group} sum_i ds_ij q~_i,   dq~_i = c sum_j ds_ij k~_j.
//
// Work unit (one CTA): one 128-key tile of one (batch, KV head). It keeps
// K and V in shared memory and its dK/dV accumulators in TMEM while it walks
// every query head of the GQA group and every 64-query step that sees the
// tile, so dK and dV are summed over the group without atomics and written
// once. Per step (transposed products, keys on the TMEM lanes):
//   S^T  = K Q^T      (M=128 keys, N=64 queries, K=128 d)   SS MMA
//   dP^T = V dO^T     (same shape)                         SS MMA
//   softmax warps: P^T = exp2(c2 S^T - lse2), dS^T = P^T (dP^T - Delta)
//                  (pairs of elements per f32x2 instruction),
//                  both as bf16 into TMEM (the step's dQ^T columns), and
//                  dS^T also into shared memory (128B-swizzled)
//   dV  += P^T dO     (M=128 keys, N=128 d, K=64)           TS MMA (P^T in TMEM)
//   dK  += dS^T Q     (same shape)                         TS MMA (dS^T in TMEM)
//   dQ^T = K^T dS^T   (M=128 d, N=64 queries, K=128 keys)   SS MMA, over the
//          P^T/dS^T columns (issued after the two TS MMAs that read them),
//          drained by the dQ warps from TMEM into a swizzled shared tile
//          that four TMA float32 add-reductions send into the dq
//          accumulator (B,T,H,D).
// Shared memory holds the MMA operands (K, V, the Q/dO ring, dS^T) and the
// dQ staging tile; at the end the ring and dS^T buffers stage dK/dV for
// their TMA stores.
// TMEM (512 columns): SP (S^T at +0, dP^T at +64) | dQ^T x2 (64 columns
// each; also P^T at +0 and dS^T at +32 before the dQ^T product) | dV | dK.
// The softmax warps release SP as soon as they have loaded it into
// registers, so the next step's S^T/dP^T run while they compute.
// Roles: warp 0 TMA, warp 1 MMA issuer + TMEM owner, warps 4-7 softmax
// (thread = key row), warps 8-11 dQ drain (thread = head_dim row of dQ^T).
#pragma once
#include "common.cuh"

namespace cswattn {
namespace bwd {

constexpr int kBN = 128;  // keys per tile
constexpr int kBQ = 64;   // queries per step
constexpr int kD = 128;
constexpr int kThreads = 384;
constexpr int kKVBytes = kBN * kD * 2;   // 32 KB
constexpr int kKVPanel = kKVBytes / 2;   // 16 KB: 128 rows x 128 B
constexpr int kQBytes = kBQ * kD * 2;    // 16 KB
constexpr int kQPanel = kQBytes / 2;     // 8 KB: 64 rows x 128 B
constexpr int kPBytes = kBN * kBQ * 2;   // 16 KB: 128 rows x 128 B

constexpr int kQStages = 3;             // Q/dO ring depth
constexpr int kStageBytes = 2 * kQBytes;  // Q then dO
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kKVBytes;
constexpr int kOffQD = kOffV + kKVBytes;                 // [kQStages] x (Q | dO)
constexpr int kOffDS = kOffQD + kQStages * kStageBytes;  // dS^T [2]
// dQ^T drain staging: 4 panels of 64 query rows x 32 float32 (128B-swizzled).
constexpr int kOffDQS = kOffDS + 2 * kPBytes;
constexpr int kDQPanel = kBQ * 128;
constexpr int kDQHalf = kDQPanel / 2;  // one panel of 32 query rows
constexpr int kOffBar = kOffDQS + 4 * kDQPanel;
// dK/dV write-out staging over the Q/dO ring and dS^T buffers: 2 x 4 panels
// of 128 rows x 32 float32.
constexpr int kF32Panel = kBN * 128;
static_assert(kOffQD + 8 * kF32Panel <= kOffDQS, "write-out staging");
constexpr int kOffRow = kOffBar + 256;         // per Q stage: nlse2[64], delta[64]
constexpr int kSmemBytes = kOffRow + kQStages * 2 * kBQ * 4 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per block");

// Register budgets after setmaxnreg (launch: 384 threads x 168 registers).
constexpr int kRegLo = 88;   // producer / MMA warpgroup
constexpr int kRegSm = 248;  // softmax warpgroup (S^T, dP^T rows + packed P, dS)
constexpr int kRegDq = 168;  // dQ drain warpgroup
static_assert(128 * (kRegLo + kRegSm + kRegDq) <= kThreads * 168, "register budget");

constexpr uint32_t kColSP = 0u;  // S^T at +0, dP^T at +64
// TMEM column of dQ^T buffer st (0 or 1).
__host__ __device__ constexpr uint32_t col_dq(int st) { return st ? 192u : 128u; }
constexpr uint32_t kColDV = 256u;
constexpr uint32_t kColDK = 384u;

struct Params {
  int B, T, H, Hk, W, g, nkv, Tpad;
  int parts;               // CTAs per KV tile (each takes a share of its steps)
  long long kv_stride;     // elements between the parts' dK/dV partial slots
  float scale_log2;  // c * log2(e)
  float scale;       // c
  const float* nlse2;  // (B,H,Tpad) -lse * log2(e), -inf past T
  const float* delta;  // (B,H,Tpad) dO.O, 0 past T
  float* dq_acc;       // (B,T,H,D), accumulated (must start at zero)
  float* dk_acc;       // [parts] x (B,T,Hk,D) partial sums
  float* dv_acc;       // [parts] x (B,T,Hk,D) partial sums
  unsigned long long wait_ns;
};

// HD: head_dim, 128 or 64 (a 64-wide head leaves the second column panel
// zero: its loads are filled with zeros, its products skipped where they
// only add zeros, its stores and reductions not issued).
template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
               const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
               const __grid_constant__ CUtensorMap tmDQ, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  pdl_launch_dependents();
  uint8_t* smem = smem_align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;      // [kQStages]
  uint64_t* q_empty = bars + 4;     // [kQStages]
  uint64_t* sp_full = bars + 7;     // S^T/dP^T in TMEM
  uint64_t* sp_free = bars + 8;     // softmax has loaded S^T/dP^T
  uint64_t* p_full = bars + 9;      // P^T/dS^T written (TMEM and shared memory)
  uint64_t* ps_empty = bars + 10;   // [2] dQ^T product done reading dS^T buffer
  uint64_t* dq_full = bars + 12;    // [2]
  uint64_t* dq_empty = bars + 14;   // [2]
  uint64_t* acc_full = bars + 16;
  uint64_t* mma_done = bars + 17;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 19);
  uint64_t* kv_staged = bars + 20;  // dK/dV rows written to shared memory
  uint64_t* dqs_full = bars + 21;   // [2] half of the dQ staging tile written (128 arrivals)
  uint64_t* dqs_free = bars + 23;   // [2] the reduction has read that half
  float* s_nlse2 = reinterpret_cast<float*>(smem + kOffRow);       // [kQStages][64]
  float* s_delta = s_nlse2 + kQStages * kBQ;                        // [kQStages][64]

  const int warp = warp_id(), lane = lane_id();

  // ---- work unit: KV block j (ascending = most queries first), part of
  // its steps, (b, hk). Heavy KV tiles are split into `parts` CTAs so that
  // the grid balances across SMs; each part writes its own dK/dV partials.
  const int BHk = p.B * p.Hk;
  const int unit = static_cast<int>(blockIdx.x) / BHk;
  const int j = unit / p.parts, part = unit % p.parts;
  const int bh = static_cast<int>(blockIdx.x) % BHk;
  const int b = bh / p.Hk, hk = bh % p.Hk;
  const int k0 = j * kBN;
  const long long q_last_ll = min(static_cast<long long>(p.T) - 1,
                                  static_cast<long long>(k0) + kBN - 1 + p.W - 1);
  const int qs_lo = k0 / kBQ;
  const int qs_hi = static_cast<int>(q_last_ll) / kBQ;
  const int nsph = qs_hi - qs_lo + 1;  // steps per head
  const int n_all = p.g * nsph;
  const int n_begin = static_cast<int>(static_cast<long long>(part) * n_all / p.parts);
  const int N = static_cast<int>(static_cast<long long>(part + 1) * n_all / p.parts) - n_begin;
  // Checked build: the work unit lies inside the tensors and the row-term
  // copies of its last step stay inside the padded (B, H, Tpad) arrays.
  if (!check_bounds(b < p.B && hk < p.Hk && j < p.nkv && part < p.parts && qs_lo <= qs_hi &&
                    (qs_hi + 1) * kBQ <= p.Tpad && n_begin + N <= n_all))
    return;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(sp_full, 1);
    mbar_init(sp_free, 128);
    mbar_init(p_full, 128);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ps_empty[s], 1);
      mbar_init(&dq_full[s], 1);
      mbar_init(&dq_empty[s], 128);
    }
    mbar_init(acc_full, 1);
    mbar_init(kv_staged, 128);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&dqs_full[s], 128);
      mbar_init(&dqs_free[s], 1);
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


  // Step n = (head within the group, 64-query block), walked without
  // divisions: every role keeps its own cursor and advances it per step.
  struct Cursor {
    int h, qs, h_end, qs_lo, qs_hi;
    __device__ void next() {
      if (++qs > qs_hi) {
        qs = qs_lo;
        ++h;
      }
    }
    __device__ int q0() const { return qs * kBQ; }
  };
  const Cursor cur0{hk * p.g + n_begin / nsph, qs_lo + n_begin % nsph, hk * p.g + p.g, qs_lo, qs_hi};

  if (warp < 4) {
    regs_dec<kRegLo>();
  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int nq[kQStages] = {0, 0, 0};
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmDO);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmDK);
      prefetch_tmap(&tmDV);
      prefetch_tmap(&tmDQ);
      Cursor c = cur0;
      int st = 0, use = 0;
      mbar_expect_tx(kv_full, 2 * kKVBytes);
      tma_load_4d(&tmK, kv_full, smem + kOffK, 0, hk, k0, b);
      tma_load_4d(&tmK, kv_full, smem + kOffK + kKVPanel, 64, hk, k0, b);
      tma_load_4d(&tmV, kv_full, smem + kOffV, 0, hk, k0, b);
      tma_load_4d(&tmV, kv_full, smem + kOffV + kKVPanel, 64, hk, k0, b);
      for (int n = 0; n < N; ++n, c.next()) {
        if (use > 0 && !mbar_wait(&q_empty[st], (use - 1) & 1, wc)) break;
        const int h = c.h, q0 = c.q0();
        mbar_expect_tx(&q_full[st], 2 * kQBytes + 2 * kBQ * 4);
        uint8_t* qd = smem + kOffQD + st * kStageBytes;
        uint8_t* od = qd + kQBytes;
        tma_load_4d(&tmQ, &q_full[st], qd, 0, h, q0, b);
        tma_load_4d(&tmQ, &q_full[st], qd + kQPanel, 64, h, q0, b);
        tma_load_4d(&tmDO, &q_full[st], od, 0, h, q0, b);
        tma_load_4d(&tmDO, &q_full[st], od + kQPanel, 64, h, q0, b);
        // Row terms of the step's 64 queries (padded layout: always in range).
        const size_t ro = (static_cast<size_t>(b) * p.H + h) * p.Tpad + q0;
        bulk_load(s_nlse2 + st * kBQ, p.nlse2 + ro, kBQ * 4, &q_full[st]);
        bulk_load(s_delta + st * kBQ, p.delta + ro, kBQ * 4, &q_full[st]);
        ++nq[st];
        if (++st == kQStages) {
          st = 0;
          ++use;
        }
      }
      drain_wait(kv_full, 0);
      for (int s = 0; s < kQStages; ++s)
        if (nq[s] > 0) drain_wait(&q_full[s], (nq[s] - 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t idS = idesc_bf16(128, 64, 0, 0);    // K Q^T, V dO^T
      constexpr uint32_t idKV = idesc_bf16(128, 128, 0, 1);  // P^T dO, dS^T Q
      constexpr uint32_t idDQ = idesc_bf16(128, 64, 1, 1);   // K^T dS^T
      const uint32_t sK = smem_u32(smem + kOffK), sV = smem_u32(smem + kOffV);
      const uint32_t sQ = smem_u32(smem + kOffQD), sDO = sQ + kQBytes;
      const uint32_t sDS = smem_u32(smem + kOffDS);
      bool ok = mbar_wait(kv_full, 0, wc);
      tc_fence_after();

      // Descriptors: a base per buffer plus a compile-time offset per k-step
      // (the start-address field holds address >> 4).
      const uint64_t dK_k = sdesc_sw128(sK, 16, 1024);         // K, K-major
      const uint64_t dV_k = sdesc_sw128(sV, 16, 1024);         // V, K-major
      const uint64_t dQ_k = sdesc_sw128(sQ, 16, 1024);         // Q, K-major
      const uint64_t dO_k = sdesc_sw128(sDO, 16, 1024);        // dO, K-major
      const uint64_t dQ_m = sdesc_sw128(sQ, kQPanel, 1024);    // Q, MN-major
      const uint64_t dO_m = sdesc_sw128(sDO, kQPanel, 1024);   // dO, MN-major
      const uint64_t dS_m = sdesc_sw128(sDS, kPBytes, 1024);   // dS^T, MN-major
      const uint64_t dK_m = sdesc_sw128(sK, kKVPanel, 1024);   // K^T, MN-major
      auto ofs = [](int bytes) { return static_cast<uint64_t>(bytes >> 4); };

      auto issue_SdP = [&](int n) -> bool {
        const int st = n % kQStages, use = n / kQStages;
        if (!mbar_wait(&q_full[st], use & 1, wc)) return false;
        if (n > 0 && !mbar_wait(sp_free, (n - 1) & 1, wc)) return false;
        tc_fence_after();
        const uint64_t qb = ofs(st * kStageBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          if (kk * 16 >= HD) break;  // zero columns of a 64-wide head
          const uint64_t okv = ofs((kk >> 2) * kKVPanel + (kk & 3) * 32);
          const uint64_t oq = ofs((kk >> 2) * kQPanel + (kk & 3) * 32);
          mma_ss(tmem + kColSP, dK_k + okv, dQ_k + qb + oq, idS, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          if (kk * 16 >= HD) break;
          const uint64_t okv = ofs((kk >> 2) * kKVPanel + (kk & 3) * 32);
          const uint64_t oq = ofs((kk >> 2) * kQPanel + (kk & 3) * 32);
          mma_ss(tmem + kColSP + 64, dV_k + okv, dO_k + qb + oq, idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(sp_full);
        return true;
      };

      if (ok && N > 0) ok = issue_SdP(0);
      for (int n = 0; ok && n < N; ++n) {
        const int st = n % kQStages;
        const int db = n & 1, duse = n >> 1;  // dQ^T TMEM buffer
        // The next step's S^T/dP^T as soon as the softmax has loaded this one.
        if (n + 1 < N && !issue_SdP(n + 1)) break;
        // The softmax has written P^T/dS^T into dQ^T buffer db (after that
        // buffer was drained) and dS^T into shared buffer db.
        if (!mbar_wait(p_full, n & 1, wc)) break;
        tc_fence_after();
        const uint64_t qb = ofs(st * kStageBytes);
        const uint32_t ptm = tmem + col_dq(db);  // P^T at +0, dS^T at +32
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // dV += P^T dO
          mma_ts(tmem + kColDV, ptm + kk * 8, dO_m + qb + ofs(kk * 2048), idKV,
                 (n > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // dK += dS^T Q
          mma_ts(tmem + kColDK, ptm + 32 + kk * 8, dQ_m + qb + ofs(kk * 2048), idKV,
                 (n > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&q_empty[st]);
        const uint64_t sb = ofs(db * kPBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // dQ^T = K^T dS^T (over P^T/dS^T, read above)
          mma_ss(ptm, dK_m + ofs(kk * 2048), dS_m + sb + ofs(kk * 2048), idDQ, kk > 0 ? 1u : 0u);
        mma_commit(&dq_full[db]);
        mma_commit(&ps_empty[db]);
        (void)duse;
      }
      mma_commit(acc_full);
      mma_commit(mma_done);
      drain_wait(mma_done, 0);
    }
  }
  } else if (warp < 8) {
    regs_inc<kRegSm>();
    // -------------------------------------------------- softmax / dS
    const int r = (warp & 3) * 32 + lane;  // key row within the tile
    const int kj = k0 + r;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float c2 = p.scale_log2;
    bool ok = true;
    Cursor c = cur0;
    for (int n = 0; n < N; ++n, c.next()) {
      const int st = n % kQStages, use = n / kQStages;
      const int q0 = c.q0();
      // S^T/dP^T of this step, and (same stage barrier as Q/dO) its nlse2/Delta.
      bool got = mbar_wait(sp_full, n & 1, wc);
      got = got && mbar_wait(&q_full[st], use & 1, wc);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[2][32], dv[2][32];
      tmem_ld32(tmem + lane_off + kColSP, sv[0]);
      tmem_ld32(tmem + lane_off + kColSP + 32, sv[1]);
      tmem_ld32(tmem + lane_off + kColSP + 64, dv[0]);
      tmem_ld32(tmem + lane_off + kColSP + 96, dv[1]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(sp_free);  // the MMA warp may overwrite SP now
      const float4* NL = reinterpret_cast<const float4*>(s_nlse2 + st * kBQ);
      const float4* DL = reinterpret_cast<const float4*>(s_delta + st * kBQ);
      const uint64_t c2x2 = f2_pack(c2, c2);
      uint32_t pp[32], dd[32];
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 l4 = NL[(c * 32 + i) >> 2];
          const float4 d4 = DL[(c * 32 + i) >> 2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int e = i + 2 * h;
            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sv[c][e]), __uint_as_float(sv[c][e + 1])), c2x2,
                                       h == 0 ? f2_pack(l4.x, l4.y) : f2_pack(l4.z, l4.w));
            float x0, x1;
            f2_unpack(x2, x0, x1);
            const uint64_t p2 = f2_pack(ex2(x0), ex2(x1));
            const uint64_t ds2 =
                f2_mul(p2, f2_sub(f2_pack(__uint_as_float(dv[c][e]), __uint_as_float(dv[c][e + 1])),
                                  h == 0 ? f2_pack(d4.x, d4.y) : f2_pack(d4.z, d4.w)));
            float p0, p1, s0, s1;
            f2_unpack(p2, p0, p1);
            f2_unpack(ds2, s0, s1);
            pp[c * 16 + e / 2] = pack_bf16x2(p0, p1);
            dd[c * 16 + e / 2] = pack_bf16x2(s0, s1);
          }
        }
      if ((q0 < k0 + kBN - 1) || (q0 + kBQ - 1 - k0 >= p.W)) {
        // Key row kj sees the queries kj <= q < kj + W: columns [a, b] of
        // the step. Pairs outside are zeroed (P and dS alike); 16-pair
        // chunks that every lane of the warp keeps whole are skipped.
        int a = max(kj - q0, 0);
        const int bq = min(kj + p.W - 1 - q0, kBQ - 1);
        unsigned span = static_cast<unsigned>(bq - a);
        if (bq < a) {
          a = 1 << 20;
          span = 0u;
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (__all_sync(0xffffffffu, a <= 32 * c && 32 * c + 31 <= bq)) continue;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const bool k0v = static_cast<unsigned>(32 * c + 2 * i - a) <= span;
            const bool k1v = static_cast<unsigned>(32 * c + 2 * i + 1 - a) <= span;
            const uint32_t keep = (k0v ? 0x0000ffffu : 0u) | (k1v ? 0xffff0000u : 0u);
            pp[c * 16 + i] &= keep;
            dd[c * 16 + i] &= keep;
          }
        }
      }
      // Buffer db (TMEM dQ^T columns and shared dS^T) was last used by step
      // n-2: wait until that step's dQ^T has been drained and its dQ^T
      // product has read the shared dS^T.
      const int db = n & 1, duse = n >> 1;
      got = duse == 0 || (mbar_wait(&dq_empty[db], (duse - 1) & 1, wc) &&
                          mbar_wait(&ps_empty[db], (duse - 1) & 1, wc));
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // P^T and dS^T rows into TMEM (A operands of the dV / dK products).
      tmem_st32(tmem + lane_off + col_dq(db), pp);
      tmem_st32(tmem + lane_off + col_dq(db) + 32, dd);
      // Row r of dS^T into shared memory: 64 bf16 = 8 chunks of 16 B, 128B-swizzled.
      uint8_t* drow = smem + kOffDS + db * kPBytes + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const int pos = (ch ^ (r & 7)) << 4;
        *reinterpret_cast<uint4*>(drow + pos) =
            make_uint4(dd[4 * ch], dd[4 * ch + 1], dd[4 * ch + 2], dd[4 * ch + 3]);
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // dK / dV write-out: thread r holds key row r of both accumulators. The
    // rows go through shared memory (the Q/dO ring and the dS^T buffers,
    // free once acc_full has fired) as four 32-column float32 panels per
    // tensor in the 128B-swizzled layout of the tensor maps; eight TMA
    // stores then write the tile (rows past T are not written).
    const bool acc_ok = ok && mbar_wait(acc_full, 0, wc);
    if (__all_sync(0xffffffffu, acc_ok)) {
      tc_fence_after();
      const float keep = N > 0 ? 1.f : 0.f;  // a part without steps writes zeros
      uint8_t* stv = smem + kOffQD;           // dV panels
      uint8_t* stk = stv + 4 * kF32Panel;     // dK panels
      auto stage_row = [&](uint8_t* panel, const uint32_t (&a)[32], float sc) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          *reinterpret_cast<float4*>(panel + r * 128 + ((k ^ (r & 7)) << 4)) =
              make_float4(__uint_as_float(a[4 * k]) * sc, __uint_as_float(a[4 * k + 1]) * sc,
                          __uint_as_float(a[4 * k + 2]) * sc, __uint_as_float(a[4 * k + 3]) * sc);
      };
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t a[32];
        tmem_ld32(tmem + lane_off + kColDV + c * 32, a);
        tmem_ld_wait();
        stage_row(stv + c * kF32Panel, a, keep);
        tmem_ld32(tmem + lane_off + kColDK + c * 32, a);
        tmem_ld_wait();
        stage_row(stk + c * kF32Panel, a, p.scale * keep);
      }
      fence_proxy_async_smem();
      mbar_arrive(kv_staged);
      if (r == 0 && mbar_wait(kv_staged, 0, wc)) {
        const int outer = part * p.B + b;  // partial slot `part` of batch b
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (32 * c >= HD) break;  // columns past head_dim are not stored
          tma_store_4d(&tmDV, stv + c * kF32Panel, 32 * c, hk, k0, outer);
          tma_store_4d(&tmDK, stk + c * kF32Panel, 32 * c, hk, k0, outer);
        }
        bulk_commit();
        bulk_wait_read0();  // shared source read; the writes finish on their own
      }
    }
  } else {
    if constexpr (kRegDq > 168)
      regs_inc<kRegDq>();
    else
      regs_dec<kRegDq>();
    // -------------------------------------------------- dQ drain
    const int d = (warp & 3) * 32 + lane;  // TMEM lane = head_dim index of dQ^T
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sc = p.scale;
    uint8_t* stile = smem + kOffDQS;
    const bool leader = threadIdx.x == 256;
    Cursor c = cur0;
    for (int n = 0; n < N; ++n, c.next()) {
      const int st = n & 1, use = n >> 1;
      const int h = c.h, q0 = c.q0();
      bool got = mbar_wait(&dq_full[st], use & 1, wc);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      uint32_t a[2][32];
      tmem_ld32(tmem + lane_off + col_dq(st), a[0]);
      tmem_ld32(tmem + lane_off + col_dq(st) + 32, a[1]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&dq_empty[st]);
      // Column q of dQ^T is row q of the step's dQ~ tile. The tile goes out
      // in two halves of 32 query rows (hq), each staged as four 32-column
      // float32 panels (128B-swizzled; the warp's 32 lanes fill one 128-byte
      // row, conflict-free) and added into dq_acc by four TMA reductions
      // (rows past T are skipped). A half is restaged only once the
      // reduction of its previous use has read it, so the reduction of one
      // half overlaps the staging of the other.
      const int chunk = (d & 31) >> 2;
      bool step_ok = true;
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {
        // Half hq of step n-1 has been read: signalled once per step.
        got = n == 0 || mbar_wait(&dqs_free[hq], (n - 1) & 1, wc);
        if (!__all_sync(0xffffffffu, got)) {
          step_ok = false;
          break;
        }
        uint8_t* prow = stile + hq * (4 * kDQHalf) + (d >> 5) * kDQHalf + (d & 3) * 4;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          *reinterpret_cast<float*>(prow + i * 128 + ((chunk ^ (i & 7)) << 4)) = __uint_as_float(a[hq][i]) * sc;
        fence_proxy_async_smem();
        mbar_arrive(&dqs_full[hq]);
        if (leader) {
          if (mbar_wait(&dqs_full[hq], n & 1, wc)) {
#pragma unroll
            for (int pc = 0; pc < 4; ++pc)
              if (32 * pc < HD)
                tma_reduce_add_4d(&tmDQ, stile + hq * (4 * kDQHalf) + pc * kDQHalf, 32 * pc, h, q0 + 32 * hq, b);
          }
          bulk_commit();
          // Every group but this one has been read: the other half's
          // previous use (half 1 of step n-1, or half 0 of this step).
          bulk_wait_read1();
          if (hq == 1 || n > 0) mbar_arrive(&dqs_free[hq ^ 1]);
        }
      }
      if (!step_ok) break;
    }
    if (leader) bulk_wait_read0();  // shared source read; the writes finish on their own
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bwd
}  // namespace cswattn
