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
//   decode_attn: CTA = (KV head, split of the window, sequence), three
//     roles: one thread streams the split's K chunks, then its V chunks
//     (128 keys each), through a TMA ring; one thread issues the tensor-core
//     products with the group's 16 head slots as N: S^T = K Q^T per chunk
//     into its own TMEM columns, then O^T = V^T P^T accumulated over the
//     chunks; four warps compute the new token's prologue (q~ rows into the
//     Q operand; k~ and v_eff to the caches), fold each chunk's scores into
//     a max per head as its product completes, and, once all are in, write
//     P^T = 2^(s - max) per V chunk and finally O and lse (or, for a split
//     sequence, the partial max, sum and O).
//   decode_combine (only when a sequence is split): one CTA per (sequence,
//     query head) merges the splits' partials (rescaled by 2^(m_s - M))
//     into O and lse.
// A cache length outside [0, T) is reported through the status word
// (CSWATTN_ERR_INVALID_ARG at the next status check) and that sequence is
// left untouched.
#pragma once
#include "prologue.cuh"

namespace cswattn {

constexpr unsigned int kStatusRange = 8u;

namespace dec {

constexpr int kKeys = 128;      // keys per chunk (one tile of the ring, one S^T product)
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
  int nmax;           // most chunks a split holds
  uint32_t tmem_cols; // TMEM columns a CTA allocates: 16 (O) + 16 per chunk, a power of two
  __nv_bfloat16* O;   // (B,H,D): written directly when nsplit == 1
  float* lse;         // (B,H): likewise
  unsigned long long wait_ns;
};

// Splits per (sequence, KV head): enough CTAs to cover the SMs (148 on a
// B200) once, at most one per chunk, and at least enough that a split's
// scores fit in TMEM (kMaxChunks chunks of 16 columns next to O's 16).
constexpr int kMaxChunks = 31;
__host__ inline int decode_nsplit(int B, int Hk, int T, int W) {
  const long long pairs = static_cast<long long>(B) * Hk;
  const int chunks = decode_splits(T, W);
  long long want = pairs >= 148 ? 1 : 148 / pairs;
  if (want > chunks) want = chunks;
  const long long need = (chunks + kMaxChunks - 1) / kMaxChunks;
  return static_cast<int>(want > need ? want : need);
}
__host__ inline int decode_nmax(int nsplit, int T, int W) {
  const int chunks = decode_splits(T, W);
  return (chunks + nsplit - 1) / nsplit;
}
__host__ inline uint32_t decode_tmem_cols(int nmax) {
  uint32_t c = 32;
  while (c < static_cast<uint32_t>(kSlots * (nmax + 1))) c *= 2;
  return c;
}

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

  // A row's inputs as loaded: x (q, k or v), and for a value row ve and
  // the gate logit.
  struct In {
    float xl[HV], xh[HV], el[HV], eh[HV];
    float gate;
  };

  __device__ static void load(const AttnParams& p, int b, int kind, int head, int sub, bool valid, In& in) {
    const int nh = kind == 0 ? p.H : p.Hk;
    const size_t src = (static_cast<size_t>(b) * nh + head) * D + sub * HV;
    const __nv_bfloat16* x = kind == 0 ? p.q : (kind == 1 ? p.k : p.v);
    in.gate = 0.f;
    if (valid) {
      HVec::load(x + src, in.xl);
      HVec::load(x + src + HALF, in.xh);
    } else {
#pragma unroll
      for (int i = 0; i < HV; ++i) in.xl[i] = in.xh[i] = 0.f;
    }
    if (valid && kind == 2 && p.has_ve) {
      in.gate = __bfloat162float(p.gate[static_cast<size_t>(b) * p.Hk + head]);
      HVec::load(p.ve + src, in.el);
      HVec::load(p.ve + src + HALF, in.eh);
    } else {
#pragma unroll
      for (int i = 0; i < HV; ++i) in.el[i] = in.eh[i] = 0.f;
    }
  }

  // Every lane of the warp takes part (row_sum shuffles).
  __device__ static void finish(const AttnParams& p, int kind, int sub, bool valid, const In& in,
                                const float* cs, const float* sn, float (&yl)[HV], float (&yh)[HV]) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < HV; ++i) ss = fmaf(in.xl[i], in.xl[i], fmaf(in.xh[i], in.xh[i], ss));
    ss = row_sum<LPR>(ss);
    if (kind == 2) {
      const float coef = (valid && p.has_ve) ? 3.0f / (1.0f + expf(-in.gate)) : 0.f;
#pragma unroll
      for (int i = 0; i < HV; ++i) {
        yl[i] = fmaf(coef, in.el[i], in.xl[i]);
        yh[i] = fmaf(coef, in.eh[i], in.xh[i]);
      }
      return;
    }
    const float rstd = rsqrtf(ss / static_cast<float>(D) + p.eps);
#pragma unroll
    for (int i = 0; i < HV; ++i) {
      const float c = cs[sub * HV + i], s = sn[sub * HV + i];
      const float nl = in.xl[i] * rstd, nh2 = in.xh[i] * rstd;
      yl[i] = fmaf(nl, c, -nh2 * s);
      yh[i] = fmaf(nl, s, nh2 * c);
    }
  }
};

// Shared memory of decode_attn_kernel<D> (dynamic, 1 KB alignment slack).
// A ring of kStages tiles of kKeys rows (D/64 swizzled panels) carries the
// split's K chunks and then its V chunks. The second product reads V^T as
// 128 rows of 64-column panels kPanel apart, so at D = 64 one panel of
// padding follows the ring (rows of the product that are never read back).
// The products' B operands are 16-row, K-major, 128B-swizzled tiles of 2 KB
// panels: Q (head slot x D) and two P^T buffers (head slot x 128 keys).
template <int D>
struct DecSmem {
  static constexpr int kStages = 4;
  static constexpr int kTile = (D / 64) * kPanel;
  static constexpr int kSPanel = kSlots * 128;               // 2 KB: 16 rows x 128 bytes
  static constexpr int kOffQ = kStages * kTile + (D == 64 ? kPanel : 0);
  static constexpr int kOffP = kOffQ + (D / 64) * kSPanel;   // 2 buffers x 2 panels
  static constexpr int kOffRed = kOffP + 4 * kSPanel;        // float [16][4] warp partials
  static constexpr int kOffStat = kOffRed + kSlots * 4 * 4;  // float [16] max, [16] sum, [16] new-key score
  static constexpr int kOffCS = kOffStat + 3 * kSlots * 4;   // float [D/2] cos, [D/2] sin
  static constexpr int kOffBar = kOffCS + D * 4;
  static constexpr int kNumBars = 2 * kStages + 7 + kMaxChunks;  // ring, the fixed ones, one per chunk's S^T
  static constexpr int kBytes = kOffBar + 8 * (kNumBars + 2) + 1024;
  static_assert(kOffQ % 1024 == 0 && kOffP % 1024 == 0, "operand tiles need 1024-byte alignment");
  static_assert(kBytes <= 232448, "shared memory per block");
};

// Byte offset of element (row, col) of a 128B-swizzled K-major tile of
// 16-row panels (64 bf16 columns per panel).
__device__ __forceinline__ int slot_tile_ofs(int row, int col) {
  return (col >> 6) * (kSlots * 128) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2;
}

constexpr int kDecThreads = 192;  // warp 0: copies, warp 1: products, warps 2-5: softmax and output
constexpr int kSoftBar = 1;       // named barrier of the 128 softmax threads

// CTA = (KV head, split, sequence): the split's share of the 128-key chunks
// covering the window (p - W, p], aligned to absolute positions. All the
// split's scores stay in TMEM: the K chunks stream through the ring into
// S^T products (16 columns per chunk), one max per head is taken over all
// of them, and the V chunks follow through the same ring into O^T = V^T P^T
// accumulated in one 16-column TMEM accumulator, chunk by chunk as the
// softmax warps write P^T. With one split the CTA writes O and lse itself.
template <int D>
__global__ void __launch_bounds__(kDecThreads, 1) decode_attn_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                     const __grid_constant__ CUtensorMap tmV,
                                                                     const AttnParams p) {
  using SM = DecSmem<D>;
  constexpr int NS = SM::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint8_t* sQ = smem + SM::kOffQ;
  uint8_t* sP = smem + SM::kOffP;  // buffer i at i * 2 panels
  float* red = reinterpret_cast<float*>(smem + SM::kOffRed);
  float* stat_m = reinterpret_cast<float*>(smem + SM::kOffStat);
  float* stat_l = stat_m + kSlots;
  float* s_new = stat_l + kSlots;  // the new key's score per head (raw q~ . k~)
  float* cs = reinterpret_cast<float*>(smem + SM::kOffCS);
  float* sn = cs + D / 2;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::kOffBar);  // [NS] tile landed
  uint64_t* empty = full + NS;                                       // [NS] tile read by its product
  uint64_t* q_ready = full + 2 * NS;      // Q tile written (128 arrivals)
  uint64_t* p_ready = full + 2 * NS + 1;  // [2] P^T buffer written, V rows fixed (128 arrivals)
  uint64_t* p_free = full + 2 * NS + 3;   // [2] P^T buffer read by its product
  uint64_t* o_done = full + 2 * NS + 5;   // O^T complete
  uint64_t* mma_drain = full + 2 * NS + 6;
  uint64_t* s_chunk = full + 2 * NS + 7;  // [kMaxChunks] S^T of chunk i done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(full + SM::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + SM::kNumBars + 1);

  // KV head fastest: the CTAs reading the same cache rows run side by side.
  const int hk = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int warp = warp_id(), lane = lane_id();
  const int g = p.g;
  pdl_launch_dependents();
  pdl_wait();
  const int pos = p.len[b];
  const bool in_range = pos >= 0 && pos < p.T;
  if (!in_range && split == 0 && hk == 0 && threadIdx.x == 0) atomicOr(&g_status, kStatusRange);
  const int lo = in_range ? max(0, pos - p.W + 1) : 0;
  const int cbase = (lo / kKeys) * kKeys;                    // first chunk of the window
  const int nch = in_range ? (pos - cbase) / kKeys + 1 : 0;  // chunks of the window
  const int ch0 = static_cast<int>(static_cast<long long>(nch) * split / p.nsplit);
  const int ch1 = static_cast<int>(static_cast<long long>(nch) * (split + 1) / p.nsplit);
  const int n = ch1 - ch0;  // this CTA's chunks; every chunk holds a key of [lo, pos]
  auto part = [&](int h) { return (static_cast<size_t>(b) * p.H + h) * p.nsplit + split; };
  if (!check_bounds(b < p.B && hk < p.Hk && split < p.nsplit && (hk + 1) * g <= p.H && g <= kSlots &&
                    n <= p.nmax))
    return;
  if (n <= 0) {
    // No chunk: an empty partial (ignored by the combine step), or, for a
    // sequence whose length is out of range, nothing at all.
    if (in_range) {
      for (int i = threadIdx.x; i < g * D; i += blockDim.x) p.part_o[part(hk * g + i / D) * D + i % D] = 0.f;
      if (threadIdx.x < g) {
        p.part_ml[part(hk * g + threadIdx.x) * 2] = -INFINITY;
        p.part_ml[part(hk * g + threadIdx.x) * 2 + 1] = 0.f;
      }
    }
    return;
  }
  const bool owns_new = ch1 == nch;  // the last chunk holds the new token's row
  if (threadIdx.x == 0) {
    for (int i = 0; i < SM::kNumBars; ++i) mbar_init(&full[i], (&full[i] == q_ready || &full[i] == p_ready ||
                                                                &full[i] == p_ready + 1) ? 128 : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, p.tmem_cols);  // O^T: columns 0-15; S^T of chunk i: 16 + 16 i
    tmem_relinquish();
  }
  // The new token's inputs (first pass of rows) are loaded before the first
  // tile copy is issued, so that they do not queue behind the copies.
  using NT = NewToken<D>;
  static_assert(NT::HV == 8, "one 16-byte chunk per half");
  constexpr int kRowsPerPass = 128 / NT::LPR;
  const int ts = static_cast<int>(threadIdx.x) - 64;  // softmax thread 0..127 (warps 2-5)
  const int sub = (ts & 127) % NT::LPR, grp = (ts & 127) / NT::LPR;
  auto row_kind = [&](int rr) { return rr < g ? 0 : (rr == g ? 1 : 2); };
  auto row_valid = [&](int rr) { return rr < g || (owns_new && rr < g + 2); };
  typename NT::In in0;
  if (warp >= 2) NT::load(p, b, row_kind(grp), row_kind(grp) == 0 ? hk * g + grp : hk, sub, row_valid(grp), in0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.wait_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ copies: K chunks, then V chunks
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued[NS] = {};
      for (int seq = 0; seq < 2 * n; ++seq) {
        const int st = seq % NS, use = seq / NS;
        if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, wc)) break;
        const bool is_v = seq >= n;
        const int c = cbase + (ch0 + (is_v ? seq - n : seq)) * kKeys;
        uint8_t* dst = smem + st * SM::kTile;
        mbar_expect_tx(&full[st], SM::kTile);
        // Rows past T read as zero; rows outside [lo, pos] are masked
        // (scores) or zeroed before their product (V).
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn)
          tma_load_4d(is_v ? &tmV : &tmK, &full[st], dst + pn * kPanel, 64 * pn, hk, c, b);
        ++issued[st];
      }
      for (int st = 0; st < NS; ++st)
        if (issued[st] > 0) drain_wait(&full[st], (issued[st] - 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ tensor-core products
      const uint32_t r0 = smem_u32(smem), q0 = smem_u32(sQ), p0 = smem_u32(sP);
      bool ok = mbar_wait(q_ready, 0, wc);
      constexpr uint32_t idS = idesc_bf16(128, kSlots, 0, 0);  // S^T = K Q^T
      constexpr uint32_t idO = idesc_bf16(128, kSlots, 1, 0);  // O^T = V^T P^T, V read MN-major
      for (int ci = 0; ok && ci < n; ++ci) {
        const int st = ci % NS;
        if (!(ok = mbar_wait(&full[st], (ci / NS) & 1, wc))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t da =
              sdesc_sw128(r0 + st * SM::kTile + (kk >> 2) * kPanel, 16, 1024) + static_cast<uint64_t>((kk & 3) * 2);
          const uint64_t db =
              sdesc_sw128(q0 + (kk >> 2) * SM::kSPanel, 16, 1024) + static_cast<uint64_t>((kk & 3) * 2);
          mma_ss(tmem + kSlots * (1 + ci), da, db, idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(&empty[st]);
        mma_commit(&s_chunk[ci]);
      }
      for (int ci = 0; ok && ci < n; ++ci) {
        const int seq = n + ci, st = seq % NS;
        if (!(ok = mbar_wait(&full[st], (seq / NS) & 1, wc))) break;
        if (!(ok = mbar_wait(&p_ready[ci & 1], (ci >> 1) & 1, wc))) break;
        tc_fence_after();
        const uint64_t dv = sdesc_sw128(r0 + st * SM::kTile, kPanel, 1024);
        const uint32_t pb = p0 + (ci & 1) * 2 * SM::kSPanel;
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          const uint64_t db = sdesc_sw128(pb + (kk >> 2) * SM::kSPanel, 16, 1024) + static_cast<uint64_t>((kk & 3) * 2);
          mma_ss(tmem, dv + static_cast<uint64_t>((kk * 16 * 128) >> 4), db, idO, (ci > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty[st]);
        mma_commit(&p_free[ci & 1]);
      }
      if (ok) mma_commit(o_done);
      mma_commit(mma_drain);  // every product issued above completes before it fires
      drain_wait(mma_drain, 0);
    }
  } else {
    // -------------------------------------------------- softmax and output (warps 2-5)
    const int quad = warp & 3;            // TMEM lanes 32 quad .. 32 quad + 31
    const int r = quad * 32 + lane;       // key row of a chunk, then column of O
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    // The new token's prologue at position pos.
    for (int i = ts; i < D / 2; i += 128) {
      float sv_, cv_;
      sincosf(static_cast<float>(pos) * p.omega[i], &sv_, &cv_);
      cs[i] = cv_;
      sn[i] = sv_;
    }
    for (int i = ts; i < (kSlots - g) * (D / 8); i += 128) {  // unused head slots: zero rows of Q
      const int row = g + i / (D / 8), col = (i % (D / 8)) * 8;
      *reinterpret_cast<uint4*>(sQ + slot_tile_ofs(row, col)) = make_uint4(0u, 0u, 0u, 0u);
    }
    for (int i = ts; i < 2 * (kSlots - g) * (kKeys / 8); i += 128) {  // ... and of both P^T buffers
      const int buf = i / ((kSlots - g) * (kKeys / 8)), k = i % ((kSlots - g) * (kKeys / 8));
      const int row = g + k / (kKeys / 8), col = (k % (kKeys / 8)) * 8;
      *reinterpret_cast<uint4*>(sP + buf * 2 * SM::kSPanel + slot_tile_ofs(row, col)) = make_uint4(0u, 0u, 0u, 0u);
    }
    named_bar(kSoftBar, 128);
    float kl[NT::HV], kh2[NT::HV], vl[NT::HV], vh[NT::HV];
    bool have_k = false, have_v = false;
    for (int base = 0; base < g + 2; base += kRowsPerPass) {
      const int rr = base + grp;
      const int kind = row_kind(rr);
      const bool valid = row_valid(rr);
      float yl[NT::HV], yh[NT::HV];
      if (base == 0) {
        NT::finish(p, kind, sub, valid, in0, cs, sn, yl, yh);
      } else {
        typename NT::In in;
        NT::load(p, b, kind, kind == 0 ? hk * g + rr : hk, sub, valid, in);
        NT::finish(p, kind, sub, valid, in, cs, sn, yl, yh);
      }
      if (!valid) continue;
      // q~, k~, v_eff as stored (bf16)
#pragma unroll
      for (int i = 0; i < NT::HV; ++i) {
        yl[i] = __bfloat162float(__float2bfloat16_rn(yl[i]));
        yh[i] = __bfloat162float(__float2bfloat16_rn(yh[i]));
      }
      if (kind == 0) {
        *reinterpret_cast<uint4*>(sQ + slot_tile_ofs(rr, sub * 8)) =
            make_uint4(pack_bf16x2(yl[0], yl[1]), pack_bf16x2(yl[2], yl[3]), pack_bf16x2(yl[4], yl[5]),
                       pack_bf16x2(yl[6], yl[7]));
        *reinterpret_cast<uint4*>(sQ + slot_tile_ofs(rr, NT::HALF + sub * 8)) =
            make_uint4(pack_bf16x2(yh[0], yh[1]), pack_bf16x2(yh[2], yh[3]), pack_bf16x2(yh[4], yh[5]),
                       pack_bf16x2(yh[6], yh[7]));
      } else {
        const size_t crow = ((static_cast<size_t>(b) * p.T + pos) * p.Hk + hk) * D + sub * NT::HV;
        __nv_bfloat16* cache = kind == 1 ? p.kc : p.vc;
        NT::HVec::store(cache + crow, yl);
        NT::HVec::store(cache + crow + NT::HALF, yh);
        if (kind == 1) {
#pragma unroll
          for (int i = 0; i < NT::HV; ++i) {
            kl[i] = yl[i];
            kh2[i] = yh[i];
          }
          have_k = true;
        } else {
#pragma unroll
          for (int i = 0; i < NT::HV; ++i) {
            vl[i] = yl[i];
            vh[i] = yh[i];
          }
          have_v = true;
        }
      }
    }
    fence_proxy_async_smem();  // the Q tile, to the tensor cores' proxy
    mbar_arrive(q_ready);
    named_bar(kSoftBar, 128);
    if (owns_new) {
      // The new key's score against each query row of the group (its row
      // of K in the staged chunk is not used: the cache row may hold
      // anything until this call writes it).
      for (int h = 0; h < g; ++h) {
        float part_dot = 0.f;
        if (have_k) {
#pragma unroll
          for (int i = 0; i < NT::HV; ++i) {
            const int dl = sub * NT::HV + i, dh = NT::HALF + sub * NT::HV + i;
            part_dot = fmaf(kl[i], __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sQ + slot_tile_ofs(h, dl))),
                            part_dot);
            part_dot = fmaf(kh2[i], __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sQ + slot_tile_ofs(h, dh))),
                            part_dot);
          }
        }
        part_dot = row_sum<NT::LPR>(part_dot);
        if (have_k && sub == 0) s_new[h] = part_dot;
      }
    }
    named_bar(kSoftBar, 128);  // s_new written
    // Pass 1, chunk by chunk as the S^T products complete (while the K
    // chunks still stream): the max per head over all of the split's keys
    // (log2 units).
    float mx[kSlots];
#pragma unroll
    for (int h = 0; h < kSlots; ++h) mx[h] = -INFINITY;
    auto score = [&](const uint32_t (&sr)[kSlots], int h, int c) {
      const int j = c + r;
      const float raw = (owns_new && j == pos) ? s_new[h] : __uint_as_float(sr[h]);
      return (j >= lo && j <= pos) ? raw * p.scale_log2 : -INFINITY;  // a select: NaN rows never leak
    };
    bool ok = true;
    for (int ci = 0; ci < n; ++ci) {
      if (!(ok = mbar_wait(&s_chunk[ci], 0, wc))) break;
      tc_fence_after();
      uint32_t sr[kSlots];
      tmem_ld16(tmem + lane_base + kSlots * (1 + ci), sr);
      tmem_ld_wait();
      const int c = cbase + (ch0 + ci) * kKeys;
#pragma unroll
      for (int h = 0; h < kSlots; ++h)
        if (h < g) mx[h] = fmaxf(mx[h], score(sr, h, c));
    }
    ok = named_bar_and(kSoftBar, 128, ok);
    if (ok) {
#pragma unroll
      for (int h = 0; h < kSlots; ++h) {
        if (h < g) {
          float m = mx[h];
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          if (lane == 0) red[h * 4 + quad] = m;
        }
      }
    }
    ok = named_bar_and(kSoftBar, 128, ok);
    float sum[kSlots];
#pragma unroll
    for (int h = 0; h < kSlots; ++h) {
      mx[h] = h < g ? fmaxf(fmaxf(red[h * 4], red[h * 4 + 1]), fmaxf(red[h * 4 + 2], red[h * 4 + 3])) : 0.f;
      sum[h] = 0.f;
    }
    // Pass 2: probabilities chunk by chunk into the P^T buffers, once the
    // chunk's V tile has landed (its rows outside [lo, pos] zeroed: a zero
    // probability times a NaN would still be NaN; row pos takes v_eff).
    for (int ci = 0; ok && ci < n; ++ci) {
      const int seq = n + ci, st = seq % NS;
      ok = mbar_wait(&full[st], (seq / NS) & 1, wc) && (ci < 2 || mbar_wait(&p_free[ci & 1], ((ci >> 1) - 1) & 1, wc));
      if (!ok) break;
      const int c = cbase + (ch0 + ci) * kKeys;
      uint8_t* sV = smem + st * SM::kTile;
      if (c + r < lo || c + r > pos) {
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<uint4*>(sV + pn * kPanel + r * 128 + ((q ^ (r & 7)) << 4)) =
                make_uint4(0u, 0u, 0u, 0u);  // chunk order rotated per row: no bank conflicts
      }
      if (have_v && pos >= c && pos < c + kKeys) {
        const int rr = pos - c;
        const int dl = sub * NT::HV, dh = NT::HALF + sub * NT::HV;
        *reinterpret_cast<uint4*>(sV + (dl >> 6) * kPanel + rr * 128 + ((((dl & 63) >> 3) ^ (rr & 7)) << 4)) =
            make_uint4(pack_bf16x2(vl[0], vl[1]), pack_bf16x2(vl[2], vl[3]), pack_bf16x2(vl[4], vl[5]),
                       pack_bf16x2(vl[6], vl[7]));
        *reinterpret_cast<uint4*>(sV + (dh >> 6) * kPanel + rr * 128 + ((((dh & 63) >> 3) ^ (rr & 7)) << 4)) =
            make_uint4(pack_bf16x2(vh[0], vh[1]), pack_bf16x2(vh[2], vh[3]), pack_bf16x2(vh[4], vh[5]),
                       pack_bf16x2(vh[6], vh[7]));
      }
      uint32_t sr[kSlots];
      tmem_ld16(tmem + lane_base + kSlots * (1 + ci), sr);
      tmem_ld_wait();
      uint8_t* pbuf = sP + (ci & 1) * 2 * SM::kSPanel;
#pragma unroll
      for (int h = 0; h < kSlots; ++h) {  // rows of unused slots stay zero
        if (h < g) {
          const float e = ex2(score(sr, h, c) - mx[h]);  // masked keys: 2^-inf = 0
          sum[h] += e;
          *reinterpret_cast<__nv_bfloat16*>(pbuf + slot_tile_ofs(h, r)) = __float2bfloat16_rn(e);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_ready[ci & 1]);
    }
    ok = named_bar_and(kSoftBar, 128, ok);
    if (ok) {
#pragma unroll
      for (int h = 0; h < kSlots; ++h) {
        if (h < g) {
          float sm = sum[h];
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
          if (lane == 0) red[h * 4 + quad] = sm;
        }
      }
    }
    ok = named_bar_and(kSoftBar, 128, ok && mbar_wait(o_done, 0, wc));
    if (ok) {
      tc_fence_after();
      uint32_t orr[kSlots];
      tmem_ld16(tmem + lane_base, orr);
      tmem_ld_wait();
      const int d = r;  // column of O
#pragma unroll
      for (int h = 0; h < kSlots; ++h) {
        if (h < g) {
          const float l = (red[h * 4] + red[h * 4 + 1]) + (red[h * 4 + 2] + red[h * 4 + 3]);
          const size_t bh = static_cast<size_t>(b) * p.H + hk * g + h;
          if (p.nsplit == 1) {
            if (d < D) p.O[bh * D + d] = __float2bfloat16_rn(__uint_as_float(orr[h]) / l);
            if (d == 0) p.lse[bh] = (mx[h] + log2f(l)) * 0.69314718055994531f;
          } else {
            if (d < D) p.part_o[part(hk * g + h) * D + d] = __uint_as_float(orr[h]);
            if (d == 0) {
              p.part_ml[part(hk * g + h) * 2] = mx[h];
              p.part_ml[part(hk * g + h) * 2 + 1] = l;
            }
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
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
