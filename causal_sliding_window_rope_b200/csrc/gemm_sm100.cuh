// gemm_sm100.cuh -- bf16 matrix product on tcgen05 tensor cores, the step
// Muon's orthogonalisation is made of (page "5만원으로 나만의 ChatGPT 훈련하는
// 방법", section "2. Muon 옵티마이저 (nanochat/optim.py)": the quintic
// Newton-Schulz iteration A = X^T X; B = b A + c A A; X = a X + X B).
//
//   C[m][n] = alpha * sum_k Aop[m][k] Bop[n][k] + beta * D[m][n]
//
// Aop[m][k] is A[m][k] of a row-major (M x K) A (K-major, A_MN = false) or
// A[k][m] of a row-major (K x M) A (MN-major, A_MN = true); Bop[n][k] is
// B[n][k] of a row-major (N x K) B or B[k][n] of a row-major (K x N) B. So
// X^T X is A_MN = B_MN = true with A = B = X, and X B is A_MN = false,
// B_MN = true. bf16 inputs and D, bf16 (or float32) C, float32 accumulation.
//
// Tiles of 128 x BN of C (BN = 128 or 256: the wider tile halves the operand
// bytes per product, which bound the narrow one), at most one CTA per SM,
// each walking tiles blockIdx.x, blockIdx.x + gridDim.x, ... Warp 0 (one
// thread) loads 64-wide K chunks of both operands by TMA into a ring (128B
// swizzle: a K-major chunk is one panel of 128 or BN rows x 64 K, an
// MN-major chunk panels of 64 K-rows x 64 elements), running ahead across
// tiles; warp 1 owns two BN-column TMEM accumulators and issues 4 MMAs
// (M = 128, N = BN, K = 16) per chunk into the one of the current tile;
// warps 2-5 read the other accumulator back (thread = row of the tile),
// apply alpha and beta D and store the row, so a tile's epilogue overlaps
// the next tile's products. Out-of-range rows, columns and K entries of a
// partial tile read as zero and are not stored.
#pragma once
#include "common.cuh"

namespace cswattn {
namespace gemm {

constexpr int kBM = 128, kBK = 64;
constexpr int kThreads = 192;
constexpr int kOpBytesA = kBM * kBK * 2;  // 16 KB: 128 rows x 64 K
constexpr int kPanelMN = 64 * kBK * 2;     // 8 KB: an MN-major panel, 64 K-rows x 64 elements

// Ring geometry of a BN-wide tile: 192 KB of stages either way.
template <int BN>
struct Geo {
  static constexpr int kOpBytesB = BN * kBK * 2;
  static constexpr int kStageBytes = kOpBytesA + kOpBytesB;
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kOffBar = kStages * kStageBytes;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};

// Up to three operand segments. Along K: the product is the sum over the
// segments of A_s B_s (each with its own K extent; the chunks of segment s
// follow those of s - 1 into the same accumulator). Along M: rows
// [mstart[s], mstart[s+1]) of C take A_s (row m - mstart[s]) with the
// shared B (maps.b[0]); every segment but the last spans whole 128-row tiles.
constexpr int kMaxSeg = 3;
struct Maps {
  CUtensorMap a[kMaxSeg];
  CUtensorMap b[kMaxSeg];
};

struct Params {
  int nseg;                // 1 .. kMaxSeg
  int along_m;             // segments concatenated along M (else along K)
  int kseg[kMaxSeg];       // along K: K extent of each segment
  int mstart[kMaxSeg + 1]; // along M: first row of each segment, then M
  int M, N, K;
  float alpha, beta;
  const __nv_bfloat16* D;  // (M x N) row-major with ldd, or null when beta == 0
  long long ldd;
  __nv_bfloat16* C;        // (M x N) row-major with ldc (bf16 output), or null
  float* C32;              // (M x N) row-major with ldc (float32 output), or null
  long long ldc;
  unsigned long long wait_ns;
};

// TMA loads of one K chunk of an operand of `rows` rows (128 or BN): rows r0..
// of the tile, K from k0. K-major: one rows x 64-K panel. MN-major: rows/64
// panels of 64 K-rows x 64 elements.
template <bool MN, int ROWS>
__device__ __forceinline__ void load_operand(const CUtensorMap* map, uint64_t* bar, uint8_t* dst, int r0,
                                             int k0) {
  if constexpr (MN) {
#pragma unroll
    for (int pn = 0; pn < ROWS / 64; ++pn) tma_load_2d(map, bar, dst + pn * kPanelMN, r0 + 64 * pn, k0);
  } else {
    tma_load_2d(map, bar, dst, k0, r0);
  }
}

// Shared-memory descriptor of an operand chunk and the offset (in 16-byte
// units) of its K-step kk (16 K entries).
template <bool MN>
__device__ __forceinline__ uint64_t operand_desc(uint32_t saddr) {
  return MN ? sdesc_sw128(saddr, kPanelMN, 1024)  // 64-element chunks 8 KB apart
            : sdesc_sw128(saddr, 16, 1024);      // 128-byte rows, 8-row groups
}
template <bool MN>
__device__ __forceinline__ uint64_t kstep_ofs(int kk) {
  return static_cast<uint64_t>((MN ? kk * 16 * 128 : kk * 32) >> 4);
}

// SEG: operands in segments (else one A and one B: maps.a[0], maps.b[0]).
template <bool A_MN, bool B_MN, int BN, bool SEG>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ Maps maps, const Params p) {
  using G = Geo<BN>;
  constexpr int kStages = G::kStages, kStageBytes = G::kStageBytes;
  extern __shared__ uint8_t smem_raw[];
  pdl_launch_dependents();
  uint8_t* smem = smem_align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G::kOffBar);
  uint64_t* full = bars;                      // [kStages]
  uint64_t* empty = bars + kStages;           // [kStages]
  uint64_t* acc_full = bars + 2 * kStages;    // [2] accumulator b holds a finished tile
  uint64_t* acc_empty = bars + 2 * kStages + 2;  // [2] accumulator b read back (4 epilogue warps)
  uint64_t* mma_drain = bars + 2 * kStages + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * kStages + 6);
  const int warp = warp_id(), lane = lane_id();
  // K chunks of a tile (along K: the segments' chunks one after the other).
  int nk = (p.K + kBK - 1) / kBK;
  if (SEG && !p.along_m)
    nk = (p.kseg[0] + kBK - 1) / kBK + (p.nseg > 1 ? (p.kseg[1] + kBK - 1) / kBK : 0) +
         (p.nseg > 2 ? (p.kseg[2] + kBK - 1) / kBK : 0);
  const int ntn = (p.N + BN - 1) / BN;
  const int ntiles = ((p.M + kBM - 1) / kBM) * ntn;
  // Tiles of this CTA: blockIdx.x, + gridDim.x, ... (row-major over the
  // tile grid, so the CTAs in flight share rows of A and columns of B).
  const int my_tiles = static_cast<int>(blockIdx.x) < ntiles
                           ? (ntiles - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                           : 0;
  if (!check_bounds(my_tiles >= 1 && nk >= 1 && p.nseg >= 1 && p.nseg <= kMaxSeg)) return;  // checked build
  auto tile_origin = [&](int li, int& m0, int& n0) {
    const int t = static_cast<int>(blockIdx.x) + li * static_cast<int>(gridDim.x);
    m0 = (t / ntn) * kBM;
    n0 = (t % ntn) * BN;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * BN);  // two accumulators: tile i in columns (i & 1) * BN
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
      // ------------------------------------------------ TMA producer (chunks of all the CTA's tiles)
      // Segment operands by constant index (no dynamic indexing of the
      // kernel parameters): c1, c2 = first chunk of segments 1 and 2 along K.
      const int c1 = (p.kseg[0] + kBK - 1) / kBK;
      const int c2 = c1 + (p.nseg > 1 ? (p.kseg[1] + kBK - 1) / kBK : 0);
      const int m1 = p.mstart[1], m2 = p.mstart[2];
      prefetch_tmap(&maps.a[0]);
      prefetch_tmap(&maps.b[0]);
      if (SEG && p.nseg > 1) {
        prefetch_tmap(&maps.a[1]);
        if (!p.along_m) prefetch_tmap(&maps.b[1]);
      }
      if (SEG && p.nseg > 2) {
        prefetch_tmap(&maps.a[2]);
        if (!p.along_m) prefetch_tmap(&maps.b[2]);
      }
      int issued[kStages] = {};
      bool ok = true;
      for (int li = 0; ok && li < my_tiles; ++li) {
        int m0, n0;
        tile_origin(li, m0, n0);
        // Along M: the tile's segment (tiles never straddle two) and its row in it.
        int sm = 0, ma = m0;
        if (SEG && p.along_m) {
          sm = (p.nseg > 2 && m0 >= m2) ? 2 : ((p.nseg > 1 && m0 >= m1) ? 1 : 0);
          ma = m0 - (sm == 2 ? m2 : (sm == 1 ? m1 : 0));
        }
        for (int c = 0; c < nk; ++c) {
          // Along K: segment of chunk c and the chunk within it.
          int sk = 0, kc = c, sb = 0;
          if constexpr (SEG) {
            sk = p.along_m ? sm : (c >= c2 && p.nseg > 2 ? 2 : (c >= c1 && p.nseg > 1 ? 1 : 0));
            kc = p.along_m ? c : c - (sk == 2 ? c2 : (sk == 1 ? c1 : 0));
            sb = p.along_m ? 0 : sk;
          }
          const CUtensorMap* mapA = sk == 2 ? &maps.a[2] : (sk == 1 ? &maps.a[1] : &maps.a[0]);
          const CUtensorMap* mapB = sb == 2 ? &maps.b[2] : (sb == 1 ? &maps.b[1] : &maps.b[0]);
          const int g = li * nk + c, s = g % kStages, use = g / kStages;
          if (use > 0 && !(ok = mbar_wait(&empty[s], (use - 1) & 1, wc))) break;
          uint8_t* st = smem + s * kStageBytes;
          mbar_expect_tx(&full[s], kStageBytes);
          load_operand<A_MN, kBM>(mapA, &full[s], st, ma, kc * kBK);
          load_operand<B_MN, BN>(mapB, &full[s], st + kOpBytesA, n0, kc * kBK);
          ++issued[s];
        }
      }
      for (int s = 0; s < kStages; ++s)
        if (issued[s] > 0) drain_wait(&full[s], (issued[s] - 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t id = idesc_bf16(kBM, BN, A_MN ? 1 : 0, B_MN ? 1 : 0);
      const uint32_t s0 = smem_u32(smem);
      bool ok = true;
      for (int li = 0; ok && li < my_tiles; ++li) {
        const int b = li & 1, u = li >> 1;
        if (u > 0 && !(ok = mbar_wait(&acc_empty[b], (u - 1) & 1, wc))) break;
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(b * BN);
        for (int kc = 0; kc < nk; ++kc) {
          const int g = li * nk + kc, s = g % kStages, use = g / kStages;
          if (!(ok = mbar_wait(&full[s], use & 1, wc))) break;
          tc_fence_after();
          const uint64_t da = operand_desc<A_MN>(s0 + s * kStageBytes);
          const uint64_t db = operand_desc<B_MN>(s0 + s * kStageBytes + kOpBytesA);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_ss(acc, da + kstep_ofs<A_MN>(kk), db + kstep_ofs<B_MN>(kk), id, (kc > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&acc_full[b]);
      }
      mma_commit(mma_drain);  // every product issued above completes before it fires
      drain_wait(mma_drain, 0);
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2-5)
    const int quad = warp & 3;  // TMEM lanes 32 quad .. 32 quad + 31
    const int r = quad * 32 + lane;
    for (int li = 0; li < my_tiles; ++li) {
      const int b = li & 1, u = li >> 1;
      const bool got = mbar_wait(&acc_full[b], u & 1, wc);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      int m0, n0;
      tile_origin(li, m0, n0);
      const int m = m0 + r;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t a[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + b * BN + c * 32, a);
        tmem_ld_wait();
        if (m >= p.M) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int n = n0 + c * 32 + q * 8;  // 8 columns = 16 bytes
          if (n >= p.N) break;
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = p.alpha * __uint_as_float(a[q * 8 + e]);
          if (p.beta != 0.f) {
            const uint4 uu = *reinterpret_cast<const uint4*>(p.D + m * p.ldd + n);
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&uu);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(h2[e]);
              v[2 * e] = fmaf(p.beta, f.x, v[2 * e]);
              v[2 * e + 1] = fmaf(p.beta, f.y, v[2 * e + 1]);
            }
          }
          if (p.C32) {
            float4* dst = reinterpret_cast<float4*>(p.C32 + m * p.ldc + n);
            dst[0] = make_float4(v[0], v[1], v[2], v[3]);
            dst[1] = make_float4(v[4], v[5], v[6], v[7]);
          } else {
            uint4 w;
            w.x = pack_bf16x2(v[0], v[1]);
            w.y = pack_bf16x2(v[2], v[3]);
            w.z = pack_bf16x2(v[4], v[5]);
            w.w = pack_bf16x2(v[6], v[7]);
            *reinterpret_cast<uint4*>(p.C + m * p.ldc + n) = w;
          }
        }
      }
      // Accumulator b is read: the MMA issuer may start tile li + 2 in it.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * BN);
  }
}

}  // namespace gemm
}  // namespace cswattn
