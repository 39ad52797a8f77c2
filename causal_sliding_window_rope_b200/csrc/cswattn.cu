// cswattn.cu -- C ABI of libcswattn.so: host-side validation, tensor maps,
// launches. Single translation unit (the kernels are in the .cuh files) so
// that every kernel shares one device status word.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <algorithm>
#include <cmath>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/cswattn.h"
#include "common.cuh"
#include "prologue.cuh"
#include "simt_f32.cuh"
#include "bwd_aux.cuh"
#include "fwd_sm100.cuh"
#include "bwd_sm100.cuh"
#include "decode.cuh"
#include "gate.cuh"
#include "gemm_sm100.cuh"
#include "qkv_sm100.cuh"
#include "fp8.cuh"

using namespace cswattn;

namespace {

thread_local std::string t_err;

// NVTX range around each entry point, so a profiler's timeline shows which
// call enqueued which kernels (header-only NVTX: a few instructions when no
// tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};
std::atomic<unsigned long long> g_wait_ns{2000000000ull};
// Floor of the caller's wait limit: far above the latency of any copy, matrix
// product or hand-off between a kernel's roles, so that a short limit only
// ends waits that would not end otherwise.
constexpr uint64_t kMinWaitNs = 1000000ull;  // 1 ms

cswattn_status fail(cswattn_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_err = buf;
  return s;
}

cswattn_status cuda_fail(cudaError_t e, const char* what) {
  return fail(CSWATTN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr int kMaxT = 1 << 20;

struct Shape {
  int B, T, H, Hk, D, W, g;
  bool bf16;
  size_t esize;
  float scale;
};

cswattn_status check_layer(const cswattn_layer* L, Shape* s) {
  if (!L) return fail(CSWATTN_ERR_INVALID_ARG, "layer is NULL");
  if (L->B < 1 || L->T < 1 || L->n_head < 1 || L->n_kv_head < 1 || L->head_dim < 1)
    return fail(CSWATTN_ERR_INVALID_ARG, "B, T, n_head, n_kv_head, head_dim must be >= 1");
  if (L->n_head % L->n_kv_head != 0)
    return fail(CSWATTN_ERR_INVALID_ARG, "n_head (%d) must be a multiple of n_kv_head (%d)",
                L->n_head, L->n_kv_head);
  if (L->window < 1) return fail(CSWATTN_ERR_INVALID_ARG, "window must be >= 1 (got %d)", L->window);
  if (L->has_ve != 0 && L->has_ve != 1) return fail(CSWATTN_ERR_INVALID_ARG, "has_ve must be 0 or 1");
  if (!(L->rope_base > 0.f) || !std::isfinite(L->rope_base))
    return fail(CSWATTN_ERR_INVALID_ARG, "rope_base must be finite and > 0");
  if (!(L->eps >= 0.f) || !std::isfinite(L->eps))
    return fail(CSWATTN_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (!(L->softmax_scale >= 0.f) || !std::isfinite(L->softmax_scale))
    return fail(CSWATTN_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  if (L->dtype != CSWATTN_F32 && L->dtype != CSWATTN_BF16)
    return fail(CSWATTN_ERR_INVALID_ARG, "dtype must be CSWATTN_F32 or CSWATTN_BF16");
  if (L->T > kMaxT) return fail(CSWATTN_ERR_UNSUPPORTED, "T = %d exceeds %d", L->T, kMaxT);
  const long long rows = static_cast<long long>(L->B) * L->T * L->n_head;
  if (rows * L->head_dim >= (1ll << 40) || static_cast<long long>(L->B) * L->n_kv_head * 2048 >= (1ll << 31))
    return fail(CSWATTN_ERR_UNSUPPORTED, "layer too large");
  if (L->dtype == CSWATTN_BF16) {
    if (L->head_dim != 128 && L->head_dim != 64)
      return fail(CSWATTN_ERR_UNSUPPORTED, "bf16 supports head_dim 64 and 128 (got %d)", L->head_dim);
  } else {
    const int d = L->head_dim;
    if (d != 4 && d != 8 && d != 16 && d != 32 && d != 64 && d != 128)
      return fail(CSWATTN_ERR_UNSUPPORTED, "f32 supports head_dim 4, 8, 16, 32, 64, 128 (got %d)", d);
  }
  s->B = L->B;
  s->T = L->T;
  s->H = L->n_head;
  s->Hk = L->n_kv_head;
  s->D = L->head_dim;
  s->W = L->window < L->T ? L->window : L->T;  // W >= T is plain causal
  s->g = L->n_head / L->n_kv_head;
  s->bf16 = L->dtype == CSWATTN_BF16;
  s->esize = s->bf16 ? 2 : 4;
  s->scale = L->softmax_scale > 0.f ? L->softmax_scale : 1.0f / std::sqrt(static_cast<float>(L->head_dim));
  return CSWATTN_OK;
}

cswattn_status check_ptr(const void* p, const char* name, size_t align) {
  if (!p) return fail(CSWATTN_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned(p, align)) return fail(CSWATTN_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
  return CSWATTN_OK;
}

#define CHECK_PTR(p, a)                                          \
  do {                                                           \
    cswattn_status st_ = check_ptr((p), #p, (a));                \
    if (st_ != CSWATTN_OK) return st_;                           \
  } while (0)

void fill_omega(float* omega, int D, float base) {
  for (int i = 0; i < D / 2; ++i)
    omega[i] = static_cast<float>(std::pow(static_cast<double>(base), -2.0 * i / D));
}

// ---------------------------------------------------------------- tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

cswattn_status get_encoder(EncodeTiledFn* fn) {
  static std::once_flag once;
  static EncodeTiledFn cached = nullptr;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) cached = reinterpret_cast<EncodeTiledFn>(f);
  });
  if (!cached) return fail(CSWATTN_ERR_CUDA, "cuTensorMapEncodeTiled unavailable: %s", cudaGetErrorString(err));
  *fn = cached;
  return CSWATTN_OK;
}

// Tensor map of a (outer, T, heads, D) row-major tensor of bf16 (or
// float32), D <= 128, viewed as 4-D (D, heads, T, outer); a box is one
// 128-byte column panel (64 bf16 or 32 float32) of `rows` rows of one head,
// 128B-swizzled; out-of-range rows and columns read as zero. The
// tensor-core kernels always move 128 columns: for D = 64 the second bf16
// panel lies past the tensor, loads fill it with zeros and stores skip it.
cswattn_status make_map(CUtensorMap* map, const void* base, int outer, int T, int heads, int rows,
                        int D, bool f32 = false) {
  EncodeTiledFn enc;
  cswattn_status s = get_encoder(&enc);
  if (s != CSWATTN_OK) return s;
  const cuuint64_t es = f32 ? 4 : 2;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(outer)};
  const cuuint64_t strides[3] = {D * es, static_cast<cuuint64_t>(heads) * D * es,
                                 static_cast<cuuint64_t>(T) * heads * D * es};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / es), 1, static_cast<cuuint32_t>(rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSWATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return CSWATTN_OK;
}

// Tensor map of a row-major bf16 (or, with `bytes`, 8-bit) matrix of
// `rows` rows of `inner` contiguous elements, `ld` elements apart, viewed as
// 2-D (inner, rows); a box is box_inner x box_rows (128B swizzle: 128-byte
// box rows), out-of-range elements read as zero.
cswattn_status make_map_2d(CUtensorMap* map, const void* base, long long inner, long long rows, long long ld,
                           int box_inner, int box_rows, bool bytes = false) {
  EncodeTiledFn enc;
  cswattn_status s = get_encoder(&enc);
  if (s != CSWATTN_OK) return s;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * (bytes ? 1 : 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSWATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return CSWATTN_OK;
}

// Tensor map of a bf16 (rows, heads, D) row-major tensor (tokens flattened),
// viewed as 3-D (D, heads, rows); a box is one 128-byte column panel of
// `box_rows` rows of one head (128B swizzle); rows past the end are not
// written by stores.
cswattn_status make_map_3d(CUtensorMap* map, const void* base, long long rows, int heads, int D, int box_rows) {
  EncodeTiledFn enc;
  cswattn_status s = get_encoder(&enc);
  if (s != CSWATTN_OK) return s;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(heads) * D * 2};
  const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSWATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return CSWATTN_OK;
}

// Raises a kernel's dynamic shared-memory limit on the current device, once
// per (kernel, device): the attribute belongs to the device's context, so a
// process that drives several GPUs sets it on each.
template <typename Kernel>
cswattn_status set_smem(Kernel k, int bytes) {
  static std::mutex mu;
  static std::vector<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const void* key = reinterpret_cast<const void*>(k);
  std::lock_guard<std::mutex> lock(mu);
  for (const auto& d : done)
    if (d.first == key && d.second == dev) return CSWATTN_OK;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  done.emplace_back(key, dev);
  return CSWATTN_OK;
}

// First failed launch of the current call on this thread, reported (and
// cleared) by launched().
thread_local cudaError_t t_launch_error = cudaSuccess;

// Launch with programmatic stream serialization: the kernel may begin
// while the previous kernel in the stream finishes (every kernel of this
// library waits for its predecessor before touching global memory).
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess && t_launch_error == cudaSuccess) t_launch_error = e;
}

cswattn_status launched(const char* what) {
  cudaError_t e = t_launch_error;
  t_launch_error = cudaSuccess;
  const cudaError_t last = cudaGetLastError();
  if (e == cudaSuccess) e = last;
  if (e != cudaSuccess) return cuda_fail(e, what);
  return CSWATTN_OK;
}

// Launch shape of a row kernel (prologue, backward preprocess, backward
// epilogue). The staged form copies a CTA's whole token block into shared
// memory up front: it takes as many tokens as fit in kRowStageTarget bytes
// (so that several CTAs per SM have their copies in flight), at most
// kPrologueTok. A layer whose single token needs more than kRowStageMax
// bytes runs the direct form (tok = 0), which reads global memory row by row.
constexpr size_t kRowStageTarget = 64u << 10;
constexpr size_t kRowStageMax = 200u << 10;

struct RowLaunch {
  int tok;       // tokens per CTA of the staged form, 0 for the direct form
  size_t smem;   // dynamic shared memory of the staged form
  unsigned grid;
};

RowLaunch row_launch(long long ntok, size_t per_tok) {
  RowLaunch r{0, 0, 0};
  if (per_tok > 0 && per_tok <= kRowStageMax) {
    r.tok = static_cast<int>(std::min<size_t>(kPrologueTok, std::max<size_t>(1, kRowStageTarget / per_tok)));
    r.smem = r.tok * per_tok;
  }
  const int per_cta = r.tok > 0 ? r.tok : kPrologueTok;
  r.grid = static_cast<unsigned>((ntok + per_cta - 1) / per_cta);
  return r;
}

// With prepare_only, sets what the launch needs (the shared-memory limit)
// and launches nothing: a call that may fail is made before anything of an
// entry point is enqueued.
template <auto STAGED_K, auto DIRECT_K, typename P>
cswattn_status launch_rows(P p, const RowLaunch& r, cudaStream_t st, bool prepare_only) {
  p.wait_ns = g_wait_ns.load();
  if (r.tok > 0) {
    cswattn_status e = set_smem(STAGED_K, static_cast<int>(kRowStageMax));
    if (e != CSWATTN_OK || prepare_only) return e;
    p.tok = r.tok;
    launch_pdl(STAGED_K, dim3(r.grid), dim3(kPrologueThreads), r.smem, st, p);
  } else {
    if (prepare_only) return CSWATTN_OK;
    p.tok = kPrologueTok;
    launch_pdl(DIRECT_K, dim3(r.grid), dim3(kPrologueThreads), 0, st, p);
  }
  return CSWATTN_OK;
}

template <typename T>
cswattn_status launch_prologue(const Shape& s, const PrologueParams& pp, cudaStream_t st) {
  const RowLaunch r = row_launch(static_cast<long long>(s.B) * s.T,
                                 prologue_stage_bytes(1, s.H, s.Hk, s.D, s.esize, pp.has_ve != 0));
#define CSW_ROWS(D_) launch_rows<prologue_kernel<T, D_, true>, prologue_kernel<T, D_, false>>(pp, r, st, false)
  switch (s.D) {
    case 4: if constexpr (sizeof(T) == 4) return CSW_ROWS(4); break;
    case 8: if constexpr (sizeof(T) == 4) return CSW_ROWS(8); break;
    case 16: if constexpr (sizeof(T) == 4) return CSW_ROWS(16); break;
    case 32: if constexpr (sizeof(T) == 4) return CSW_ROWS(32); break;
    case 64: return CSW_ROWS(64);
    default: return CSW_ROWS(128);
  }
#undef CSW_ROWS
  return fail(CSWATTN_ERR_UNSUPPORTED, "prologue: head_dim %d", s.D);
}

template <typename T>
cswattn_status launch_epilogue(const Shape& s, const EpiParams& ep, cudaStream_t st, bool prepare_only) {
  const RowLaunch r = row_launch(static_cast<long long>(s.B) * s.T,
                                 epilogue_stage_bytes(1, s.H, s.Hk, s.D, s.esize, ep.parts, ep.has_ve != 0));
#define CSW_ROWS(D_) launch_rows<epilogue_kernel<T, D_, true>, epilogue_kernel<T, D_, false>>(ep, r, st, prepare_only)
  switch (s.D) {
    case 4: if constexpr (sizeof(T) == 4) return CSW_ROWS(4); break;
    case 8: if constexpr (sizeof(T) == 4) return CSW_ROWS(8); break;
    case 16: if constexpr (sizeof(T) == 4) return CSW_ROWS(16); break;
    case 32: if constexpr (sizeof(T) == 4) return CSW_ROWS(32); break;
    case 64: return CSW_ROWS(64);
    default: return CSW_ROWS(128);
  }
#undef CSW_ROWS
  return fail(CSWATTN_ERR_UNSUPPORTED, "epilogue: head_dim %d", s.D);
}

template <typename T>
cswattn_status launch_preprocess(const Shape& s, const PreParams& pp, cudaStream_t st, bool prepare_only) {
  const RowLaunch r = row_launch(static_cast<long long>(s.B) * s.T,
                                 preprocess_stage_bytes(1, s.H, s.D, s.esize));
#define CSW_ROWS(D_) launch_rows<preprocess_kernel<T, D_, true>, preprocess_kernel<T, D_, false>>(pp, r, st, prepare_only)
  switch (s.D) {
    case 4: if constexpr (sizeof(T) == 4) return CSW_ROWS(4); break;
    case 8: if constexpr (sizeof(T) == 4) return CSW_ROWS(8); break;
    case 16: if constexpr (sizeof(T) == 4) return CSW_ROWS(16); break;
    case 32: if constexpr (sizeof(T) == 4) return CSW_ROWS(32); break;
    case 64: return CSW_ROWS(64);
    default: return CSW_ROWS(128);
  }
#undef CSW_ROWS
  return fail(CSWATTN_ERR_UNSUPPORTED, "preprocess: head_dim %d", s.D);
}

void launch_simt_fwd(const Shape& s, const SimtParams& sp, cudaStream_t st) {
  const long long rows = static_cast<long long>(s.B) * s.H * s.T;
  const unsigned grid = static_cast<unsigned>((rows + 127) / 128);
  switch (s.D) {
    case 4: simt_fwd_kernel<4><<<grid, 128, 0, st>>>(sp); break;
    case 8: simt_fwd_kernel<8><<<grid, 128, 0, st>>>(sp); break;
    case 16: simt_fwd_kernel<16><<<grid, 128, 0, st>>>(sp); break;
    case 32: simt_fwd_kernel<32><<<grid, 128, 0, st>>>(sp); break;
    case 64: simt_fwd_kernel<64><<<grid, 128, 0, st>>>(sp); break;
    default: simt_fwd_kernel<128><<<grid, 128, 0, st>>>(sp); break;
  }
}

void launch_simt_bwd(const Shape& s, const SimtParams& sp, cudaStream_t st) {
  const long long qrows = static_cast<long long>(s.B) * s.H * s.T;
  const long long krows = static_cast<long long>(s.B) * s.Hk * s.T;
  const unsigned gq = static_cast<unsigned>((qrows + 127) / 128);
  const unsigned gk = static_cast<unsigned>((krows + 127) / 128);
  switch (s.D) {
#define CSW_CASE(DD)                                        \
  case DD:                                                  \
    simt_bwd_dq_kernel<DD><<<gq, 128, 0, st>>>(sp);         \
    simt_bwd_dkv_kernel<DD><<<gk, 128, 0, st>>>(sp);        \
    break;
    CSW_CASE(4)
    CSW_CASE(8)
    CSW_CASE(16)
    CSW_CASE(32)
    CSW_CASE(64)
    default:
      simt_bwd_dq_kernel<128><<<gq, 128, 0, st>>>(sp);
      simt_bwd_dkv_kernel<128><<<gk, 128, 0, st>>>(sp);
      break;
#undef CSW_CASE
  }
}

// ---------------------------------------------------------------- self-test

// One thread waits, with the kernels' bounded wait, on a barrier nothing
// arrives on; the wait runs out and records the timeout status.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
    const WaitCtx wc{&abort_flag, limit_ns};
    (void)mbar_wait(&bar, 0, wc);
  }
}

// ---------------------------------------------------------------- timing

std::atomic<int> g_timing{0};
std::mutex g_timing_mu;
struct EventPair {
  cudaEvent_t a = nullptr, b = nullptr;
  int kind = 0;
};
std::vector<EventPair> g_pool;   // created once, reused
size_t g_used = 0;

// Records a start event for `kind` when timing is on; returns the pair index
// (or -1). Call timing_end(idx) after the launch.
long timing_begin(int kind, cudaStream_t st) {
  if (!g_timing.load()) return -1;
  std::lock_guard<std::mutex> lk(g_timing_mu);
  if (g_used == g_pool.size()) {
    EventPair e;
    if (cudaEventCreate(&e.a) != cudaSuccess || cudaEventCreate(&e.b) != cudaSuccess) return -1;
    g_pool.push_back(e);
  }
  EventPair& e = g_pool[g_used];
  e.kind = kind;
  if (cudaEventRecord(e.a, st) != cudaSuccess) return -1;
  return static_cast<long>(g_used++);
}

void timing_end(long idx, cudaStream_t st) {
  if (idx < 0) return;
  std::lock_guard<std::mutex> lk(g_timing_mu);
  cudaEventRecord(g_pool[static_cast<size_t>(idx)].b, st);
}

struct ScopedTiming {
  long idx;
  cudaStream_t st;
  ScopedTiming(int kind, cudaStream_t s) : idx(timing_begin(kind, s)), st(s) {}
  ~ScopedTiming() { timing_end(idx, st); }
};

size_t pad256(size_t x) { return (x + 255) & ~size_t(255); }

struct Workspace {
  float *dq_acc, *dk_acc, *dv_acc, *delta, *nlse2;
  int Tpad;
  size_t bytes;
};

int padded_T(int T) { return (T + 63) / 64 * 64; }

// CTAs per KV tile in the tensor-core backward: heavy tiles (many query
// steps) are split so that the largest CTA holds at most about half the
// average work of an SM (148 SMs). 1 for the fp32 path.
int bwd_parts(const Shape& s) {
  if (!s.bf16) return 1;
  const int nkv = (s.T + 127) / 128;
  long long total = 0, nmax = 0;
  for (int j = 0; j < nkv; ++j) {
    const long long last = std::min<long long>(s.T - 1, static_cast<long long>(j) * 128 + 127 + s.W - 1);
    const long long n = static_cast<long long>(s.g) * (last / 64 - 2 * j + 1);
    total += n;
    nmax = std::max(nmax, n);
  }
  total *= static_cast<long long>(s.B) * s.Hk;
  // Parts per key tile: about 1.5 x (heaviest tile / average work per SM of
  // a 148-SM B200), measured best on the d24 workload among 1, 1.5, 2 and 3.
  const long long want = (3 * nmax * 148 + 2 * total - 1) / std::max(2 * total, 1ll);
  return static_cast<int>(std::min<long long>(8, std::max<long long>(1, want)));
}

Workspace carve(const Shape& s, void* base) {
  const size_t nq = static_cast<size_t>(s.B) * s.H * s.T * s.D;
  const size_t nk = static_cast<size_t>(s.B) * s.T * s.Hk * s.D * bwd_parts(s);
  const size_t nr = static_cast<size_t>(s.B) * s.H * padded_T(s.T);
  Workspace w;
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  w.dq_acc = reinterpret_cast<float*>(p + off);
  off += pad256(nq * 4);
  w.dk_acc = reinterpret_cast<float*>(p + off);
  off += pad256(nk * 4);
  w.dv_acc = reinterpret_cast<float*>(p + off);
  off += pad256(nk * 4);
  w.delta = reinterpret_cast<float*>(p + off);
  off += pad256(nr * 4);
  w.nlse2 = reinterpret_cast<float*>(p + off);
  off += pad256(nr * 4);
  w.Tpad = padded_T(s.T);
  w.bytes = off;
  return w;
}

// ---------------------------------------------------------------- fixed scratch

// Backward scratch of attn_bwd_noalloc, for callers that cannot allocate
// device memory. Every GPU that loads this library holds it until exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[CSWATTN_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// that device current, on every call: the lookup is a host-side table read
// once the module is loaded, and a fresh lookup stays right after a device
// reset gives the array a new address. (Under lazy module loading the first
// lookup on a device loads the module, which reserves the array there.)
cswattn_status noalloc_scratch(void** out) {
  void* ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
  *out = ptr;
  return CSWATTN_OK;
}

}  // namespace

// ---------------------------------------------------------------- matrix product

struct GemmArgs {
  int M, N, K;
  bool a_mn, b_mn;
  const void *A, *B, *D;
  long long lda, ldb, ldd, ldc;
  float alpha, beta;
  void* C;
  bool c_f32 = false;  // C is float32 (else bf16)
};

// With `operands` false (a segmented product) A, B, lda and ldb are the
// segments' and are checked per segment by run_gemm.
cswattn_status check_gemm(const GemmArgs& g, bool operands = true) {
  if (g.M < 1 || g.N < 1 || g.K < 1) return fail(CSWATTN_ERR_INVALID_ARG, "M, N, K must be >= 1");
  if (g.M > (1 << 30) || g.N > (1 << 30) || g.K > (1 << 30)) return fail(CSWATTN_ERR_UNSUPPORTED, "matrix too large");
  if (g.N % 8 != 0) return fail(CSWATTN_ERR_UNSUPPORTED, "N must be a multiple of 8 (got %d)", g.N);
  const long long a_inner = g.a_mn ? g.M : g.K, b_inner = g.b_mn ? g.N : g.K;
  if ((operands && (g.lda < a_inner || g.ldb < b_inner)) || g.ldc < g.N || (g.beta != 0.f && g.ldd < g.N))
    return fail(CSWATTN_ERR_INVALID_ARG, "a leading dimension is smaller than its row");
  if ((operands && (g.lda % 8 || g.ldb % 8)) || g.ldc % 8 || (g.beta != 0.f && g.ldd % 8))
    return fail(CSWATTN_ERR_INVALID_ARG, "leading dimensions must be multiples of 8 elements");
  if (g.c_f32 && g.beta != 0.f) return fail(CSWATTN_ERR_UNSUPPORTED, "a float32 C takes no beta D term");
  if (operands) {
    CHECK_PTR(g.A, 16);
    CHECK_PTR(g.B, 16);
  }
  CHECK_PTR(g.C, 16);
  if (g.beta != 0.f) CHECK_PTR(g.D, 16);
  if (g.C == g.A || g.C == g.B) return fail(CSWATTN_ERR_INVALID_ARG, "C must not alias A or B");
  if (!std::isfinite(g.alpha) || !std::isfinite(g.beta)) return fail(CSWATTN_ERR_INVALID_ARG, "alpha, beta must be finite");
  return CSWATTN_OK;
}

// Tile width of a product: 256 columns when that still gives at least one
// tile per SM (148), else 128 (more, smaller tiles fill the SMs better).
int gemm_bn(int M, int N) {
  const long long t256 = static_cast<long long>((M + gemm::kBM - 1) / gemm::kBM) * ((N + 255) / 256);
  return t256 >= 148 ? 256 : 128;
}

template <bool AMN, bool BMN, int BN>
cswattn_status launch_gemm_t(const gemm::Maps& maps, const gemm::Params& gp, int M, int N, cudaStream_t st,
                             bool prepare_only) {
  constexpr int kSmem = gemm::Geo<BN>::kSmemBytes;
  auto kern = gp.nseg > 1 ? gemm::gemm_kernel<AMN, BMN, BN, true> : gemm::gemm_kernel<AMN, BMN, BN, false>;
  const cswattn_status e = set_smem(kern, kSmem);
  if (e != CSWATTN_OK || prepare_only) return e;
  // Persistent: at most one CTA per SM (148), each walking its share of the tiles.
  const long long tiles = static_cast<long long>((N + BN - 1) / BN) * ((M + gemm::kBM - 1) / gemm::kBM);
  const dim3 grid(static_cast<unsigned>(std::min<long long>(tiles, 148)));
  launch_pdl(kern, grid, dim3(gemm::kThreads), kSmem, st, maps, gp);
  return CSWATTN_OK;
}

template <int BN>
cswattn_status launch_gemm_bn(int which, const gemm::Maps& maps, const gemm::Params& gp, int M, int N,
                              cudaStream_t st, bool prepare_only) {
  switch (which) {
    case 0: return launch_gemm_t<false, false, BN>(maps, gp, M, N, st, prepare_only);
    case 1: return launch_gemm_t<false, true, BN>(maps, gp, M, N, st, prepare_only);
    case 2: return launch_gemm_t<true, false, BN>(maps, gp, M, N, st, prepare_only);
    default: return launch_gemm_t<true, true, BN>(maps, gp, M, N, st, prepare_only);
  }
}

// Operand segments of one product (see gemm::Maps): segment s has operands
// A[s], B[s] (along M: B[0] alone) with leading dimensions lda[s], ldb[s],
// and extent ext[s]: its K (along K) or its rows of M (along M).
struct GemmSegs {
  int n = 0;  // 0: the product of the GemmArgs alone
  bool along_m = false;
  const void* A[gemm::kMaxSeg] = {};
  const void* B[gemm::kMaxSeg] = {};
  long long lda[gemm::kMaxSeg] = {}, ldb[gemm::kMaxSeg] = {};
  int ext[gemm::kMaxSeg] = {};
};

// Validated product, tensor maps built and shared-memory limits set before
// the launch; nothing is enqueued when a check fails. With segments, g holds
// the whole product's M, N, K, layouts and output (its A, B, lda, ldb are
// not used).
cswattn_status run_gemm(const GemmArgs& g, cudaStream_t st, const GemmSegs* sg = nullptr) {
  cswattn_status e = check_gemm(g, sg == nullptr);
  if (e != CSWATTN_OK) return e;
  if ((g.M + gemm::kBM - 1) / gemm::kBM > 65535) return fail(CSWATTN_ERR_UNSUPPORTED, "M too large");
  GemmSegs one;
  if (!sg) {
    one.n = 1;
    one.A[0] = g.A;
    one.B[0] = g.B;
    one.lda[0] = g.lda;
    one.ldb[0] = g.ldb;
    one.ext[0] = g.K;
    sg = &one;
  }
  if (sg->n < 1 || sg->n > gemm::kMaxSeg) return fail(CSWATTN_ERR_INVALID_ARG, "1 to 3 operand segments");
  const int bn = gemm_bn(g.M, g.N);
  gemm::Maps maps;
  gemm::Params gp;
  gp.nseg = sg->n;
  gp.along_m = sg->along_m ? 1 : 0;
  int sum = 0;
  for (int s = 0; s < sg->n; ++s) {
    const int ext = sg->ext[s];
    const int Ms = sg->along_m ? ext : g.M, Ks = sg->along_m ? g.K : ext;
    if (ext < 1) return fail(CSWATTN_ERR_INVALID_ARG, "an operand segment is empty");
    if (sg->along_m && s + 1 < sg->n && ext % gemm::kBM != 0)
      return fail(CSWATTN_ERR_UNSUPPORTED, "along M, every segment but the last spans whole 128-row tiles");
    CHECK_PTR(sg->A[s], 16);
    const long long a_inner = g.a_mn ? Ms : Ks;
    if (sg->lda[s] < a_inner || sg->lda[s] % 8) return fail(CSWATTN_ERR_INVALID_ARG, "segment lda");
    if ((e = g.a_mn ? make_map_2d(&maps.a[s], sg->A[s], Ms, Ks, sg->lda[s], 64, 64)
                    : make_map_2d(&maps.a[s], sg->A[s], Ks, Ms, sg->lda[s], 64, 128)) != CSWATTN_OK)
      return e;
    if (!sg->along_m || s == 0) {
      CHECK_PTR(sg->B[s], 16);
      const long long b_inner = g.b_mn ? g.N : Ks;
      if (sg->ldb[s] < b_inner || sg->ldb[s] % 8) return fail(CSWATTN_ERR_INVALID_ARG, "segment ldb");
      if ((e = g.b_mn ? make_map_2d(&maps.b[s], sg->B[s], g.N, Ks, sg->ldb[s], 64, 64)
                      : make_map_2d(&maps.b[s], sg->B[s], Ks, g.N, sg->ldb[s], 64, bn)) != CSWATTN_OK)
        return e;
    } else {
      maps.b[s] = maps.b[0];
    }
    gp.kseg[s] = Ks;
    gp.mstart[s] = sum;
    sum += ext;
  }
  for (int s = sg->n; s < gemm::kMaxSeg; ++s) {
    maps.a[s] = maps.a[0];
    maps.b[s] = maps.b[0];
    gp.kseg[s] = 0;
    gp.mstart[s] = sum;
  }
  gp.mstart[gemm::kMaxSeg] = sum;
  if (sum != (sg->along_m ? g.M : g.K))
    return fail(CSWATTN_ERR_INVALID_ARG, "the segments do not add up to %s", sg->along_m ? "M" : "K");
  const int which = (g.a_mn ? 2 : 0) + (g.b_mn ? 1 : 0);
  gp.M = g.M;
  gp.N = g.N;
  gp.K = g.K;
  gp.alpha = g.alpha;
  gp.beta = g.beta;
  gp.D = static_cast<const __nv_bfloat16*>(g.D);
  gp.ldd = g.ldd;
  gp.C = g.c_f32 ? nullptr : static_cast<__nv_bfloat16*>(g.C);
  gp.C32 = g.c_f32 ? static_cast<float*>(g.C) : nullptr;
  gp.ldc = g.ldc;
  gp.wait_ns = g_wait_ns.load();
  e = bn == 256 ? launch_gemm_bn<256>(which, maps, gp, g.M, g.N, st, true)
                : launch_gemm_bn<128>(which, maps, gp, g.M, g.N, st, true);
  if (e != CSWATTN_OK) return e;
  {
    ScopedTiming tm(CSWATTN_K_GEMM, st);
    e = bn == 256 ? launch_gemm_bn<256>(which, maps, gp, g.M, g.N, st, false)
                  : launch_gemm_bn<128>(which, maps, gp, g.M, g.N, st, false);
  }
  if (e != CSWATTN_OK) return e;
  return launched("matrix product launch");
}

struct NsWorkspace {
  void *A, *B, *X;
  size_t bytes;
};

NsWorkspace carve_ns(int m, int n, void* base) {
  uint8_t* p = static_cast<uint8_t*>(base);
  NsWorkspace w;
  size_t off = 0;
  w.A = p + off;
  off += pad256(static_cast<size_t>(n) * n * 2);
  w.B = p + off;
  off += pad256(static_cast<size_t>(n) * n * 2);
  w.X = p + off;
  off += pad256(static_cast<size_t>(m) * n * 2);
  w.bytes = off;
  return w;
}

// ---------------------------------------------------------------- decode

struct DecodeWorkspace {
  float *part_ml, *part_o;
  int nsplit;
  size_t bytes;
};

DecodeWorkspace carve_decode(const Shape& s, void* base) {
  DecodeWorkspace w;
  w.nsplit = dec::decode_nsplit(s.B, s.Hk, s.T, s.W);
  const size_t rows = static_cast<size_t>(s.B) * s.H;
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  w.part_ml = reinterpret_cast<float*>(p + off);
  off += pad256(rows * w.nsplit * 2 * 4);
  w.part_o = reinterpret_cast<float*>(p + off);
  off += pad256(rows * w.nsplit * s.D * 4);
  w.bytes = off;
  return w;
}

cswattn_status check_decode_layer(const cswattn_layer* layer, Shape* s) {
  cswattn_status st = check_layer(layer, s);
  if (st != CSWATTN_OK) return st;
  if (!s->bf16) return fail(CSWATTN_ERR_UNSUPPORTED, "attn_decode supports bf16 layers only");
  if (s->g > dec::kMaxGroup)
    return fail(CSWATTN_ERR_UNSUPPORTED, "attn_decode supports up to %d query heads per KV head (got %d)",
                dec::kMaxGroup, s->g);
  if (s->B > 65535 || dec::decode_nsplit(s->B, s->Hk, s->T, s->W) > 65535)  // grid of the split-KV kernel
    return fail(CSWATTN_ERR_UNSUPPORTED, "attn_decode supports B <= 65535 and at most 65535 key chunks");
  return CSWATTN_OK;
}

template <int D>
cswattn_status launch_decode(const Shape& s, const CUtensorMap& mk, const CUtensorMap& mv,
                             const dec::AttnParams& ap, const dec::CombineParams& cp, cudaStream_t st) {
  constexpr int kSmem = dec::DecSmem<D>::kBytes;
  cswattn_status e = set_smem(dec::decode_attn_kernel<D>, kSmem);
  if (e != CSWATTN_OK) return e;
  launch_pdl(dec::decode_attn_kernel<D>, dim3(s.Hk, ap.nsplit, s.B), dim3(dec::kDecThreads), kSmem, st, mk, mv,
             ap);
  // With one split per (sequence, KV head) the attention kernel writes O and lse itself.
  if (ap.nsplit > 1) launch_pdl(dec::decode_combine_kernel<D>, dim3(s.B * s.H), dim3(D), 0, st, cp);
  return CSWATTN_OK;
}

extern "C" {

int cswattn_version(void) { return (1 << 16) | 0; }

const char* cswattn_last_error(void) { return t_err.c_str(); }

uint64_t cswattn_set_wait_limit_ns(uint64_t ns) {
  const uint64_t v = ns < kMinWaitNs ? kMinWaitNs : ns;
  g_wait_ns.store(v);
  return v;
}

cswattn_status cswattn_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1000) limit_ns = 1000;
  if (limit_ns > 1000000000ull) limit_ns = 1000000000ull;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  return launched("self-test launch");
}

void cswattn_set_timing(int enable) { g_timing.store(enable ? 1 : 0); }

cswattn_status cswattn_kernel_times(double* ms, int* launches) {
  std::lock_guard<std::mutex> lk(g_timing_mu);
  double acc[CSWATTN_NUM_KERNELS] = {0};
  int cnt[CSWATTN_NUM_KERNELS] = {0};
  cswattn_status st = CSWATTN_OK;
  for (size_t i = 0; i < g_used; ++i) {
    float t = 0.f;
    cudaError_t e = cudaEventSynchronize(g_pool[i].b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, g_pool[i].a, g_pool[i].b);
    if (e != cudaSuccess) {
      st = cuda_fail(e, "cudaEventElapsedTime");
      continue;
    }
    acc[g_pool[i].kind] += t;
    cnt[g_pool[i].kind] += 1;
  }
  g_used = 0;
  for (int k = 0; k < CSWATTN_NUM_KERNELS; ++k) {
    if (ms) ms[k] = acc[k];
    if (launches) launches[k] = cnt[k];
  }
  return st;
}

cswattn_status cswattn_sync_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, g_status, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol");
  if (v != 0) {
    e = cudaMemcpyToSymbol(g_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyToSymbol");
    if (v & kStatusBounds)
      return fail(CSWATTN_ERR_BOUNDS, "a device-side bounds check failed; the access was skipped (status 0x%x)", v);
    if (v & kStatusTimeout) return fail(CSWATTN_ERR_TIMEOUT, "a device-side wait ran out (status 0x%x)", v);
    if (v & kStatusRange)
      return fail(CSWATTN_ERR_INVALID_ARG, "a decode step met a cache length outside [0, T) (status 0x%x)", v);
  }
  return CSWATTN_OK;
}

}  // extern "C"

namespace {

// The gate's projection inputs of attn_prologue_gated (null for attn_prologue).
struct GateIn {
  const void* x;
  long long x_stride;
  int channels;
  const void* w;
  void* logits_out;
};

cswattn_status prologue_impl(const cswattn_layer* layer, const void* q, const void* k, const void* v,
                             const void* ve, const void* gate, const GateIn* gi, void* q_out,
                             void* k_out, void* v_out, float* rstd_q, float* rstd_k, void* stream) {
  Shape s;
  cswattn_status st = check_layer(layer, &s);
  if (st != CSWATTN_OK) return st;
  CHECK_PTR(q, 16);
  CHECK_PTR(k, 16);
  CHECK_PTR(v, 16);
  CHECK_PTR(q_out, 16);
  CHECK_PTR(k_out, 16);
  CHECK_PTR(v_out, 16);
  CHECK_PTR(rstd_q, 4);
  CHECK_PTR(rstd_k, 4);
  if (layer->has_ve) {
    CHECK_PTR(ve, 16);
    if (!gi) CHECK_PTR(gate, s.esize);
  }
  if (gi) {
    if (!layer->has_ve)
      return fail(CSWATTN_ERR_INVALID_ARG, "the gate projection needs a value embedding (has_ve = 1)");
    if (gi->channels < 1 || gi->x_stride < gi->channels)
      return fail(CSWATTN_ERR_INVALID_ARG, "gate_channels must be >= 1 and <= x_stride (got %d, %lld)",
                  gi->channels, gi->x_stride);
    CHECK_PTR(gi->x, s.esize);
    CHECK_PTR(gi->w, s.esize);
    CHECK_PTR(gi->logits_out, s.esize);
  }
  if (q_out == q || k_out == k || v_out == v || q_out == k_out || k_out == v_out || q_out == v_out)
    return fail(CSWATTN_ERR_INVALID_ARG, "prologue outputs must not alias its inputs or each other");
  PrologueParams pp;
  pp.B = s.B;
  pp.T = s.T;
  pp.H = s.H;
  pp.Hk = s.Hk;
  pp.has_ve = layer->has_ve;
  pp.eps = layer->eps;
  fill_omega(pp.omega, s.D, layer->rope_base);
  pp.q = q;
  pp.k = k;
  pp.v = v;
  pp.ve = ve;
  pp.gate = gate;
  pp.q_out = q_out;
  pp.k_out = k_out;
  pp.v_out = v_out;
  pp.rstd_q = rstd_q;
  pp.rstd_k = rstd_k;
  pp.xg = gi ? gi->x : nullptr;
  pp.x_stride = gi ? gi->x_stride : 0;
  pp.gc = gi ? gi->channels : 0;
  pp.w_gate = gi ? gi->w : nullptr;
  pp.gate_out = gi ? gi->logits_out : nullptr;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  {
    ScopedTiming tm(CSWATTN_K_PROLOGUE, cs);
    st = s.bf16 ? launch_prologue<__nv_bfloat16>(s, pp, cs) : launch_prologue<float>(s, pp, cs);
  }
  if (st != CSWATTN_OK) return st;
  return launched("prologue launch");
}

}  // namespace

extern "C" {

cswattn_status attn_prologue(const cswattn_layer* layer, const void* q, const void* k,
                             const void* v, const void* ve, const void* gate, void* q_out,
                             void* k_out, void* v_out, float* rstd_q, float* rstd_k,
                             void* stream) {
  const NvtxRange nvtx_range("attn_prologue");
  return prologue_impl(layer, q, k, v, ve, gate, nullptr, q_out, k_out, v_out, rstd_q, rstd_k, stream);
}

cswattn_status attn_prologue_gated(const cswattn_layer* layer, const void* q, const void* k,
                                   const void* v, const void* ve, const void* x, long long x_stride,
                                   int gate_channels, const void* w_gate, void* gate_out, void* q_out,
                                   void* k_out, void* v_out, float* rstd_q, float* rstd_k,
                                   void* stream) {
  const NvtxRange nvtx_range("attn_prologue_gated");
  const GateIn gi{x, x_stride, gate_channels, w_gate, gate_out};
  return prologue_impl(layer, q, k, v, ve, nullptr, &gi, q_out, k_out, v_out, rstd_q, rstd_k, stream);
}

cswattn_status attn_gate_bwd(const cswattn_layer* layer, const void* x, long long x_stride,
                             int gate_channels, const void* w_gate, const void* dgate, void* dx,
                             float* dw_gate, void* stream) {
  const NvtxRange nvtx_range("attn_gate_bwd");
  Shape s;
  cswattn_status st = check_layer(layer, &s);
  if (st != CSWATTN_OK) return st;
  if (!layer->has_ve)
    return fail(CSWATTN_ERR_INVALID_ARG, "the gate projection needs a value embedding (has_ve = 1)");
  if (gate_channels < 1 || x_stride < gate_channels)
    return fail(CSWATTN_ERR_INVALID_ARG, "gate_channels must be >= 1 and <= x_stride (got %d, %lld)",
                gate_channels, x_stride);
  CHECK_PTR(x, s.esize);
  CHECK_PTR(w_gate, s.esize);
  CHECK_PTR(dgate, s.esize);
  CHECK_PTR(dx, s.esize);
  CHECK_PTR(dw_gate, 4);
  GateBwdParams gp;
  gp.ntok = static_cast<long long>(s.B) * s.T;
  gp.x_stride = x_stride;
  gp.Hk = s.Hk;
  gp.C = gate_channels;
  gp.dw_blocks = s.Hk * ((gate_channels + 31) / 32) * kGateCluster;
  gp.x = x;
  gp.w = w_gate;
  gp.dgate = dgate;
  gp.dx = dx;
  gp.dw = dw_gate;
  // dx blocks rounded up to whole clusters (the extra blocks have no entries).
  long long dx_blocks = (gp.ntok * gate_channels + kGateDwThreads - 1) / kGateDwThreads;
  dx_blocks = (dx_blocks + kGateCluster - 1) / kGateCluster * kGateCluster;
  if (gp.dw_blocks + dx_blocks > 0x7fffffffll) return fail(CSWATTN_ERR_UNSUPPORTED, "gate backward too large");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(gp.dw_blocks + dx_blocks));
  cfg.blockDim = dim3(kGateDwThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kGateCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  {
    ScopedTiming tm(CSWATTN_K_GATE_BWD, cfg.stream);
    const cudaError_t e = s.bf16 ? cudaLaunchKernelEx(&cfg, gate_bwd_kernel<__nv_bfloat16>, gp)
                                 : cudaLaunchKernelEx(&cfg, gate_bwd_kernel<float>, gp);
    if (e != cudaSuccess) return cuda_fail(e, "gate backward launch");
  }
  return launched("gate backward launch");
}

cswattn_status attn_fwd(const cswattn_layer* layer, const void* q_out, const void* k_out,
                        const void* v_out, void* O, float* lse, void* stream) {
  const NvtxRange nvtx_range("attn_fwd");
  Shape s;
  cswattn_status st = check_layer(layer, &s);
  if (st != CSWATTN_OK) return st;
  CHECK_PTR(q_out, 16);
  CHECK_PTR(k_out, 16);
  CHECK_PTR(v_out, 16);
  CHECK_PTR(O, 16);
  CHECK_PTR(lse, 4);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (!s.bf16) {
    SimtParams sp{};
    sp.B = s.B;
    sp.T = s.T;
    sp.H = s.H;
    sp.Hk = s.Hk;
    sp.W = s.W;
    sp.scale = s.scale;
    sp.q = static_cast<const float*>(q_out);
    sp.k = static_cast<const float*>(k_out);
    sp.v = static_cast<const float*>(v_out);
    sp.out_O = static_cast<float*>(O);
    sp.out_lse = lse;
    {
      ScopedTiming tm(CSWATTN_K_FWD, cs);
      launch_simt_fwd(s, sp, cs);
    }
    return launched("fp32 forward launch");
  }
  CUtensorMap mq, mk, mv;
  if ((st = make_map(&mq, q_out, s.B, s.T, s.H, fwd::kBM, s.D)) != CSWATTN_OK) return st;
  if ((st = make_map(&mk, k_out, s.B, s.T, s.Hk, fwd::kBM, s.D)) != CSWATTN_OK) return st;
  if ((st = make_map(&mv, v_out, s.B, s.T, s.Hk, fwd::kBM, s.D)) != CSWATTN_OK) return st;
  CUtensorMap mo;
  if ((st = make_map(&mo, O, s.B, s.T, s.H, fwd::kBM, s.D)) != CSWATTN_OK) return st;
  if ((st = s.D == 64 ? set_smem(fwd::fwd_kernel<64>, fwd::kSmemBytes)
                      : set_smem(fwd::fwd_kernel<128>, fwd::kSmemBytes)) != CSWATTN_OK)
    return st;
  fwd::Params fp;
  fp.B = s.B;
  fp.T = s.T;
  fp.H = s.H;
  fp.Hk = s.Hk;
  fp.W = s.W;
  fp.g = s.g;
  fp.nq = (s.T + fwd::kBM - 1) / fwd::kBM;
  fp.npairs = (fp.nq * s.g + 1) / 2;
  fp.scale_log2 = s.scale * 1.4426950408889634f;
  fp.O = static_cast<__nv_bfloat16*>(O);
  fp.lse = lse;
  fp.wait_ns = g_wait_ns.load();
  const unsigned grid = static_cast<unsigned>(fp.npairs) * s.B * s.Hk;
  {
    ScopedTiming tm(CSWATTN_K_FWD, cs);
    if (s.D == 64)
      launch_pdl(fwd::fwd_kernel<64>, dim3(grid), dim3(fwd::kThreads), fwd::kSmemBytes, cs, mq, mk, mv, mo, fp);
    else
      launch_pdl(fwd::fwd_kernel<128>, dim3(grid), dim3(fwd::kThreads), fwd::kSmemBytes, cs, mq, mk, mv, mo, fp);
  }
  return launched("forward launch");
}

size_t attn_bwd_workspace_bytes(const cswattn_layer* layer) {
  Shape s;
  if (check_layer(layer, &s) != CSWATTN_OK) return 0;
  return carve(s, nullptr).bytes;
}

cswattn_status attn_bwd(const cswattn_layer* layer, const void* q, const void* k,
                        const void* ve, const void* gate, const void* q_out,
                        const void* k_out, const void* v_out, const float* rstd_q,
                        const float* rstd_k, const void* O, const float* lse, const void* dO,
                        void* dQ, void* dK, void* dV, void* dve, void* dgate, void* workspace,
                        size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx_range("attn_bwd");
  Shape s;
  cswattn_status st = check_layer(layer, &s);
  if (st != CSWATTN_OK) return st;
  CHECK_PTR(q, 16);
  CHECK_PTR(k, 16);
  CHECK_PTR(q_out, 16);
  CHECK_PTR(k_out, 16);
  CHECK_PTR(v_out, 16);
  CHECK_PTR(rstd_q, 4);
  CHECK_PTR(rstd_k, 4);
  CHECK_PTR(O, 16);
  CHECK_PTR(lse, 4);
  CHECK_PTR(dO, 16);
  CHECK_PTR(dQ, 16);
  CHECK_PTR(dK, 16);
  CHECK_PTR(dV, 16);
  CHECK_PTR(workspace, 256);
  if (layer->has_ve) {
    CHECK_PTR(ve, 16);
    CHECK_PTR(gate, s.esize);
    CHECK_PTR(dve, 16);
    CHECK_PTR(dgate, s.esize);
  }
  const Workspace w = carve(s, workspace);
  if (workspace_bytes < w.bytes)
    return fail(CSWATTN_ERR_INVALID_ARG, "workspace has %zu bytes, needs %zu", workspace_bytes, w.bytes);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int parts = bwd_parts(s);

  // Delta = rowsum(dO * O)
  PreParams pre;
  pre.rows = static_cast<long long>(s.B) * s.T * s.H;
  pre.T = s.T;
  pre.H = s.H;
  pre.Tpad = w.Tpad;
  pre.O = O;
  pre.dO = dO;
  pre.lse = lse;
  pre.delta = w.delta;
  pre.nlse2 = w.nlse2;
  // The tensor-core backward accumulates dq~ with reductions: zero it here.
  pre.dq_zero = s.bf16 ? w.dq_acc : nullptr;

  EpiParams ep;
  ep.B = s.B;
  ep.T = s.T;
  ep.H = s.H;
  ep.Hk = s.Hk;
  ep.has_ve = layer->has_ve;
  fill_omega(ep.omega, s.D, layer->rope_base);
  ep.q = q;
  ep.k = k;
  ep.ve = ve;
  ep.gate = gate;
  ep.rstd_q = rstd_q;
  ep.rstd_k = rstd_k;
  ep.dq_acc = w.dq_acc;
  ep.dk_acc = w.dk_acc;
  ep.dv_acc = w.dv_acc;
  ep.parts = parts;
  ep.kv_stride = static_cast<long long>(s.B) * s.T * s.Hk * s.D;
  ep.dq = dQ;
  ep.dk = dK;
  ep.dv = dV;
  ep.dve = dve;
  ep.dgate = dgate;

  // Everything that can fail short of a launch (tensor maps, shared-memory
  // limits) is done before the first kernel is enqueued, so that a rejected
  // call leaves the stream untouched.
  CUtensorMap mq, mdo, mk, mv, mdk, mdv, mdq;
  bwd::Params bp{};
  if (s.bf16) {
    if ((st = make_map(&mq, q_out, s.B, s.T, s.H, bwd::kBQ, s.D)) != CSWATTN_OK) return st;
    if ((st = make_map(&mdo, dO, s.B, s.T, s.H, bwd::kBQ, s.D)) != CSWATTN_OK) return st;
    if ((st = make_map(&mk, k_out, s.B, s.T, s.Hk, bwd::kBN, s.D)) != CSWATTN_OK) return st;
    if ((st = make_map(&mv, v_out, s.B, s.T, s.Hk, bwd::kBN, s.D)) != CSWATTN_OK) return st;
    if ((st = make_map(&mdk, w.dk_acc, s.B * parts, s.T, s.Hk, bwd::kBN, s.D, true)) != CSWATTN_OK) return st;
    if ((st = make_map(&mdv, w.dv_acc, s.B * parts, s.T, s.Hk, bwd::kBN, s.D, true)) != CSWATTN_OK) return st;
    if ((st = make_map(&mdq, w.dq_acc, s.B, s.T, s.H, bwd::kBQ / 2, s.D, true)) != CSWATTN_OK) return st;
    if ((st = s.D == 64 ? set_smem(bwd::bwd_kernel<64>, bwd::kSmemBytes)
                        : set_smem(bwd::bwd_kernel<128>, bwd::kSmemBytes)) != CSWATTN_OK)
      return st;
    bp.B = s.B;
    bp.T = s.T;
    bp.H = s.H;
    bp.Hk = s.Hk;
    bp.W = s.W;
    bp.g = s.g;
    bp.nkv = (s.T + bwd::kBN - 1) / bwd::kBN;
    bp.scale_log2 = s.scale * 1.4426950408889634f;
    bp.scale = s.scale;
    bp.Tpad = w.Tpad;
    bp.nlse2 = w.nlse2;
    bp.delta = w.delta;
    bp.dq_acc = w.dq_acc;
    bp.dk_acc = w.dk_acc;
    bp.dv_acc = w.dv_acc;
    bp.parts = parts;
    bp.kv_stride = static_cast<long long>(s.B) * s.T * s.Hk * s.D;
    bp.wait_ns = g_wait_ns.load();
  }
  st = s.bf16 ? launch_preprocess<__nv_bfloat16>(s, pre, cs, true) : launch_preprocess<float>(s, pre, cs, true);
  if (st != CSWATTN_OK) return st;
  st = s.bf16 ? launch_epilogue<__nv_bfloat16>(s, ep, cs, true) : launch_epilogue<float>(s, ep, cs, true);
  if (st != CSWATTN_OK) return st;

  {
    ScopedTiming tm(CSWATTN_K_BWD_PRE, cs);
    st = s.bf16 ? launch_preprocess<__nv_bfloat16>(s, pre, cs, false) : launch_preprocess<float>(s, pre, cs, false);
  }
  if (st != CSWATTN_OK) return st;
  if ((st = launched("preprocess launch")) != CSWATTN_OK) return st;

  if (!s.bf16) {
    SimtParams sp{};
    sp.B = s.B;
    sp.T = s.T;
    sp.H = s.H;
    sp.Hk = s.Hk;
    sp.W = s.W;
    sp.scale = s.scale;
    sp.q = static_cast<const float*>(q_out);
    sp.k = static_cast<const float*>(k_out);
    sp.v = static_cast<const float*>(v_out);
    sp.O = static_cast<const float*>(O);
    sp.dO = static_cast<const float*>(dO);
    sp.lse = lse;
    sp.delta = w.delta;
    sp.Tpad = w.Tpad;
    sp.dq_acc = w.dq_acc;
    sp.dk_acc = w.dk_acc;
    sp.dv_acc = w.dv_acc;
    {
      ScopedTiming tm(CSWATTN_K_BWD, cs);
      launch_simt_bwd(s, sp, cs);
    }
    if ((st = launched("fp32 backward launch")) != CSWATTN_OK) return st;
  } else {
    const unsigned grid = static_cast<unsigned>(bp.nkv) * bp.parts * s.B * s.Hk;
    {
      ScopedTiming tm(CSWATTN_K_BWD, cs);
      if (s.D == 64)
        launch_pdl(bwd::bwd_kernel<64>, dim3(grid), dim3(bwd::kThreads), bwd::kSmemBytes, cs, mq, mdo, mk, mv,
                   mdk, mdv, mdq, bp);
      else
        launch_pdl(bwd::bwd_kernel<128>, dim3(grid), dim3(bwd::kThreads), bwd::kSmemBytes, cs, mq, mdo, mk, mv,
                   mdk, mdv, mdq, bp);
    }
    if ((st = launched("backward launch")) != CSWATTN_OK) return st;
  }

  {
    ScopedTiming tm(CSWATTN_K_BWD_EPI, cs);
    st = s.bf16 ? launch_epilogue<__nv_bfloat16>(s, ep, cs, false) : launch_epilogue<float>(s, ep, cs, false);
  }
  if (st != CSWATTN_OK) return st;
  return launched("epilogue launch");
}

size_t attn_decode_workspace_bytes(const cswattn_layer* layer) {
  Shape s;
  if (check_decode_layer(layer, &s) != CSWATTN_OK) return 0;
  return carve_decode(s, nullptr).bytes;
}

cswattn_status attn_decode(const cswattn_layer* layer, const void* q, const void* k, const void* v,
                           const void* ve, const void* gate, const int* cache_len, void* k_cache,
                           void* v_cache, void* O, float* lse, void* workspace, size_t workspace_bytes,
                           void* stream) {
  const NvtxRange nvtx_range("attn_decode");
  Shape s;
  cswattn_status st = check_decode_layer(layer, &s);
  if (st != CSWATTN_OK) return st;
  CHECK_PTR(q, 16);
  CHECK_PTR(k, 16);
  CHECK_PTR(v, 16);
  CHECK_PTR(cache_len, 4);
  CHECK_PTR(k_cache, 16);
  CHECK_PTR(v_cache, 16);
  CHECK_PTR(O, 16);
  CHECK_PTR(lse, 4);
  CHECK_PTR(workspace, 256);
  if (layer->has_ve) {
    CHECK_PTR(ve, 16);
    CHECK_PTR(gate, 2);
  }
  if (k_cache == v_cache) return fail(CSWATTN_ERR_INVALID_ARG, "k_cache and v_cache must differ");
  const DecodeWorkspace w = carve_decode(s, workspace);
  if (workspace_bytes < w.bytes)
    return fail(CSWATTN_ERR_INVALID_ARG, "decode workspace too small: %zu < %zu bytes", workspace_bytes, w.bytes);
  CUtensorMap mk, mv;
  if ((st = make_map(&mk, k_cache, s.B, s.T, s.Hk, dec::kKeys, s.D)) != CSWATTN_OK) return st;
  if ((st = make_map(&mv, v_cache, s.B, s.T, s.Hk, dec::kKeys, s.D)) != CSWATTN_OK) return st;
  dec::AttnParams ap;
  ap.B = s.B;
  ap.T = s.T;
  ap.H = s.H;
  ap.Hk = s.Hk;
  ap.W = s.W;
  ap.g = s.g;
  ap.nsplit = w.nsplit;
  ap.nmax = dec::decode_nmax(w.nsplit, s.T, s.W);
  ap.tmem_cols = dec::decode_tmem_cols(ap.nmax);
  ap.scale_log2 = s.scale * 1.4426950408889634f;
  ap.has_ve = layer->has_ve;
  ap.eps = layer->eps;
  fill_omega(ap.omega, s.D, layer->rope_base);
  ap.len = cache_len;
  ap.q = static_cast<const __nv_bfloat16*>(q);
  ap.k = static_cast<const __nv_bfloat16*>(k);
  ap.v = static_cast<const __nv_bfloat16*>(v);
  ap.ve = static_cast<const __nv_bfloat16*>(ve);
  ap.gate = static_cast<const __nv_bfloat16*>(gate);
  ap.kc = static_cast<__nv_bfloat16*>(k_cache);
  ap.vc = static_cast<__nv_bfloat16*>(v_cache);
  ap.part_ml = w.part_ml;
  ap.part_o = w.part_o;
  ap.O = static_cast<__nv_bfloat16*>(O);
  ap.lse = lse;
  ap.wait_ns = g_wait_ns.load();
  dec::CombineParams cp;
  cp.B = s.B;
  cp.H = s.H;
  cp.nsplit = w.nsplit;
  cp.len = cache_len;
  cp.T = s.T;
  cp.part_ml = w.part_ml;
  cp.part_o = w.part_o;
  cp.O = static_cast<__nv_bfloat16*>(O);
  cp.lse = lse;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  {
    ScopedTiming tm(CSWATTN_K_DECODE, cs);
    st = s.D == 64 ? launch_decode<64>(s, mk, mv, ap, cp, cs) : launch_decode<128>(s, mk, mv, ap, cp, cs);
  }
  if (st != CSWATTN_OK) return st;
  return launched("decode launch");
}

cswattn_status cswattn_gemm_bf16(int M, int N, int K, int a_mn, const void* A, long long lda, int b_mn,
                                 const void* B, long long ldb, float alpha, float beta, const void* D,
                                 long long ldd, void* C, long long ldc, void* stream) {
  const NvtxRange nvtx_range("cswattn_gemm_bf16");
  const GemmArgs g{M, N, K, a_mn != 0, b_mn != 0, A, B, D, lda, ldb, ldd, ldc, alpha, beta, C};
  return run_gemm(g, static_cast<cudaStream_t>(stream));
}

size_t muon_ns_workspace_bytes(int m, int n) {
  if (m < 1 || n < 1) return 0;
  return carve_ns(m, n, nullptr).bytes;
}

cswattn_status muon_newton_schulz(int m, int n, const float* coeffs, int steps, const void* X, void* Y,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx_range("muon_newton_schulz");
  if (m < 1 || n < 1) return fail(CSWATTN_ERR_INVALID_ARG, "m, n must be >= 1");
  if (n % 8 != 0) return fail(CSWATTN_ERR_UNSUPPORTED, "n must be a multiple of 8 (got %d)", n);
  if (steps < 1 || steps > 64) return fail(CSWATTN_ERR_INVALID_ARG, "steps must be in [1, 64]");
  if (!coeffs) return fail(CSWATTN_ERR_INVALID_ARG, "coeffs is NULL");
  for (int i = 0; i < 3 * steps; ++i)
    if (!std::isfinite(coeffs[i])) return fail(CSWATTN_ERR_INVALID_ARG, "coefficients must be finite");
  CHECK_PTR(X, 16);
  CHECK_PTR(Y, 16);
  CHECK_PTR(workspace, 256);
  if (X == Y) return fail(CSWATTN_ERR_INVALID_ARG, "X and Y must be different buffers");
  const NsWorkspace w = carve_ns(m, n, workspace);
  if (workspace_bytes < w.bytes)
    return fail(CSWATTN_ERR_INVALID_ARG, "workspace has %zu bytes, needs %zu", workspace_bytes, w.bytes);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const void* cur = X;
  for (int st_i = 0; st_i < steps; ++st_i) {
    const float a = coeffs[3 * st_i], b = coeffs[3 * st_i + 1], c = coeffs[3 * st_i + 2];
    void* out = ((steps - 1 - st_i) % 2 == 0) ? Y : w.X;  // the last step writes Y
    // A = X^T X (n x n): both operands are X read MN-major, K = m.
    GemmArgs g1{n, n, m, true, true, cur, cur, nullptr, n, n, 0, n, 1.f, 0.f, w.A};
    // B = c A A + b A: A K-major, A again as the MN-major (K x N) operand.
    GemmArgs g2{n, n, n, false, true, w.A, w.A, w.A, n, n, n, n, c, b, w.B};
    // X' = X B + a X: X K-major (m x n), B MN-major.
    GemmArgs g3{m, n, n, false, true, cur, w.B, cur, n, n, n, n, 1.f, a, out};
    cswattn_status e;
    if ((e = run_gemm(g1, cs)) != CSWATTN_OK) return e;
    if ((e = run_gemm(g2, cs)) != CSWATTN_OK) return e;
    if ((e = run_gemm(g3, cs)) != CSWATTN_OK) return e;
    cur = out;
  }
  return CSWATTN_OK;
}

}  // extern "C"

namespace {

// Workspace of the FP8 projection: the two operands' amax bit patterns, then
// the E4M3 codes of x (B*T x C) and of W ((H + 2 Hk) D x C).
struct Fp8Workspace {
  unsigned int* amax;
  uint8_t *x8, *w8;
  size_t bytes;
};

Fp8Workspace carve_fp8(const Shape& s, int C, void* base) {
  uint8_t* p = static_cast<uint8_t*>(base);
  Fp8Workspace w;
  size_t off = 0;
  w.amax = reinterpret_cast<unsigned int*>(p + off);
  off += 256;
  w.x8 = p + off;
  off += pad256(static_cast<size_t>(s.B) * s.T * C);
  w.w8 = p + off;
  off += pad256(static_cast<size_t>(s.H + 2 * s.Hk) * s.D * C);
  w.bytes = off;
  return w;
}

// The fused projection; with `f8` (workspace and scales) the operands are
// first quantized to E4M3 with tensor-wise scales.
cswattn_status qkv_impl(const cswattn_layer* layer, const void* x, long long x_stride, int C, const void* w_qkv,
                        const void* ve, const void* gate, void* q, void* k, void* q_out, void* k_out, void* v_out,
                        float* rstd_q, float* rstd_k, float* scales, void* workspace, size_t workspace_bytes,
                        bool f8, void* stream) {
  Shape s;
  cswattn_status st = check_layer(layer, &s);
  if (st != CSWATTN_OK) return st;
  if (!s.bf16) return fail(CSWATTN_ERR_UNSUPPORTED, "the QKV projection supports bf16 layers only");
  if (C < 1 || C % 8 != 0 || x_stride < C || x_stride % 8 != 0)
    return fail(CSWATTN_ERR_INVALID_ARG, "C must be a positive multiple of 8 and x_stride >= C a multiple of 8");
  if (f8 && C % 16 != 0) return fail(CSWATTN_ERR_INVALID_ARG, "the FP8 projection needs C a multiple of 16");
  const long long BT = static_cast<long long>(s.B) * s.T;
  if (BT > 65535ll * qkv::kBM) return fail(CSWATTN_ERR_UNSUPPORTED, "too many tokens (%lld)", BT);
  CHECK_PTR(x, 16);
  CHECK_PTR(w_qkv, 16);
  CHECK_PTR(q, 16);
  CHECK_PTR(k, 16);
  CHECK_PTR(q_out, 16);
  CHECK_PTR(k_out, 16);
  CHECK_PTR(v_out, 16);
  CHECK_PTR(rstd_q, 4);
  CHECK_PTR(rstd_k, 4);
  if (layer->has_ve) {
    CHECK_PTR(ve, 16);
    CHECK_PTR(gate, 2);
  }
  Fp8Workspace fw{};
  if (f8) {
    CHECK_PTR(scales, 4);
    CHECK_PTR(workspace, 256);
    fw = carve_fp8(s, C, workspace);
    if (workspace_bytes < fw.bytes)
      return fail(CSWATTN_ERR_INVALID_ARG, "workspace has %zu bytes, needs %zu", workspace_bytes, fw.bytes);
  }
  const int nh = s.H + 2 * s.Hk;
  CUtensorMap mx, mw, mq, mk, mqo, mko, mvo;
  if (f8) {
    if ((st = make_map_2d(&mx, fw.x8, C, BT, C, 128, qkv::kBM, true)) != CSWATTN_OK) return st;
    if ((st = make_map_2d(&mw, fw.w8, C, static_cast<long long>(nh) * s.D, C, 128, qkv::kNH * s.D, true)) !=
        CSWATTN_OK)
      return st;
  } else {
    if ((st = make_map_2d(&mx, x, C, BT, x_stride, 64, qkv::kBM)) != CSWATTN_OK) return st;
    if ((st = make_map_2d(&mw, w_qkv, C, static_cast<long long>(nh) * s.D, C, 64, qkv::kNH * s.D)) != CSWATTN_OK)
      return st;
  }
  if ((st = make_map_3d(&mq, q, BT, s.H, s.D, qkv::kBM)) != CSWATTN_OK) return st;
  if ((st = make_map_3d(&mk, k, BT, s.Hk, s.D, qkv::kBM)) != CSWATTN_OK) return st;
  if ((st = make_map_3d(&mqo, q_out, BT, s.H, s.D, qkv::kBM)) != CSWATTN_OK) return st;
  if ((st = make_map_3d(&mko, k_out, BT, s.Hk, s.D, qkv::kBM)) != CSWATTN_OK) return st;
  if ((st = make_map_3d(&mvo, v_out, BT, s.Hk, s.D, qkv::kBM)) != CSWATTN_OK) return st;
  auto kern = s.D == 64 ? (f8 ? qkv::qkv_kernel<64, true> : qkv::qkv_kernel<64, false>)
                        : (f8 ? qkv::qkv_kernel<128, true> : qkv::qkv_kernel<128, false>);
  if ((st = set_smem(kern, qkv::kSmemBytes)) != CSWATTN_OK) return st;
  qkv::Params qp;
  qp.BT = static_cast<int>(BT);
  qp.T = s.T;
  qp.H = s.H;
  qp.Hk = s.Hk;
  qp.C = C;
  qp.has_ve = layer->has_ve;
  qp.eps = layer->eps;
  fill_omega(qp.omega, s.D, layer->rope_base);
  qp.ve = static_cast<const __nv_bfloat16*>(ve);
  qp.gate = static_cast<const __nv_bfloat16*>(gate);
  qp.rstd_q = rstd_q;
  qp.rstd_k = rstd_k;
  qp.scales = f8 ? scales : nullptr;
  qp.wait_ns = g_wait_ns.load();
  const dim3 grid(static_cast<unsigned>((nh + qkv::kNH - 1) / qkv::kNH),
                  static_cast<unsigned>((BT + qkv::kBM - 1) / qkv::kBM));
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  {
    ScopedTiming tm(CSWATTN_K_PROLOGUE, cs);
    if (f8) {
      // Tensor-wise scales, then the E4M3 codes of both operands.
      Fp8QuantParams fq;
      fq.a = static_cast<const __nv_bfloat16*>(x);
      fq.rows_a = BT;
      fq.lda = x_stride;
      fq.b = static_cast<const __nv_bfloat16*>(w_qkv);
      fq.rows_b = static_cast<long long>(nh) * s.D;
      fq.cols = C;
      fq.amax_bits = fw.amax;
      fq.a8 = fw.x8;
      fq.b8 = fw.w8;
      fq.scales = scales;
      const cudaError_t e = cudaMemsetAsync(fw.amax, 0, 2 * sizeof(unsigned int), cs);
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
      const long long n8 = (BT + fq.rows_b) * (C / 8);  // 8-element vectors
      const unsigned g = static_cast<unsigned>(std::min<long long>((n8 + kFp8Threads - 1) / kFp8Threads, 148 * 8));
      fp8_amax_kernel<<<g, kFp8Threads, 0, cs>>>(fq);  // ordinary launch: strictly after the memset
      launch_pdl(fp8_quant_kernel, dim3(g), dim3(kFp8Threads), 0, cs, fq);
    }
    launch_pdl(kern, grid, dim3(qkv::kThreads), qkv::kSmemBytes, cs, mx, mw, mq, mk, mqo, mko, mvo, qp);
  }
  return launched("QKV projection launch");
}

}  // namespace

extern "C" {

cswattn_status attn_qkv_prologue(const cswattn_layer* layer, const void* x, long long x_stride, int C,
                                 const void* w_qkv, const void* ve, const void* gate, void* q, void* k,
                                 void* q_out, void* k_out, void* v_out, float* rstd_q, float* rstd_k,
                                 void* stream) {
  const NvtxRange nvtx_range("attn_qkv_prologue");
  return qkv_impl(layer, x, x_stride, C, w_qkv, ve, gate, q, k, q_out, k_out, v_out, rstd_q, rstd_k, nullptr,
                  nullptr, 0, false, stream);
}

size_t attn_qkv_fp8_workspace_bytes(const cswattn_layer* layer, int C) {
  Shape s;
  if (check_layer(layer, &s) != CSWATTN_OK || C < 1) return 0;
  return carve_fp8(s, C, nullptr).bytes;
}

cswattn_status attn_qkv_prologue_fp8(const cswattn_layer* layer, const void* x, long long x_stride, int C,
                                     const void* w_qkv, const void* ve, const void* gate, void* q, void* k,
                                     void* q_out, void* k_out, void* v_out, float* rstd_q, float* rstd_k,
                                     float* scales, void* workspace, size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx_range("attn_qkv_prologue_fp8");
  return qkv_impl(layer, x, x_stride, C, w_qkv, ve, gate, q, k, q_out, k_out, v_out, rstd_q, rstd_k, scales,
                  workspace, workspace_bytes, true, stream);
}

cswattn_status attn_qkv_bwd(const cswattn_layer* layer, const void* x, long long x_stride, int C,
                            const void* w_qkv, const void* dQ, const void* dK, const void* dV, void* dx,
                            float* dw_qkv, void* stream) {
  const NvtxRange nvtx_range("attn_qkv_bwd");
  Shape s;
  cswattn_status st = check_layer(layer, &s);
  if (st != CSWATTN_OK) return st;
  if (!s.bf16) return fail(CSWATTN_ERR_UNSUPPORTED, "attn_qkv_bwd supports bf16 layers only");
  if (C < 1 || C % 8 != 0 || x_stride < C || x_stride % 8 != 0)
    return fail(CSWATTN_ERR_INVALID_ARG, "C must be a positive multiple of 8 and x_stride >= C a multiple of 8");
  const long long BT = static_cast<long long>(s.B) * s.T;
  if (BT > (1ll << 30)) return fail(CSWATTN_ERR_UNSUPPORTED, "too many tokens");
  CHECK_PTR(dx, 16);
  CHECK_PTR(dw_qkv, 16);
  const int M = static_cast<int>(BT);
  const long long hq = static_cast<long long>(s.H) * s.D, hk = static_cast<long long>(s.Hk) * s.D;
  const __nv_bfloat16* w = static_cast<const __nv_bfloat16*>(w_qkv);
  const int nr = static_cast<int>(hq + 2 * hk);  // rows of the stacked weight
  CHECK_PTR(dQ, 16);
  CHECK_PTR(dK, 16);
  CHECK_PTR(dV, 16);
  CHECK_PTR(x, 16);
  CHECK_PTR(w_qkv, 16);
  // dx = dQ W_q + dK W_k + dV W_v: one product whose K is the three segments
  // (W_* rows of the stacked weight, MN-major), so dx is rounded once.
  const GemmArgs gx{M, C, nr, false, true, dQ, w, nullptr, hq, C, 0, C, 1.f, 0.f, dx};
  GemmSegs sx;
  sx.n = 3;
  sx.along_m = false;
  const void* dys[3] = {dQ, dK, dV};
  const long long lds[3] = {hq, hk, hk};
  for (int i = 0; i < 3; ++i) {
    sx.A[i] = dys[i];
    sx.B[i] = w + (i == 0 ? 0 : (i == 1 ? hq : hq + hk)) * C;
    sx.lda[i] = lds[i];
    sx.ldb[i] = C;
    sx.ext[i] = static_cast<int>(lds[i]);
  }
  // dW = [dQ dK dV]^T x (float32 rows of the stacked gradient): one product
  // with M made of the three segments when the query and key blocks span
  // whole 128-row tiles, else three products.
  const GemmArgs gw{nr, C, M, true, true, dQ, x, nullptr, hq, x_stride, 0, C, 1.f, 0.f, dw_qkv, true};
  GemmSegs sw;
  sw.n = 3;
  sw.along_m = true;
  for (int i = 0; i < 3; ++i) {
    sw.A[i] = dys[i];
    sw.lda[i] = lds[i];
    sw.ext[i] = static_cast<int>(lds[i]);
  }
  sw.B[0] = x;
  sw.ldb[0] = x_stride;
  const bool w_one = hq % gemm::kBM == 0 && hk % gemm::kBM == 0;
  const GemmArgs gws[3] = {
      {static_cast<int>(hq), C, M, true, true, dQ, x, nullptr, hq, x_stride, 0, C, 1.f, 0.f, dw_qkv, true},
      {static_cast<int>(hk), C, M, true, true, dK, x, nullptr, hk, x_stride, 0, C, 1.f, 0.f, dw_qkv + hq * C, true},
      {static_cast<int>(hk), C, M, true, true, dV, x, nullptr, hk, x_stride, 0, C, 1.f, 0.f, dw_qkv + (hq + hk) * C,
       true},
  };
  if ((st = check_gemm(gx, false)) != CSWATTN_OK) return st;
  if (w_one) {
    if ((st = check_gemm(gw, false)) != CSWATTN_OK) return st;
  } else {
    for (const auto& a : gws)
      if ((st = check_gemm(a)) != CSWATTN_OK) return st;
  }
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if ((st = run_gemm(gx, cs, &sx)) != CSWATTN_OK) return st;
  if (w_one) return run_gemm(gw, cs, &sw);
  for (const auto& a : gws)
    if ((st = run_gemm(a, cs)) != CSWATTN_OK) return st;
  return CSWATTN_OK;
}

cswattn_status attn_bwd_noalloc(const cswattn_layer* layer, const void* q, const void* k,
                                const void* ve, const void* gate, const void* q_out,
                                const void* k_out, const void* v_out, const float* rstd_q,
                                const float* rstd_k, const void* O, const float* lse,
                                const void* dO, void* dQ, void* dK, void* dV, void* dve,
                                void* dgate, void* stream) {
  const NvtxRange nvtx_range("attn_bwd_noalloc");
  Shape s;
  cswattn_status st = check_layer(layer, &s);
  if (st != CSWATTN_OK) return st;
  const size_t need = carve(s, nullptr).bytes;
  if (need > CSWATTN_NOALLOC_SCRATCH_BYTES)
    return fail(CSWATTN_ERR_UNSUPPORTED,
                "attn_bwd_noalloc: this layer needs %zu bytes of scratch, the fixed array holds %u; "
                "use attn_bwd with a caller workspace",
                need, static_cast<unsigned>(CSWATTN_NOALLOC_SCRATCH_BYTES));
  void* ws = nullptr;
  if ((st = noalloc_scratch(&ws)) != CSWATTN_OK) return st;
  return attn_bwd(layer, q, k, ve, gate, q_out, k_out, v_out, rstd_q, rstd_k, O, lse, dO, dQ, dK,
                  dV, dve, dgate, ws, CSWATTN_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
