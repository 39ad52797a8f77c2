/*
 * cswattn.h -- C ABI of the causal sliding-window RoPE attention library
 * (libcswattn.so), built for NVIDIA B200 (sm_100a).
 *
 * The library computes one attention layer of a nanochat-style GPT block,
 * forward and backward, as described on the page
 * "5만원으로 나만의 ChatGPT 훈련하는 방법" (apidog.com):
 *   - section "1. GPT 모델 (nanochat/gpt.py)", architecture list: rotary
 *     position embeddings (RoPE), QK normalisation, grouped-query attention
 *     (fewer KV heads than query heads) and sliding-window attention with a
 *     per-layer pattern such as "SSSL";
 *   - same section, "값 임베딩 (Value Embeddings, ResFormer)": the value
 *     embedding is viewed per KV head and mixed in as v + 3*sigmoid(gate)*ve;
 *   - section "5. 플래시 어텐션 통합 (nanochat/flash_attention.py)": the
 *     attention is a causal call with a window size on (B, T, H, D) tensors.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout: all tensors are dense row-major, head_dim contiguous:
 *   q, q_out, O, dO, dQ          (B, T, n_head, head_dim)
 *   k, v, ve, k_out, v_out,
 *   dK, dV, dve                  (B, T, n_kv_head, head_dim)
 *   gate, dgate                  (B, T, n_kv_head)
 *   rstd_q                       (B, T, n_head)       float32
 *   rstd_k                       (B, T, n_kv_head)    float32
 *   lse                          (B, n_head, T)       float32, natural log
 * Element type: layer->dtype for every tensor except rstd and lse (float32).
 * Query head h reads KV head h / (n_head / n_kv_head).
 * Window: a query at position i sees keys j with i - window < j <= i, itself
 * included; window >= T is plain causal attention, window = 1 sees itself.
 * RoPE: pairs (i, i + head_dim/2) rotated by angle t * rope_base^(-2i/head_dim),
 * positions t = 0 .. T-1. RMSNorm: x * (mean(x^2) + eps)^(-1/2), no weight.
 *
 * Ownership: every pointer is caller-owned device memory (except where a
 * function says host). The library allocates no device memory; the backward's
 * scratch is the caller's `workspace`. Pointers to element tensors must be
 * 16-byte aligned; rstd/lse/gate pointers 4-byte (2-byte for bf16 gate).
 * Streams: every call is asynchronous on `stream` (a cudaStream_t; NULL is
 * the legacy default stream) and returns once the work is enqueued. The bf16
 * kernels are launched with programmatic stream serialization: a kernel may
 * be scheduled while the previous kernel on the stream is finishing, but it
 * touches no global memory until that kernel has completed, so stream order
 * holds as for ordinary launches.
 * Errors: arguments are validated on the host before anything is enqueued;
 * a rejected call returns CSWATTN_ERR_INVALID_ARG or CSWATTN_ERR_UNSUPPORTED
 * and enqueues nothing. A failed launch returns CSWATTN_ERR_CUDA. Device-side
 * waits are bounded: a kernel whose wait runs out records CSWATTN_ERR_TIMEOUT
 * in a device status word and returns; cswattn_sync_status() reports it.
 * cswattn_last_error() gives a message for the last failure on this thread.
 */
#ifndef CSWATTN_H
#define CSWATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CSWATTN_OK = 0,
  CSWATTN_ERR_INVALID_ARG = 1,
  CSWATTN_ERR_UNSUPPORTED = 2,
  CSWATTN_ERR_CUDA = 3,
  CSWATTN_ERR_TIMEOUT = 4,
  CSWATTN_ERR_BOUNDS = 5 /* a device-side bounds check failed (CSWATTN_CHECK=1 build only) */
} cswattn_status;

typedef enum { CSWATTN_F32 = 0, CSWATTN_BF16 = 1 } cswattn_dtype;

/* Shape of one attention layer. Supported: bf16 with head_dim 64 or 128
 * (tensor cores; a 64-wide head runs the 128-wide tiles with its second half
 * zero), f32 with head_dim in {4, 8, 16, 32, 64, 128} (CUDA cores, fp32
 * throughout). Anything else returns CSWATTN_ERR_UNSUPPORTED.
 * n_head % n_kv_head == 0, window >= 1, T <= 2^20. */
typedef struct {
  int B, T, n_head, n_kv_head, head_dim;
  int window;          /* keys visible to a query, itself included */
  float rope_base;     /* > 0; 10000 in the d12/d24 workloads */
  float eps;           /* >= 0; RMSNorm epsilon inside the square root */
  float softmax_scale; /* > 0, or 0 for 1/sqrt(head_dim) */
  int has_ve;          /* 1: the value embedding and its gate are present */
  cswattn_dtype dtype;
} cswattn_layer;

/* Prologue: q_out = RoPE(RMSNorm(q)), k_out = RoPE(RMSNorm(k)),
 * v_out = v + 3*sigmoid(gate)*ve (v_out = v when has_ve == 0), and the
 * RMSNorm factors rstd_q = (mean(q^2)+eps)^(-1/2), rstd_k likewise.
 * Page sections "1. GPT 모델" (architecture list; value-embedding code).
 * ve and gate are read only when has_ve and may be NULL otherwise.
 * Outputs must not alias inputs. */
cswattn_status attn_prologue(const cswattn_layer* layer, const void* q, const void* k,
                             const void* v, const void* ve, const void* gate,
                             void* q_out, void* k_out, void* v_out, float* rstd_q,
                             float* rstd_k, void* stream);

/* Prologue with the value-embedding gate computed from the block input
 * instead of given as logits: page section "1. GPT 모델", value-embedding
 * code, where the gate is 3*sigmoid(ve_gate(x[..., :C])) and ve_gate is a
 * linear map from the first C channels of the block input x to one logit
 * per KV head (no bias: the page shows none).
 *   gate_out[b,t,h] = sum_{c<C} x[b,t,c] * w_gate[h,c], rounded to the layer
 *   dtype; v_out = v + 3*sigmoid(gate_out)*ve; q_out, k_out, rstd_q, rstd_k
 *   as for attn_prologue.
 * x: (B, T, x_stride) in the layer dtype, only the first gate_channels
 * entries of each token's row are read (1 <= gate_channels <= x_stride);
 * w_gate: (n_kv_head, gate_channels); gate_out: (B, T, n_kv_head), the
 * logits, to be passed as `gate` to attn_bwd. Requires has_ve = 1 (else
 * CSWATTN_ERR_INVALID_ARG). Pointers aligned to the element size. */
cswattn_status attn_prologue_gated(const cswattn_layer* layer, const void* q, const void* k,
                                   const void* v, const void* ve, const void* x, long long x_stride,
                                   int gate_channels, const void* w_gate, void* gate_out, void* q_out,
                                   void* k_out, void* v_out, float* rstd_q, float* rstd_k,
                                   void* stream);

/* Backward of the gate's projection (same page section), given dgate, the
 * gradient of the loss with respect to the gate logits (attn_bwd's dgate):
 *   dx[b,t,c]      = sum_h dgate[b,t,h] * w_gate[h,c]    (B, T, gate_channels)
 *   dw_gate[h,c]   = sum_{b,t} dgate[b,t,h] * x[b,t,c]   (n_kv_head, gate_channels)
 * dx is the contribution to the gradient of x[..., :gate_channels] (the
 * caller adds it to its own); dx in the layer dtype, dw_gate float32 and
 * deterministic (a fixed summation order). x, x_stride, gate_channels,
 * w_gate as for attn_prologue_gated. Requires has_ve = 1. */
cswattn_status attn_gate_bwd(const cswattn_layer* layer, const void* x, long long x_stride,
                             int gate_channels, const void* w_gate, const void* dgate, void* dx,
                             float* dw_gate, void* stream);

/* The QKV projection fused with the prologue: page section "1. GPT 모델
 * (nanochat/gpt.py)", where the block input is projected to the query, key
 * and value heads by bias-free Linear layers before RoPE, QK normalisation
 * and the value residual. With the stacked weight w_qkv ((n_head +
 * 2 n_kv_head) * head_dim rows, C columns; rows: the query heads, then the
 * key heads, then the value heads, each head_dim rows):
 *   y = x[..., :C] w_qkv^T, rounded to bf16, split into q (B, T, n_head, D),
 *   k and v (B, T, n_kv_head, D);
 *   q, k: written raw (attn_bwd needs them); q_out, k_out, rstd_q, rstd_k,
 *   v_out as attn_prologue computes them from (q, k, v, ve, gate).
 * x: (B, T, x_stride) bf16, columns [0, C) read; C and x_stride multiples
 * of 8. bf16 layers only; ve and gate only when has_ve. One kernel: the
 * product on the tensor cores with RMSNorm, RoPE and the value residual in
 * its epilogue. */
cswattn_status attn_qkv_prologue(const cswattn_layer* layer, const void* x, long long x_stride, int C,
                                 const void* w_qkv, const void* ve, const void* gate, void* q, void* k,
                                 void* q_out, void* k_out, void* v_out, float* rstd_q, float* rstd_k,
                                 void* stream);

/* Bytes of device scratch attn_qkv_prologue_fp8 needs for this layer and C:
 * 256 bytes of amax state, then the E4M3 codes of x (B*T*C bytes, padded to
 * 256) and of w_qkv ((n_head + 2 n_kv_head) * head_dim * C bytes, padded).
 * 0 for an invalid layer or C < 1. */
size_t attn_qkv_fp8_workspace_bytes(const cswattn_layer* layer, int C);

/* The FP8 variant of attn_qkv_prologue: page section "3. 정밀도 관리
 * (nanochat/common.py)", where --fp8 turns the Linear layers into
 * Float8Linear with tensor-wise scaling. Each operand t of the projection
 * (x[..., :C] and w_qkv) gets one scale s_t = amax|t| / 448 (1 for an
 * all-zero tensor) and is replaced by s_t * E4M3(t / s_t) (round to nearest
 * even, saturated to +-448, the division in float32); the product runs on
 * the tensor cores in E4M3 with float32 accumulation and is multiplied by
 * s_x s_w, then rounded to bf16 and handed to the same prologue epilogue.
 * scales: 2 floats, device, written (s_x, s_w). workspace: device, 256-byte
 * aligned, at least attn_qkv_fp8_workspace_bytes; the codes are left in it
 * (x's at byte 256, w's after them). C a multiple of 16; otherwise as
 * attn_qkv_prologue. Three launches: the amax reduction, the quantization,
 * the fused projection. The backward is attn_qkv_bwd on the bf16 x and
 * w_qkv (the quantization passes gradients straight through). */
cswattn_status attn_qkv_prologue_fp8(const cswattn_layer* layer, const void* x, long long x_stride, int C,
                                     const void* w_qkv, const void* ve, const void* gate, void* q, void* k,
                                     void* q_out, void* k_out, void* v_out, float* rstd_q, float* rstd_k,
                                     float* scales, void* workspace, size_t workspace_bytes, void* stream);

/* Backward of the projection (same page section), given attn_bwd's dQ, dK,
 * dV (gradients of the raw q, k, v):
 *   dx     = dQ w_q + dK w_k + dV w_v         (B, T, C), bf16, row stride C
 *   dw_qkv = [dQ dK dV]^T x[..., :C]           ((n_head + 2 n_kv_head) D, C), float32
 * Two tensor-core matrix products (the kernel of cswattn_gemm_bf16 with
 * operands in three segments): dx in one accumulator over the three weight
 * blocks (rounded to bf16 once), dw_qkv over the three gradient blocks (three
 * products when n_head * D or n_kv_head * D is not a multiple of 128). x,
 * x_stride, C, w_qkv as for attn_qkv_prologue; all pointers 16-byte aligned;
 * bf16 layers only. */
cswattn_status attn_qkv_bwd(const cswattn_layer* layer, const void* x, long long x_stride, int C,
                            const void* w_qkv, const void* dQ, const void* dK, const void* dV, void* dx,
                            float* dw_qkv, void* stream);

/* Forward: O_i = sum_j softmax_j(scale * q_out_i . k_out_j) v_out_j over the
 * causal window, and lse_i = log sum_j exp(scale * q_out_i . k_out_j).
 * Page section "5. 플래시 어텐션 통합" (causal call with window_size).
 * Inputs are the prologue's outputs. */
cswattn_status attn_fwd(const cswattn_layer* layer, const void* q_out, const void* k_out,
                        const void* v_out, void* O, float* lse, void* stream);

/* Bytes of device scratch attn_bwd needs for this layer (the backward of
 * the page section "5. 플래시 어텐션 통합" call, see attn_bwd): float32
 * accumulators of dq_out (B, T, n_head, head_dim), P partial sums each of
 * dk_out and dv_out (B, T, n_kv_head, head_dim) (P = 1..8, the number of
 * CTAs the bf16 backward splits a key tile's work into; 1 for f32), and two
 * row terms (dO.O and lse*log2(e)),
 * each (B, n_head, Tpad) with Tpad = T rounded up to a multiple of 64;
 * every part padded to 256 bytes. Returns 0 for an invalid layer. */
size_t attn_bwd_workspace_bytes(const cswattn_layer* layer);

/* Backward of prologue + forward for the loss L with dL/dO = dO: the
 * gradient of the causal windowed attention call of page section
 * "5. 플래시 어텐션 통합 (nanochat/flash_attention.py)" and of the
 * steps before it in section "1. GPT 모델" (RoPE and QK normalisation of
 * the architecture list, the value-embedding code), written out:
 *   p = softmax(scale q_out k_out^T) over the window, dp = dO v_out^T,
 *   ds = p (dp - rowsum(dO * O)), dq_out = scale ds k_out,
 *   dk_out = scale ds^T q_out and dv_out = p^T dO summed over each KV
 *   head's group of query heads, then back through RoPE and RMSNorm:
 * dQ, dK (through RoPE^-1 and RMSNorm), dV = dL/dv_out, and when has_ve
 * dve = 3*sigmoid(gate)*dV and dgate = 3*sigmoid(gate)*(1-sigmoid(gate)) *
 * sum_d dV*ve. q, k, ve, gate are the prologue's inputs; q_out, k_out, v_out,
 * rstd_q, rstd_k its outputs; O and lse the forward's outputs.
 * workspace: caller-owned device scratch of at least
 * attn_bwd_workspace_bytes(layer) bytes, 256-byte aligned, whose contents on
 * entry do not matter; it must not be used by another call in flight.
 * dve and dgate are written only when has_ve (may be NULL otherwise). */
cswattn_status attn_bwd(const cswattn_layer* layer, const void* q, const void* k,
                        const void* ve, const void* gate, const void* q_out,
                        const void* k_out, const void* v_out, const float* rstd_q,
                        const float* rstd_k, const void* O, const float* lse,
                        const void* dO, void* dQ, void* dK, void* dV, void* dve,
                        void* dgate, void* workspace, size_t workspace_bytes,
                        void* stream);

/* Size of the fixed scratch array that attn_bwd_noalloc uses: 32 MiB. */
#define CSWATTN_NOALLOC_SCRATCH_BYTES (32u << 20)

/* attn_bwd without a caller-provided workspace, for callers that cannot
 * allocate device memory. The web pages this library follows describe no
 * such entry point; it exists for library users only.
 *
 * Who needs it: code whose device memory is owned entirely by another
 * allocator (a framework's caching allocator or a fixed arena that must
 * account for every byte), and code that may not call cudaMalloc in its
 * step loop because cudaMalloc can synchronize the device and stall other
 * work. Such callers can still pass their input and output tensors, but
 * they cannot hand over the few tens of megabytes of float32 scratch that
 * attn_bwd needs.
 *
 * Behaviour: identical arguments and results to attn_bwd, minus
 * `workspace`/`workspace_bytes`. The scratch is a static array of
 * CSWATTN_NOALLOC_SCRATCH_BYTES inside this library; every GPU that loads
 * the library holds it until the process exits. Layers whose
 * attn_bwd_workspace_bytes() exceeds that size are rejected with
 * CSWATTN_ERR_UNSUPPORTED before anything is enqueued (use attn_bwd with
 * your own workspace for those). No call allocates device memory
 * through cudaMalloc or any allocator: the array is part of the library's
 * device code. Under lazy module loading (the CUDA default) that code, and
 * with it the array, is loaded onto a device by the first call of this
 * library there, which may synchronize that device; make one warm-up call
 * on each device outside the step loop and before any stream capture.
 * Every call looks up the array's address on the device current at the
 * call (a host-side lookup), so the entry point keeps working after a
 * device reset. All calls on a device share the one array: two calls
 * that may overlap on the GPU (different streams, no ordering between
 * them) race and corrupt each other's results, so order them, for example
 * by issuing them on one stream. The array keeps whatever the last call
 * left in it; each call clears what must start at zero itself. */
cswattn_status attn_bwd_noalloc(const cswattn_layer* layer, const void* q, const void* k,
                                const void* ve, const void* gate, const void* q_out,
                                const void* k_out, const void* v_out, const float* rstd_q,
                                const float* rstd_k, const void* O, const float* lse,
                                const void* dO, void* dQ, void* dK, void* dV, void* dve,
                                void* dgate, void* stream);

/* Bytes of device scratch attn_decode needs for this layer (layer->T is the
 * cache capacity): per query head, the partial results of the splits of the
 * window (max, sum and head_dim partial outputs per split), each part padded
 * to 256 bytes. A sequence's window is split only while B * n_kv_head is
 * below 148 (one split per SM), into at most one split per 128-key chunk it
 * can straddle. 0 for an invalid or unsupported layer. */
size_t attn_decode_workspace_bytes(const cswattn_layer* layer);

/* Decode step with a key/value cache: page section "6. 추론 엔진
 * (nanochat/engine.py)" (generation over a pre-filled KV cache,
 * flash_attn_with_kvcache), one new token per sequence.
 * layer: bf16, head_dim 64 or 128, n_head / n_kv_head <= 16; T is the cache
 * capacity (rows per sequence), window as in attn_fwd.
 * cache_len (device int32, B): tokens already in sequence b's cache; the
 * new token's position is p = cache_len[b], which must lie in [0, T) (a
 * value outside is not checked on the host: the sequence is left untouched
 * and the next cswattn_sync_status() returns CSWATTN_ERR_INVALID_ARG).
 * q (B, n_head, head_dim), k, v, ve (B, n_kv_head, head_dim), gate
 * (B, n_kv_head): the new token's projections, as for attn_prologue with
 * T = 1; ve and gate only when has_ve.
 * k_cache, v_cache (B, T, n_kv_head, head_dim): rows 0..p-1 hold the k~ and
 * v_eff rows of earlier tokens (prologue outputs). The call writes row p of
 * both (k~ = RoPE_p(RMSNorm(k)), v_eff = v + 3*sigmoid(gate)*ve); it does
 * not change cache_len (the caller advances it).
 * O (B, n_head, head_dim), lse (B, n_head), natural log: attention of
 * q~ = RoPE_p(RMSNorm(q)) over cache rows (p - window, p].
 * workspace: caller-owned device scratch of at least
 * attn_decode_workspace_bytes(layer) bytes, 256-byte aligned. */
cswattn_status attn_decode(const cswattn_layer* layer, const void* q, const void* k,
                           const void* v, const void* ve, const void* gate, const int* cache_len,
                           void* k_cache, void* v_cache, void* O, float* lse, void* workspace,
                           size_t workspace_bytes, void* stream);

/* bf16 matrix product on the tensor cores, the step Muon's orthogonalisation
 * is made of (page section "2. Muon 옵티마이저 (nanochat/optim.py)"):
 *   C[m][n] = alpha * sum_k Aop[m][k] * Bop[n][k] + beta * D[m][n]
 * Aop[m][k] = A[m*lda + k] (a_mn = 0: A is M x K, K contiguous) or
 * A[k*lda + m] (a_mn = 1: A is K x M, M contiguous); Bop[n][k] = B[n*ldb + k]
 * (b_mn = 0) or B[k*ldb + n] (b_mn = 1). So a_mn = 0, b_mn = 1 is the plain
 * product of row-major A (M x K) and B (K x N). C and D: M x N, row-major
 * with ldc, ldd (D read only when beta != 0; D may be C). bf16 A, B, C, D,
 * float32 accumulation. N and every leading dimension a multiple of 8
 * elements, pointers 16-byte aligned, C not aliasing A or B; other sizes
 * are free (partial tiles read zeros past the edges). */
cswattn_status cswattn_gemm_bf16(int M, int N, int K, int a_mn, const void* A, long long lda, int b_mn,
                                 const void* B, long long ldb, float alpha, float beta, const void* D,
                                 long long ldd, void* C, long long ldc, void* stream);

/* Bytes of device scratch muon_newton_schulz needs for an m x n matrix:
 * A and B (n x n) and one m x n iterate, bf16, each padded to 256 bytes.
 * 0 for m or n < 1. */
size_t muon_ns_workspace_bytes(int m, int n);

/* Muon's orthogonalisation by the quintic Newton-Schulz ("Polar Express")
 * iteration of page section "2. Muon 옵티마이저 (nanochat/optim.py)", in
 * the page's order and notation, one step per coefficient triple:
 *   A = X^T X;  B = b*A + c*(A A);  X = a*X + X B
 * coeffs: host array of 3*steps floats (a, b, c per step; the page prints
 * the first two triples, (8.156, -22.483, 15.879) and (4.043, -2.809, 0.5),
 * and elides the rest). X (m x n, row-major, bf16) is the input iterate
 * (the caller scales it as it wishes beforehand; the iteration is
 * equivariant under transposition, so a wide matrix may be passed
 * transposed to make A the smaller product); Y (m x n, bf16) receives the
 * result and must not alias X. Every product is a cswattn_gemm_bf16 with
 * bf16 intermediates. n a multiple of 8, 1 <= steps <= 64; workspace of at
 * least muon_ns_workspace_bytes(m, n), 256-byte aligned. */
cswattn_status muon_newton_schulz(int m, int n, const float* coeffs, int steps, const void* X, void* Y,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* Error reporting of the device side (no counterpart on the pages, which
 * describe no error handling): waits for `stream`, then returns and clears
 * the device status word of the
 * current device: CSWATTN_ERR_TIMEOUT if a kernel's bounded wait ran out
 * since the last check, CSWATTN_ERR_INVALID_ARG if a decode step met a cache
 * length outside [0, T), CSWATTN_ERR_BOUNDS if a bounds check of the
 * checked build (libcswattn_check.so, compiled with CSWATTN_CHECK=1) failed
 * (the access was skipped), CSWATTN_ERR_CUDA on a CUDA error, else
 * CSWATTN_OK. */
cswattn_status cswattn_sync_status(void* stream);

/* Self-test of the bounded-wait path: launches one small kernel whose thread
 * waits on a barrier that nothing ever arrives on, using the same bounded
 * wait as the attention kernels, with a limit of `limit_ns` (clamped to
 * [1000, 1e9]). The wait runs out, the kernel records CSWATTN_ERR_TIMEOUT in
 * the device status word and returns; a following cswattn_sync_status()
 * reports (and clears) it. Touches no TMEM and issues no copies. */
cswattn_status cswattn_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/* Upper bound, in nanoseconds, of the device-side waits of later launches
 * on each other's progress (default 2e9); returns the limit applied. Values
 * below 1e6 (1 ms) are raised to 1e6. Process-wide. This limit does not
 * bound a kernel's final waits for its own copies and matrix products in
 * flight (they have a fixed bound of 10 s), so a short limit never lets a
 * kernel exit, or free its tensor memory, while they are still running. */
uint64_t cswattn_set_wait_limit_ns(uint64_t ns);

/* Kernel kinds reported by cswattn_kernel_times(). */
enum {
  CSWATTN_K_PROLOGUE = 0, /* fused RMSNorm + RoPE + value residual */
  CSWATTN_K_FWD = 1,      /* attention forward (tensor cores, or fp32 CUDA cores) */
  CSWATTN_K_BWD_PRE = 2,  /* backward row terms Delta = rowsum(dO * O) */
  CSWATTN_K_BWD = 3,      /* attention backward main kernel(s) */
  CSWATTN_K_BWD_EPI = 4,  /* backward epilogue: RoPE^-1, RMSNorm', dv/dve/dgate */
  CSWATTN_K_DECODE = 5,   /* decode step: new-token prologue, split-KV attention, combine */
  CSWATTN_K_GATE_BWD = 6, /* backward of the value-embedding gate's projection */
  CSWATTN_K_GEMM = 7,     /* bf16 matrix product (the Newton-Schulz steps) */
  CSWATTN_NUM_KERNELS = 8
};

/* Per-kernel device timing for measurement tools. With enable != 0, every
 * later call records a CUDA event pair around each kernel it launches, on the
 * caller's stream (events are created once and reused; no device memory is
 * allocated). Process-wide; off by default. */
void cswattn_set_timing(int enable);

/* Waits for the recorded event pairs, writes the summed milliseconds and the
 * launch count of each kernel kind into ms[CSWATTN_NUM_KERNELS] and
 * launches[CSWATTN_NUM_KERNELS] (host arrays, either may be NULL), and clears
 * the record. Returns CSWATTN_ERR_CUDA if an event query fails. */
cswattn_status cswattn_kernel_times(double* ms, int* launches);

/* Message for the last failed call on this thread ("" if none). The string
 * is owned by the library and valid until the next call on this thread. */
const char* cswattn_last_error(void);

/* Library ABI version, (major << 16) | minor. */
int cswattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CSWATTN_H */
