/*
 * agent_attn.h -- C ABI of the B200 (sm_100a) Agent Attention forward pass.
 *
 * The operation (per batch b and head h, "slice"):
 *
 *   A   = agents: pool_h x pool_w adaptive average pool of Q over its
 *         grid_h x grid_w token grid, or externally supplied learnable agents.
 *         [Agent Attention: On the Integration of Softmax and Linear Attention,
 *          arXiv:2312.08874v3 summary, §4 "Efficiency" (pooling is the default
 *          agent source; learnable parameters are another) and §6 (A = f(Q)).]
 *   V_A = softmax(A K^T * scale) V            agent aggregation  (k x d)
 *   O   = softmax(Q A^T * scale) V_A          agent broadcast    (N x d)
 *         [jsqmd.com, "Agent Attention：Transformer计算量太大？试试这个'代理令牌'
 *          的轻量化方案", §1 two-stage pseudocode (scale 1/sqrt(d) in both
 *          softmaxes); arXiv:2312.08874v3 summary §4 "Agent Attention".]
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Tensors are contiguous row-major [B, H, N, d] device buffers of the element
 * type `dtype` (AA_FP32: float, AA_BF16: bfloat16).  Tokens are row-major on
 * the grid, token n = y * grid_w + x; agent j = py * pool_w + px.  Adaptive
 * pooling bin i of an axis of length G cut into P bins covers tokens
 * [floor(i*G/P), ceil((i+1)*G/P)); neighbouring bins may share a row when P
 * does not divide G.  `scale` multiplies the logits of both softmaxes (the
 * pages use 1/sqrt(d)).
 *
 * Limits: B, H, N >= 1; N == grid_h * grid_w for pooled agents;
 * 1 <= pool_h <= grid_h, 1 <= pool_w <= grid_w; 1 <= k <= 256 agents;
 * 8 <= d <= 128 with d % 8 == 0; every pointer 16-byte aligned; scale finite
 * and > 0; `out` must not alias an input.
 *
 * Ownership: the caller owns every buffer.  The library keeps no pointer to
 * them after a call returns.  Its global state is per device and created on
 * first use: a cache of the SM count and of each kernel's raised
 * shared-memory limit; a library-owned stream-ordered memory pool (release
 * threshold = unlimited) from which the entry points without a caller
 * workspace take their scratch; one non-blocking side stream (used only by
 * agent_attn_forward_host); the in-kernel watchdog word read by
 * agent_attn_check_device_error; and the fixed scratch array of
 * agent_attn_stage_aggregate_static.  Calls on different streams are
 * independent.
 *
 * Errors: every call validates all arguments before it launches anything and
 * returns an aa_status.  AA_ERR_CUDA means a CUDA call or launch failed; the
 * CUDA error text of the last such failure on the calling thread is then
 * available from agent_attn_status_string(AA_ERR_CUDA).  Calls are
 * asynchronous on `stream` (a cudaStream_t; NULL = the legacy default stream)
 * unless stated otherwise.
 */
#ifndef AGENT_ATTN_H_
#define AGENT_ATTN_H_

#include <stddef.h>

#if defined(__GNUC__)
#define AA_API __attribute__((visibility("default")))
#else
#define AA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  AA_OK = 0,
  AA_ERR_NULL = 1,         /* a required pointer is NULL                              */
  AA_ERR_SHAPE = 2,        /* sizes inconsistent (N != grid_h*grid_w, pool > grid...) */
  AA_ERR_UNSUPPORTED = 3,  /* dtype, d or k outside the supported set                 */
  AA_ERR_ALIGN = 4,        /* a pointer is not 16-byte aligned                        */
  AA_ERR_WORKSPACE = 5,    /* caller workspace too small                              */
  AA_ERR_CUDA = 6,         /* a CUDA runtime / driver call or a launch failed         */
  AA_ERR_VALUE = 7,        /* scale not finite or not > 0                              */
  AA_ERR_TIMEOUT = 8       /* a kernel's bounded wait expired (see check_device_error) */
} aa_status;

typedef enum { AA_FP32 = 0, AA_BF16 = 1 } aa_dtype;

/* Whole forward pass with pooled agents.
 *   q, k, v, out : [B, H, N, d] device buffers of `dtype`.
 *   agents_or_null: NULL -> agents are pooled from q (pool_h x pool_w of them);
 *                   non-NULL -> [H, pool_h*pool_w, d] learnable agents of
 *                   `dtype`, shared over the batch (grid only checked vs N).
 * Scratch memory (agents, partial aggregation state, V_A) is taken from the
 * library's stream-ordered pool on `stream` and returned to it (freed in
 * stream order) before the call returns.  bf16 slices of at most 256 tokens
 * with at most 128 agents (pooled or given) and d <= 64 run as one fused
 * kernel (one CTA per slice, no scratch); the result is the same
 * computation. */
AA_API int agent_attn_forward(const void* q, const void* k, const void* v, const void* agents_or_null,
                       void* out, int B, int H, int N, int d, int grid_h, int grid_w, int pool_h,
                       int pool_w, float scale, int dtype, void* stream);

/* Same as agent_attn_forward, with caller-provided scratch: `workspace` is a
 * device buffer of at least agent_attn_workspace_bytes(B, H, N, d,
 * pool_h*pool_w, dtype) bytes, 256-byte aligned; AA_ERR_WORKSPACE otherwise.
 * Its contents on entry do not matter and are garbage on exit. */
AA_API int agent_attn_forward_ws(const void* q, const void* k, const void* v, const void* agents_or_null,
                          void* out, int B, int H, int N, int d, int grid_h, int grid_w,
                          int pool_h, int pool_w, float scale, int dtype, void* workspace,
                          size_t ws_bytes, void* stream);

/* Forward pass with externally supplied (learnable) agents; pooling is skipped.
 *   agents: n_agents x d agent rows of `dtype`; slice (b, h) reads
 *           agents + b*agents_batch_stride + h*n_agents*d (elements), so a
 *           stride of 0 shares one [H, n_agents, d] set over the batch and a
 *           stride of H*n_agents*d reads a full [B, H, n_agents, d] tensor.
 *           agents_batch_stride must be 0 or a multiple of 8 elements. */
AA_API int agent_attn_forward_agents(const void* q, const void* k, const void* v, const void* agents,
                              int n_agents, long long agents_batch_stride, void* out, int B,
                              int H, int N, int d, float scale, int dtype, void* stream);

/* Scratch bytes the forward pass needs for this problem on the current
 * device (it depends on the device's SM count).  Returns 0 if the arguments
 * are invalid or no device is visible. */
AA_API size_t agent_attn_workspace_bytes(int B, int H, int N, int d, int n_agents, int dtype);

/* Synchronous convenience call on HOST buffers: copies q, k, v (and agents,
 * if non-NULL: [H, pool_h*pool_w, d]) to the device, runs the forward pass
 * and copies the result back into out_host, then synchronizes `stream`.
 * The slices are cut into up to 8 chunks (whole batches when agents are
 * given) whose upload, forward pass and download alternate between `stream`
 * and a second, library-owned stream, so one chunk's upload overlaps the
 * previous chunk's compute and download.  Device buffers come from the
 * library's stream-ordered pool.  Host buffers should be page-locked for the
 * copies to run asynchronously at full link speed; pageable memory also works. */
AA_API int agent_attn_forward_host(const void* q_host, const void* k_host, const void* v_host,
                            const void* agents_host_or_null, void* out_host, int B, int H, int N,
                            int d, int grid_h, int grid_w, int pool_h, int pool_w, float scale,
                            int dtype, void* stream);

/* ---- single stages (the same kernels the forward pass launches) ---- */

/* Agent pooling only: agents_f32 [B, H, pool_h*pool_w, d] float (may be NULL)
 * and agents_lowp [B, H, pool_h*pool_w, d] of `dtype` (may be NULL; ignored
 * for AA_FP32).  At least one output must be non-NULL. */
AA_API int agent_attn_stage_pool(const void* q, float* agents_f32, void* agents_lowp, int B, int H, int N,
                          int d, int grid_h, int grid_w, int pool_h, int pool_w, int dtype,
                          void* stream);

/* Agent aggregation (split over keys, then the log-sum-exp merge of the
 * splits): va_f32 [B, H, n_agents, d] float (may be NULL) and va_lowp
 * [B, H, n_agents, d] of `dtype` (may be NULL for AA_FP32).  agents is
 * addressed as in agent_attn_forward_agents.  Scratch from the library's
 * stream-ordered pool. */
AA_API int agent_attn_stage_aggregate(const void* agents, long long agents_batch_stride, const void* k,
                               const void* v, float* va_f32, void* va_lowp, int B, int H, int N,
                               int d, int n_agents, float scale, int dtype, void* stream);

/* Agent broadcast: out [B, H, N, d] of `dtype` from q, agents (addressed as
 * in agent_attn_forward_agents) and va [B, H, n_agents, d] of `dtype`. */
AA_API int agent_attn_stage_broadcast(const void* q, const void* agents, long long agents_batch_stride,
                               const void* va, void* out, int B, int H, int N, int d,
                               int n_agents, float scale, int dtype, void* stream);

/* ---- aggregation without any allocation ----
 *
 * No counterpart in the paper: this entry point exists for callers that may
 * not allocate device memory themselves, e.g. code running as a plugin inside
 * a host framework that owns and budgets all device memory, or a real-time
 * loop that forbids allocation after start-up.
 *
 * Same inputs, outputs and semantics as agent_attn_stage_aggregate, but the
 * split-over-keys partial state lives in one fixed array inside the library
 * (a file-scope __device__ array of AA_STATIC_SCRATCH_BYTES bytes, present on
 * every device that loads the library until the process exits) instead of
 * memory taken from a pool.  The call allocates and frees nothing.
 *   - Problems whose partial state exceeds AA_STATIC_SCRATCH_BYTES are
 *     rejected with AA_ERR_WORKSPACE before anything is launched.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture on the device.
 *   - Every call shares the one array and it keeps the last call's contents;
 *     nothing in it needs to start at zero (each call writes every partial it
 *     reads back).  Calls whose work overlaps on the GPU (different streams,
 *     or several host threads) race on the array: serialise them. */
#define AA_STATIC_SCRATCH_BYTES (16u << 20)

AA_API int agent_attn_stage_aggregate_static(const void* agents, long long agents_batch_stride,
                                             const void* k, const void* v, float* va_f32,
                                             void* va_lowp, int B, int H, int N, int d,
                                             int n_agents, float scale, int dtype, void* stream);

/* ---- agent bias ----
 *
 * Bias terms added to the logits of both softmaxes (arXiv:2312.08874v3
 * summary, §4 "Module Enhancements": B1 and B2 enter both attention
 * operations; §6 "Implementation Details": column, row and block components
 * build the full bias).  Read here, per head h, agent a and grid token
 * n = y*grid_w + x, as
 *   bias[h, a, n] = row[h, a, y] + col[h, a, x] + block[h, a, cell(y, x)],
 *   cell(y, x) = floor(y*pool_h/grid_h)*pool_w + floor(x*pool_w/grid_w)
 * (the floor partition of the grid into the pool_h x pool_w agent cells).
 *   aggregation: V_A[a] = softmax_n(scale * A_a . K_n + B1[h, a, n]) V
 *   broadcast:   O[n]   = softmax_a(scale * Q_n . A_a + B2[h, a, n]) V_A
 * Components are fp32 device buffers shared over the batch (4-byte aligned):
 *   *_row [H, k, grid_h], *_col [H, k, grid_w], *_block [H, k, pool_h*pool_w],
 * k = pool_h*pool_w; each may be NULL (contributes zero).  Other arguments as
 * in agent_attn_forward.  bf16 problems first build a dense copy of each bias
 * (B * log2(e) as fp16: 11-bit significands, values saturated at +-65504,
 * i.e. |B| up to about 45000) and add it inside the tensor-core score tiles;
 * fp32 problems, and grids whose components do not fit the builder's shared
 * memory (grid_h + grid_w above about 20000), add the fp32 components on the
 * SIMT kernels.  Scratch for the dense copies (2 bytes per agent, token and
 * head for B1; twice that for B2, built tokens-contiguous and then
 * transposed) comes from the library's stream-ordered pool. */
AA_API int agent_attn_forward_bias(const void* q, const void* k, const void* v,
                                   const void* agents_or_null, const float* b1_row,
                                   const float* b1_col, const float* b1_block,
                                   const float* b2_row, const float* b2_col,
                                   const float* b2_block, void* out, int B, int H, int N, int d,
                                   int grid_h, int grid_w, int pool_h, int pool_w, float scale,
                                   int dtype, void* stream);

/* ---- backward pass ----
 *
 * Gradients of agent_attn_forward (pooled agents, agents_or_null == NULL) or
 * of the forward pass with given agents [H, k, d] (agents_or_null), for
 * finetuning through both softmax stages (arXiv:2312.08874v3 summary, C.4
 * "AgentSD for finetuning": agent attention is used during finetuning).  The
 * pages give no formulas; the gradients are the derivatives of the forward
 * definition:
 *   dV_A = P2^T dO, dS2 = P2 .* (dO V_A^T - rowsum(P2 .* dO V_A^T)),
 *   dQ = s dS2 A (+ the pooling adjoint of dA for pooled agents),
 *   dS1 = P1 .* (dV_A V^T - rowsum(P1 .* dV_A V^T)), dK = s dS1^T A,
 *   dV = P1^T dV_A, dA = s dS2^T Q + s dS1 K,
 * with P1 = softmax_rows(s A K^T), P2 = softmax_rows(s Q A^T).
 *   dout            : [B, H, N, d] gradient of the output, `dtype`.
 *   dq, dk, dv      : [B, H, N, d] outputs, `dtype` (16-byte aligned).
 *   dagents_or_null : [B, H, k, d] fp32 output (gradient of each slice's
 *                     agents; sum over B for agents shared over the batch),
 *                     or NULL.
 * The gradient kernels are SIMT with fp32 arithmetic.  The forward statistics
 * are recomputed; for bf16 with d <= 64 on the tensor cores, which also
 * supply the exponentials of both softmaxes as bf16 (the values the forward
 * pass's P V products use), so the scratch holds one [B, H, N, k rounded up
 * to 16] bf16 array beside the fp32 accumulators.  The per-agent sums use
 * fp32 atomic additions, so results may differ from run to run at rounding
 * level.  B*H <= 65535. */
AA_API int agent_attn_backward(const void* q, const void* k, const void* v,
                               const void* agents_or_null, const void* dout, void* dq, void* dk,
                               void* dv, float* dagents_or_null, int B, int H, int N, int d,
                               int grid_h, int grid_w, int pool_h, int pool_w, float scale,
                               int dtype, void* stream);

/* ---- the depth-wise convolution term of the full module ----
 *
 * The full Agent Attention module adds a depth-wise convolution term to the
 * attention output (arXiv:2312.08874v3 summary, §4 "Module Enhancements": the
 * full module adds a depth-wise convolution term, cost k^2 N C with k = 3).
 * Read here as a 3x3 depth-wise convolution of V over the token grid, one
 * kernel per (head, channel), zero padding, output on the same grid:
 *   DWC(V)[b,h,y*grid_w+x,c] = bias[h,c]
 *       + sum_{ty,tx in 0..2} w[h,c,ty,tx] * V[b,h,(y+ty-1)*grid_w+(x+tx-1),c]
 * (positions outside the grid contribute zero).
 *
 * agent_attn_dwc: out (+)= DWC(v).
 *   v, out        : [B, H, grid_h*grid_w, d] device buffers of `dtype`
 *                   (16-byte aligned); out may not alias v.
 *   w             : [H, d, 3, 3] fp32 device buffer (4-byte aligned).
 *   bias_or_null  : [H, d] fp32 device buffer, or NULL for no bias.
 *   accumulate    : 0 -> out = DWC(v); non-zero -> out = out + DWC(v)
 *                   (computed in fp32, rounded once to `dtype`).
 * Same d / dtype rules as the forward pass, and grid_h*grid_w*d/8 < 2^31
 * (else AA_ERR_SHAPE); asynchronous on `stream`. */
AA_API int agent_attn_dwc(const void* v, const float* w, const float* bias_or_null, void* out,
                          int B, int H, int grid_h, int grid_w, int d, int dtype, int accumulate,
                          void* stream);

/* The full module output: out = AgentAttention(q, k, v) + DWC(v), i.e.
 * agent_attn_forward followed by agent_attn_dwc(accumulate = 1) on the same
 * stream (the convolution kernel reads its V taps while the broadcast is
 * still running and waits for it only before touching out).  Arguments as
 * in agent_attn_forward and agent_attn_dwc. */
AA_API int agent_attn_forward_dwc(const void* q, const void* k, const void* v,
                                  const void* agents_or_null, const float* dwc_w,
                                  const float* dwc_bias_or_null, void* out, int B, int H, int N,
                                  int d, int grid_h, int grid_w, int pool_h, int pool_w,
                                  float scale, int dtype, void* stream);

/* Human-readable text for a status code (for AA_ERR_CUDA, includes the last
 * CUDA error text seen on the calling thread).  Never NULL. */
AA_API const char* agent_attn_status_string(int status);

/* Reads and clears the device-side watchdog of the current device.  Every
 * wait inside the tensor-core kernels is bounded (2 s); a wait that expires
 * makes its CTA skip the rest of its work, leaves the outputs invalid and
 * sets the watchdog.  Returns AA_ERR_TIMEOUT if it was set since the last
 * check, AA_OK otherwise.  Synchronous with respect to the device. */
AA_API int agent_attn_check_device_error(void);

/* Test hook for the exponential that the tensor-core softmax kernels take on
 * the FMA pipe for part of each score row instead of the SFU.  No counterpart
 * in the pages: it exists so that this function can be checked against
 * CUDA's exp2f.  It computes 2^x by the Cody-Waite split x = j + f
 * (j = rint(x), f in [-1/2, 1/2]), a degree-3 polynomial for 2^f fitted to
 * the smallest maximum relative error on [-1/2, 1/2] (7.5e-5) and the
 * exponent-field insertion of j; arguments below -125 give about 2^-125.
 *   x     : [n] device floats (4-byte aligned), the arguments;
 *   y_fma : [n] device floats, the FMA-pipe exponential of x;
 *   y_ref : [n] device floats, exp2f(x).
 * n >= 0 (0 launches nothing); asynchronous on `stream`. */
AA_API int agent_attn_selftest_exp2(const float* x, float* y_fma, float* y_ref, int n,
                                    void* stream);

/* Library version, "major.minor.patch". */
AA_API const char* agent_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* AGENT_ATTN_H_ */
