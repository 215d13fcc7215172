/*
 * gla.h - C ABI of libgla.so: gated bidirectional ReLU linear attention on
 * NVIDIA B200 (sm_100a).
 *
 * The operator (per batch element b and head h, head dim d, N = T*H*W latent
 * tokens in raster order n = (t*H + h)*W + w):
 *
 *   q_hat = RMSNorm(q), k_hat = RMSNorm(k)       over d, no weight, eps 1e-6
 *   q_pls = ReLU(q_hat), k_pls = ReLU(k_hat)
 *   q_til = RoPE3D(q_pls), k_til = RoPE3D(k_pls)  (rotation after the ReLU)
 *   S     = sum_n v_n (beta_n k_til_n)^T            d x d, S[a][c]
 *   z     = sum_n k_pls_n                           d
 *   den_j = z . q_pls_j + eps                       (no rotation: stays > 0)
 *   o_j   = RMSNorm( sigmoid(g_j) * (S q_til_j) / den_j )
 *
 * Sources: the SANA-Video 2.0 summary (paper.rainbus.top), prerequisites
 * "Gated Bilinear Linear Attention" (the read-out o_j, normalised q/k, phi =
 * ReLU, write gate beta, sigmoid output gate g, bidirectional sum) and
 * "Linear Attention" (S = sum_n v_n (beta_n k_n)^T); the SANA-Video notes
 * (papernotes.org), key design 1 (RoPE(ReLU(x)), RoPE in the numerator only so
 * the denominator stays positive) and key design 2 (block-causal linear
 * attention carries the running sums of S and of the key features).  The
 * output projection W_o of the read-out formula is not part of this library.
 *
 * 3D RoPE (the pages fix no split; this is the library's normative spec):
 *   P = d/2 rotation pairs.  Time gets P - 2*floor(P/3) pairs, height and
 *   width floor(P/3) each (22/21/21 for d = 128, 6/5/5 for d = 32), as
 *   contiguous channel chunks in the order t, h, w.  Inside an axis chunk of
 *   p pairs, pair i is channels (2i, 2i+1), frequency theta^(-i/p), angle
 *   pos * frequency, and (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos).
 *   Positions are integers from 0; the time position is t0 + local frame in
 *   gla_block_causal_step (0 in gla_forward).  rope_theta <= 0 disables RoPE.
 *
 * Layouts (all caller-owned DEVICE memory unless stated, contiguous, 16-byte
 * aligned):  q, k, v, g, out: [batch][N][heads][head_dim] in `dtype`;
 * beta: [batch][N][heads] in `dtype` (taken as given: apply its sigmoid
 * before the call); g holds gate logits (the operator applies the sigmoid).
 * State S: [batch][heads][d][d] fp32 with S[a][c] = sum_n v_n[a] beta_n
 * k_til_n[c]; z: [batch][heads][d] fp32.
 *
 * Supported: dtype F32 or BF16; head_dim 32, 64 or 128.  BF16 with
 * head_dim 128 runs on the tcgen05 tensor-core path (TMA-fed state reduction
 * and read-out); every other case, or path GLA_PATH_SIMT, runs on CUDA cores
 * with fp32 arithmetic.  Accumulation is always fp32.  On the tensor path the
 * state MMA's operand beta*k_til is rounded to bf16 (v arrives in bf16), and
 * the read-out MMA's operands q_til and S to fp16 (q_til is bounded by
 * sqrt(d) after the RMSNorm; S carries one power-of-two scale per head that
 * puts its largest entry in [2^13, 2^14)); outputs are rounded to nearest
 * even.
 *
 * Errors: every entry point validates its arguments first and returns an
 * error code with nothing launched.  A CUDA launch failure returns
 * GLA_ERR_CUDA.  Calls are asynchronous on `stream` (a cudaStream_t passed as
 * void*; NULL = legacy default stream) and stream-ordered.  On the tensor
 * path the kernels of a call chain by programmatic dependent launch: the
 * first may start its set-up while the preceding kernel on the stream is
 * finishing, but reads no input before that kernel has completed.
 * Device-side wait timeouts (the tensor path's bounded mbarrier waits) are
 * recorded in a library-owned device word and reported by
 * gla_get_device_status().
 *
 * Determinism: the state is reduced in a fixed split order, so the same
 * inputs on the same GPU model give bitwise-identical results.
 *
 * Memory: the library allocates no device memory.  Scratch space is the
 * caller's `workspace` of at least *_workspace_size() bytes, 256-byte
 * aligned; its contents need no initialisation and are overwritten.  The
 * only resources it creates itself are, per device and on first use by
 * gla_forward_host with batch >= 2, one non-blocking stream and nine events,
 * kept until the process exits.
 */
#ifndef GLA_H
#define GLA_H

#include <stddef.h>

#if defined(__GNUC__)
#define GLA_API __attribute__((visibility("default")))
#else
#define GLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gla_status {
  GLA_OK = 0,
  GLA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, eps <= 0 */
  GLA_ERR_UNSUPPORTED = 2,  /* head_dim/dtype/path combination not built */
  GLA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required */
  GLA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  GLA_ERR_TIMEOUT = 5       /* a device-side bounded wait expired */
} gla_status;

typedef enum gla_dtype { GLA_DTYPE_F32 = 0, GLA_DTYPE_BF16 = 1 } gla_dtype;

typedef enum gla_path {
  GLA_PATH_AUTO = 0,   /* tensor path when supported, else SIMT */
  GLA_PATH_SIMT = 1,   /* CUDA-core fp32 kernels */
  GLA_PATH_TENSOR = 2  /* tcgen05 + TMA kernels (bf16, head_dim 128 only) */
} gla_path;

/* RMSNorm epsilon used for q, k and the output (a fixed library constant). */
#define GLA_RMS_EPS 1e-6f

/* Library version, major*10000 + minor*100 + patch. */
GLA_API int gla_version(void);

/* Human-readable name of a status code (static string, never NULL). */
GLA_API const char* gla_status_string(int status);

/* Bytes of workspace gla_forward / gla_forward_ex / gla_forward_debug need
 * for this problem (independent of the GPU).  0 for invalid sizes. */
GLA_API size_t gla_forward_workspace_size(int batch, int heads, int head_dim, int T, int H,
                                  int W, int dtype);

/* The bidirectional operator over all N = T*H*W tokens (the read-out formula
 * of the "Gated Bilinear Linear Attention" prerequisite).  Writes out; reads
 * q, k, v, beta, g.  eps > 0 is the denominator epsilon. */
GLA_API gla_status gla_forward(const void* q, const void* k, const void* v, const void* beta,
                       const void* g, int batch, int heads, int head_dim, int T, int H,
                       int W, float rope_theta, float eps, int dtype, void* out,
                       void* workspace, size_t workspace_bytes, void* stream);

/* gla_forward with an explicit path (gla_path). */
GLA_API gla_status gla_forward_ex(const void* q, const void* k, const void* v, const void* beta,
                          const void* g, int batch, int heads, int head_dim, int T, int H,
                          int W, float rope_theta, float eps, int dtype, void* out,
                          void* workspace, size_t workspace_bytes, void* stream, int path);

/* gla_forward that also exports the hidden intermediates (tests):
 * S_out [batch][heads][d][d] fp32, z_out [batch][heads][d] fp32,
 * den_out [batch][N][heads] fp32 (den_j), x_out [batch][N][heads][d] fp32
 * (sigmoid(g_j) * S q_til_j / den_j, before the output RMSNorm).  Any of the
 * four may be NULL.  Slower than gla_forward. */
GLA_API gla_status gla_forward_debug(const void* q, const void* k, const void* v, const void* beta,
                             const void* g, int batch, int heads, int head_dim, int T,
                             int H, int W, float rope_theta, float eps, int dtype,
                             void* out, void* workspace, size_t workspace_bytes,
                             void* stream, int path, float* S_out, float* z_out,
                             float* den_out, float* x_out);

/* gla_forward that also records caller-created CUDA events (cudaEvent_t
 * passed as void*) on `stream` around its kernels: events[0] before the state
 * reduction, events[1] after it, events[2] after the combine, events[3] after
 * the read-out.  For per-kernel timing in benchmarks; `events` may be NULL and
 * any of its four entries may be NULL. */
GLA_API gla_status gla_forward_timed(const void* q, const void* k, const void* v,
                                     const void* beta, const void* g, int batch, int heads,
                                     int head_dim, int T, int H, int W, float rope_theta,
                                     float eps, int dtype, void* out, void* workspace,
                                     size_t workspace_bytes, void* stream, int path,
                                     void* const* events);

/* Workspace bytes of gla_block_causal_step for one block of T_blk*H*W tokens. */
GLA_API size_t gla_block_causal_workspace_size(int batch, int heads, int head_dim, int T_blk,
                                       int H, int W, int dtype);

/* One step of the block-causal variant (key design 2 of the SANA-Video notes:
 * a new block only adds its own state to the carried running sums).
 * state [batch][heads][d][d] fp32 and z [batch][heads][d] fp32 are caller-owned
 * device memory, read and updated in place: state += sum over the block of
 * v_n (beta_n k_til_n)^T, z += sum over the block of k_pls_n (added in a fixed
 * order).  The block's tokens are then read out against the UPDATED state (a
 * block sees itself).  RoPE time positions are t0 + local frame.  Zero state
 * and z before the first step. */
GLA_API gla_status gla_block_causal_step(float* state, float* z, const void* q, const void* k,
                                 const void* v, const void* beta, const void* g,
                                 int batch, int heads, int head_dim, int T_blk, int H,
                                 int W, int t0, float rope_theta, float eps, int dtype,
                                 void* out, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* gla_block_causal_step with an explicit path (gla_path). */
GLA_API gla_status gla_block_causal_step_ex(float* state, float* z, const void* q, const void* k,
                                    const void* v, const void* beta, const void* g,
                                    int batch, int heads, int head_dim, int T_blk, int H,
                                    int W, int t0, float rope_theta, float eps, int dtype,
                                    void* out, void* workspace, size_t workspace_bytes,
                                    void* stream, int path);

/* Workspace bytes of gla_causal_step / gla_causal_step_ex (the tensor path's
 * state partials and per-partial starting states; independent of the GPU). */
GLA_API size_t gla_causal_workspace_size(int batch, int heads, int head_dim, int T, int H,
                                         int W, int dtype);

/* Token-level causal variant over one call of T*H*W tokens, continuing a
 * sequence (SANA-Video notes, key design 2: causal linear attention needs only
 * the running sums of the per-token states v_n (beta_n k_til_n)^T and of the
 * key features k_pls_n).  Token j is read out against
 *   S_j = state + sum_{n <= j} v_n (beta_n k_til_n)^T,
 *   z_j = z     + sum_{n <= j} k_pls_n              (a token sees itself),
 * with den_j = z_j . q_pls_j + eps and the rest of the read-out as in
 * gla_forward.  state [batch][heads][d][d] fp32 and z [batch][heads][d] fp32
 * are caller-owned device memory holding the sums before the call's first
 * token (zero them to start a sequence); on return they hold the sums after
 * its last token, so consecutive calls over consecutive segments give the
 * causal read-out of the whole sequence.  RoPE time positions are t0 + local
 * frame.  Workspace: gla_causal_workspace_size() bytes, 256-byte aligned (the
 * CUDA-core path uses none and accepts NULL).  Other layouts, errors and
 * stream semantics as for gla_forward; the state is reduced in a fixed order,
 * so results are bitwise reproducible. */
GLA_API gla_status gla_causal_step(float* state, float* z, const void* q, const void* k,
                                   const void* v, const void* beta, const void* g, int batch,
                                   int heads, int head_dim, int T, int H, int W, int t0,
                                   float rope_theta, float eps, int dtype, void* out,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* gla_causal_step with an explicit path (gla_path) and optional exports of the
 * hidden intermediates (tests): den_out [batch][N][heads] fp32 (den_j) and
 * x_out [batch][N][heads][d] fp32 (sigmoid(g_j) * S_j q_til_j / den_j, before
 * the output RMSNorm); either may be NULL. */
GLA_API gla_status gla_causal_step_ex(float* state, float* z, const void* q, const void* k,
                                      const void* v, const void* beta, const void* g,
                                      int batch, int heads, int head_dim, int T, int H, int W,
                                      int t0, float rope_theta, float eps, int dtype, void* out,
                                      void* workspace, size_t workspace_bytes, void* stream,
                                      int path, float* den_out, float* x_out);

/* gla_causal_step_ex that also records caller-created CUDA events (cudaEvent_t
 * passed as void*) on `stream` around the tensor path's kernels: events[0]
 * before the state partials, events[1] after them, events[2] after their
 * prefix, events[3] after the causal read-out (the CUDA-core path records
 * events[0] only).  For per-kernel timing in benchmarks; `events` and any of
 * its entries may be NULL. */
GLA_API gla_status gla_causal_step_timed(float* state, float* z, const void* q, const void* k,
                                         const void* v, const void* beta, const void* g,
                                         int batch, int heads, int head_dim, int T, int H, int W,
                                         int t0, float rope_theta, float eps, int dtype,
                                         void* out, void* workspace, size_t workspace_bytes,
                                         void* stream, int path, float* den_out, float* x_out,
                                         void* const* events);

/* ------------------------------------------------------------------------
 * FP8 operator inputs (OCP microscaling "MX" format).  The SANA-Video 2.0
 * summary (results and limitations) trains with MXFP8 activations for the
 * GEMMs, keeps attention in BF16 and names low-precision attention kernels as
 * future work; these entry points take the operator's q, k, v and g in that
 * activation format.  q, k, v, g: E4M3 codes [batch][N][heads][128], one byte
 * per element (sign, 4 exponent bits with bias 7, 3 mantissa bits; no
 * infinities, S.1111.111 is NaN); q_scale .. g_scale: E8M0 scales
 * [batch][N][heads][4], one byte per 32 consecutive channels (value
 * 2^(byte - 127)).  Element i of a row is e4m3(code_i) * 2^(scale[i / 32] -
 * 127).  beta stays bf16 [batch][N][heads]; out is bf16 [batch][N][heads][128].
 * The operator is gla_forward's, on the decoded values (which bf16 represents
 * exactly).  head_dim 128 only.  All pointers 16-byte aligned device memory. */

/* Workspace bytes of gla_forward_mx_ex for `path` (GLA_PATH_SIMT also holds
 * the inputs decoded to bf16); 0 for invalid sizes. */
GLA_API size_t gla_forward_mx_workspace_size(int batch, int heads, int head_dim, int T, int H,
                                             int W, int path);

/* The bidirectional operator on MX inputs (tensor path: the state reduction
 * and read-out decode the fp8 tiles in their transform warps). */
GLA_API gla_status gla_forward_mx(const void* q, const void* q_scale, const void* k,
                                  const void* k_scale, const void* v, const void* v_scale,
                                  const void* beta, const void* g, const void* g_scale,
                                  int batch, int heads, int head_dim, int T, int H, int W,
                                  float rope_theta, float eps, void* out, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* gla_forward_mx with an explicit path (GLA_PATH_SIMT decodes the inputs to
 * bf16 in the workspace and runs the CUDA-core kernels), the hidden
 * intermediates of gla_forward_debug (S_out, z_out, den_out, x_out, each may
 * be NULL) and the kernel events of gla_forward_timed (`events` may be NULL).
 * GLA_PATH_AUTO falls back to the CUDA-core path where the tensor path does
 * not fit, if the workspace is large enough for it. */
GLA_API gla_status gla_forward_mx_ex(const void* q, const void* q_scale, const void* k,
                                     const void* k_scale, const void* v, const void* v_scale,
                                     const void* beta, const void* g, const void* g_scale,
                                     int batch, int heads, int head_dim, int T, int H, int W,
                                     float rope_theta, float eps, void* out, void* workspace,
                                     size_t workspace_bytes, void* stream, int path,
                                     float* S_out, float* z_out, float* den_out, float* x_out,
                                     void* const* events);

/* ------------------------------------------------------------------------
 * The layer around the operator.  The "Gated Bilinear Linear Attention"
 * prerequisite of the SANA-Video 2.0 summary reads o_j = W_o RMSNorm[...]: the
 * heads' normalised read-outs, concatenated over the heads (width
 * heads*head_dim), times W_o.  The pages print no input projection; here q, k,
 * v, g and the beta logits are one linear map of the layer input x, and beta is
 * the sigmoid of its logits.  All matrices are bf16, row-major, device memory,
 * 16-byte aligned, owned by the caller; products accumulate in fp32 on the
 * tensor cores (tcgen05).  Every call is asynchronous on `stream` and checks
 * its arguments before any launch: GLA_ERR_INVALID_ARG for non-positive or
 * unaligned sizes and null or misaligned pointers, GLA_ERR_UNSUPPORTED for
 * widths the kernels do not take (stated per call), GLA_ERR_WORKSPACE for a
 * short or misaligned workspace, GLA_ERR_CUDA for a failed launch. */

/* C [M][N] = A [M][K] B[N][K]^T, bf16 out (rounded to nearest even).  K and N
 * multiples of 8 (16-byte rows). */
GLA_API gla_status gla_gemm_bf16(const void* A, const void* B, void* C, int M, int N, int K,
                                 void* stream);

/* The input projection with the operator's inputs written straight from the
 * product: x [tokens][C] times W_in [4*heads*head_dim + heads][C]^T, columns
 * [0, HD) to q, [HD, 2HD) to k, then v and g ([tokens][HD] each, HD =
 * heads*head_dim, i.e. the operator's [B][N][heads][head_dim] layout), and
 * the last `heads` columns to beta [tokens][heads] after a sigmoid.  C a
 * multiple of 8, HD a multiple of 32. */
GLA_API gla_status gla_project_in(const void* x, const void* W_in, int tokens, int C, int heads,
                                  int head_dim, void* q, void* k, void* v, void* g, void* beta,
                                  void* stream);

/* Workspace bytes of gla_layer_forward (q, k, v, g, beta, the operator's output
 * and the operator's workspace). */
GLA_API size_t gla_layer_workspace_size(int batch, int heads, int head_dim, int T, int H, int W);

/* y [batch*N][C_out] = W_o applied to gla_forward of the projections of x
 * [batch*N][C]: gla_project_in, gla_forward, gla_gemm_bf16, each kernel a
 * programmatic dependent of the one before.  W_in [4*heads*head_dim +
 * heads][C], W_o [C_out][heads*head_dim]; C and C_out multiples of 8 and
 * heads*head_dim of 32 (GLA_ERR_UNSUPPORTED otherwise); rope_theta and eps as
 * for gla_forward. */
GLA_API gla_status gla_layer_forward(const void* x, const void* W_in, const void* W_o, int batch,
                                     int C, int C_out, int heads, int head_dim, int T, int H,
                                     int W, float rope_theta, float eps, void* y,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * The gated softmax anchor.  The "softmax anchors and hybrid attention"
 * section of the SANA-Video 2.0 summary keeps one full softmax attention
 * layer in four; its anchor layers normalise q and k, rotate them with the
 * same 3D RoPE and gate the read-out with sigmoid(g).  Per head:
 *   q_til = RoPE3D(RMSNorm(q)), k_til = RoPE3D(RMSNorm(k))   (no ReLU here)
 *   o_j   = sigmoid(g_j) * sum_n softmax_n(q_til_j . k_til_n / sqrt(d)) v_n
 * over all N tokens of the call (bidirectional).  RMSNorm has no weight and
 * epsilon 1e-6; q, k, v, g and out are bf16 [batch][N][heads][head_dim]
 * device buffers (16-byte aligned), N = T*H*W in raster order; head_dim 128
 * (GLA_ERR_UNSUPPORTED otherwise); rope_theta <= 0 turns the rotation off.
 * Scores are taken on the tensor cores from fp16 q_til, k_til (fp32
 * accumulate); the exponentials need no shift by the row maximum, because
 * the normalisation bounds every score by sqrt(head_dim); the softmax
 * weights are rounded to bf16 for P*V and the row sums add those rounded
 * weights in fp32.  batch * heads <= 65535.  The caller owns every buffer;
 * the call is asynchronous on `stream`.  Errors: GLA_ERR_INVALID_ARG for bad
 * sizes or pointers, GLA_ERR_UNSUPPORTED for head_dim != 128 or too many
 * heads, GLA_ERR_WORKSPACE for a short or misaligned workspace (256-byte
 * aligned), GLA_ERR_CUDA for a failed launch. */

/* Workspace bytes of gla_softmax_anchor (fp16 q_til and k_til), 0 for
 * unsupported sizes. */
GLA_API size_t gla_softmax_anchor_workspace_size(int batch, int heads, int head_dim, int T, int H,
                                                 int W);

GLA_API gla_status gla_softmax_anchor(const void* q, const void* k, const void* v, const void* g,
                                      int batch, int heads, int head_dim, int T, int H, int W,
                                      float rope_theta, void* out, void* workspace,
                                      size_t workspace_bytes, void* stream);

/* gla_softmax_anchor that also records caller-created CUDA events (cudaEvent_t
 * passed as void*) on `stream`: events[0] before the q/k preparation,
 * events[1] after it, events[2] after the attention kernel.  `events` and any
 * of its entries may be NULL. */
GLA_API gla_status gla_softmax_anchor_timed(const void* q, const void* k, const void* v,
                                            const void* g, int batch, int heads, int head_dim,
                                            int T, int H, int W, float rope_theta, void* out,
                                            void* workspace, size_t workspace_bytes,
                                            void* stream, void* const* events);

/* Bytes of the device arena gla_causal_step_host needs: room for the call's
 * five inputs, its output and its workspace. */
GLA_API size_t gla_causal_host_arena_size(int batch, int heads, int head_dim, int T, int H,
                                          int W, int dtype);

/* gla_causal_step on HOST buffers: q_h .. g_h and out_h are host memory
 * (pinned memory gives asynchronous copies); state and z stay in the caller's
 * DEVICE memory, carried between calls.  Enqueues on `stream` the
 * host-to-device copies of the inputs into the caller's device `arena` (at
 * least gla_causal_host_arena_size() bytes, 256-byte aligned), the step, and
 * the device-to-host copy of the output; returns after enqueueing.  The output
 * equals gla_causal_step's on the same inputs bit for bit. */
GLA_API gla_status gla_causal_step_host(float* state, float* z, const void* q_h, const void* k_h,
                                        const void* v_h, const void* beta_h, const void* g_h,
                                        int batch, int heads, int head_dim, int T, int H, int W,
                                        int t0, float rope_theta, float eps, int dtype,
                                        void* out_h, void* arena, size_t arena_bytes,
                                        void* stream);

/* Bytes of the device arena gla_forward_host needs: room for the five inputs,
 * the output and the workspace. */
GLA_API size_t gla_forward_host_arena_size(int batch, int heads, int head_dim, int T, int H, int W,
                                   int dtype);

/* gla_forward on HOST buffers (q_h .. out_h; pinned memory gives asynchronous
 * copies).  Enqueues on `stream`: host-to-device copies of the inputs into the
 * caller's device `arena`, the operator, and device-to-host copies of the
 * output.  With batch >= 2 the call runs per group of batch elements (at most
 * 8 groups; batch elements are independent): each group's output copy is
 * issued on a helper stream the library owns (one per device, created on the
 * first such call) so that it overlaps the next group's input copies, and the
 * helper is joined back into `stream` before the call's work ends.  Each
 * group is one gla_forward call over its batch elements, so the output equals
 * that of gla_forward on the same groups bit for bit, and a whole-batch
 * gla_forward call within rounding (the split-N partition differs).  Returns
 * after enqueueing; synchronise `stream` before reading out_h.  The arena is
 * caller-owned device memory of at least gla_forward_host_arena_size() bytes,
 * 256-byte aligned.  Not for use inside a CUDA graph capture when batch >= 2
 * (the helper stream is not part of the capture). */
GLA_API gla_status gla_forward_host(const void* q_h, const void* k_h, const void* v_h,
                            const void* beta_h, const void* g_h, int batch, int heads,
                            int head_dim, int T, int H, int W, float rope_theta, float eps,
                            int dtype, void* out_h, void* arena, size_t arena_bytes,
                            void* stream);

/* Bytes of the device arena gla_block_causal_step_host needs: room for one
 * block's five inputs, its output and the step's workspace. */
GLA_API size_t gla_block_causal_host_arena_size(int batch, int heads, int head_dim, int T_blk,
                                                int H, int W, int dtype);

/* gla_block_causal_step on HOST buffers for one block (key design 2 of the
 * SANA-Video notes: each block adds its own terms to the running sums that
 * stay resident on the GPU).  q_h .. g_h and out_h are host memory (pinned
 * memory gives asynchronous copies); state and z are the caller's DEVICE
 * memory, carried between calls as in gla_block_causal_step.  Enqueues on
 * `stream`: host-to-device copies of the block's inputs into the caller's
 * device `arena` (at least gla_block_causal_host_arena_size() bytes, 256-byte
 * aligned), the step, and the device-to-host copy of the block's output.
 * Returns after enqueueing; synchronise `stream` before reading out_h.  The
 * output equals gla_block_causal_step's on the same inputs bit for bit. */
GLA_API gla_status gla_block_causal_step_host(float* state, float* z, const void* q_h,
                                              const void* k_h, const void* v_h,
                                              const void* beta_h, const void* g_h, int batch,
                                              int heads, int head_dim, int T_blk, int H, int W,
                                              int t0, float rope_theta, float eps, int dtype,
                                              void* out_h, void* arena, size_t arena_bytes,
                                              void* stream);

/* Size of the scratch array built into the library for gla_forward_noalloc. */
#define GLA_NOALLOC_SCRATCH_BYTES (24u << 20)

/* gla_forward for callers that cannot allocate device memory: code running
 * where cudaMalloc is unavailable or forbidden (inside a memory-pool-managed
 * runtime that owns every allocation, in a plugin that must not grow the
 * process footprint at call time, or on a path that may not synchronise the
 * device, which cudaMalloc can do).  The operator's scratch space (split-N
 * partial states, the combined state, its fp16 image and the RoPE table)
 * comes from one
 * array of GLA_NOALLOC_SCRATCH_BYTES compiled into this library; every GPU
 * that loads the library holds that array until the process exits.  The
 * caller still passes the inputs and `out`.  No counterpart on the pages: it
 * is a packaging choice of this library.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  Every call shares the one array and leaves its contents behind:
 * calls whose kernels overlap on the GPU (different streams, or different
 * host threads on the same device without ordering) race on it and give
 * wrong results, so order them on one stream.  Nothing in the array needs to
 * start at zero.  Problems whose scratch would exceed the array return
 * GLA_ERR_WORKSPACE with nothing launched; it allocates nothing, ever. */
GLA_API gla_status gla_forward_noalloc(const void* q, const void* k, const void* v,
                                       const void* beta, const void* g, int batch, int heads,
                                       int head_dim, int T, int H, int W, float rope_theta,
                                       float eps, int dtype, void* out, void* stream);

/* Synchronises `stream`, then reports and clears the library's device error
 * word: GLA_ERR_TIMEOUT if a kernel gave up a bounded wait since the last
 * call, GLA_ERR_CUDA if the synchronisation itself failed, else GLA_OK. */
GLA_API gla_status gla_get_device_status(void* stream);

/* Self-test of the failure-detection path.  Launches one CTA on `stream` whose
 * threads wait on an mbarrier that nothing arrives on, through the same
 * bounded wait every pipeline stage of the library uses, but with a limit of
 * `limit_us` microseconds (1 .. 1000000) instead of the pipelines' 2 s.  The
 * wait gives up, records the timeout in the device error word as a stalled
 * pipeline would, and the kernel returns; nothing faults or hangs.  A later
 * gla_get_device_status() reports GLA_ERR_TIMEOUT and clears it.  Returns
 * GLA_ERR_INVALID_ARG for a limit outside that range (nothing launched),
 * GLA_ERR_CUDA if the launch fails, else GLA_OK. */
GLA_API gla_status gla_selftest_wait_timeout(unsigned int limit_us, void* stream);

/* Self-test of the tensor pipelines' abort path (tests only; no fault, no
 * hang).  Runs gla_forward on the tensor path (bf16, head_dim 128; arguments
 * as gla_forward) with two changes in the state-reduction kernel: every
 * pipeline wait gives up after `limit_us` microseconds (1 .. 1000000) instead
 * of 2 s, and the producer of CTA 0 withholds the arrival that announces its
 * first tile.  The transform warps' wait for that tile runs out: the kernel
 * records GLA_ERR_TIMEOUT in the device error word, raises its abort flag, and
 * every role leaves its loop, lets its copies and MMAs in flight complete,
 * frees TMEM and returns; the rest of the call runs to completion on the
 * partial sums it has.  `out` then holds no meaningful result, a later
 * gla_get_device_status() reports GLA_ERR_TIMEOUT (and clears it), and the
 * next call computes normally.  Returns GLA_ERR_INVALID_ARG for a limit out
 * of range, GLA_ERR_UNSUPPORTED where the tensor path does not apply. */
GLA_API gla_status gla_selftest_pipeline_stall(const void* q, const void* k, const void* v,
                                               const void* beta, const void* g, int batch,
                                               int heads, int head_dim, int T, int H, int W,
                                               float rope_theta, float eps, void* out,
                                               void* workspace, size_t workspace_bytes,
                                               unsigned int limit_us, void* stream);

/* Host-only self-check of the tensor read-out's RoPE table copies (tests; no
 * GPU needed): for every read-out CTA of this problem on num_sms SMs, the bulk
 * copies that bring its table window from the whole-call table are 16-byte
 * aligned, stay inside both tables and the CTA's shared-memory table, and
 * bring every entry the CTA looks up from the whole-call entry of the same
 * rotation pair and absolute position.  GLA_OK, GLA_ERR_UNSUPPORTED (no
 * tensor path for this head dim) or GLA_ERR_INVALID_ARG (bad sizes, or a
 * violated check). */
GLA_API gla_status gla_check_rope_copy(int batch, int heads, int head_dim, int T, int H, int W,
                                       int num_sms);

/* Host-only planning query (no GPU needed): the grid of the state-reduction
 * kernel and the tokens per tile for this problem on a GPU with `num_sms`
 * SMs and the given path.  Returns GLA_OK and fills *grid, *tile_tokens,
 * *path_used; used by tests to check the split-N partition. */
GLA_API gla_status gla_plan(int batch, int heads, int head_dim, int T, int H, int W, int dtype,
                    int path, int num_sms, int* grid, int* tile_tokens, int* path_used);

#ifdef __cplusplus
}
#endif

#endif /* GLA_H */
