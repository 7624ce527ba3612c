/*
 * h3b -- C ABI of a B200 (sm_100a) engine for the forward pass of a dense
 * single-stream diffusion-transformer (DiT) block over a joint video + audio
 * token sequence, its stack with mid-stack token reduction, the INT8 W8A8
 * variant, and the flow-matching Euler update with whole-velocity reuse.
 *
 * Sources (MiniMax H3 / h3.c web pages):
 *   [model]   "MiniMax H3: video and audio generated together" (mobbang.com,
 *             model section): a dense single-stream omni transformer; every
 *             frame and the audio track are denoised at once.
 *   [fusion]  "h3.c MiniMax H3 inference engine for Mac" (jdon.com,
 *             33B-parameter section): fused kernels, activation-arena reuse,
 *             token reduction by pairing adjacent video tokens.
 *   [arena]   "antirez/h3.c" (siami.tw, memory-strategy section): the QKV
 *             arena serves the attention heads and then the normalised MLP
 *             input; the attention-output arena becomes the MLP output.
 *   [control] same page, speed/quality control table: whole-denoiser reuse
 *             (20/11/8 fresh evaluations for reuse 1/2/3 at 20 steps) and
 *             token reduction in the middle blocks.
 *   [int8]    same page, data section, and the 21cto.com page's M5 Max
 *             section: INT8 MLP, QKV and attention-output GEMMs; jdon.com
 *             speed/quality section: INT8 FC2 with one activation scale per
 *             row.
 * The block's internals (RMSNorm eps 1e-6, 3D/1D RoPE, exact-erf GELU, head
 * sizes) follow the workload specification; the pages do not give them.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller and must be
 *     16-byte aligned.  Layouts are row-major; one token is one row.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call only enqueues work on that stream: it does not
 *     synchronise and does not allocate device memory.  Scratch space is the
 *     caller's workspace.
 *   - Return value: H3B_OK (0) or a negative H3B_ERR_* code.  Argument errors
 *     are detected on the host before anything is enqueued.  H3B_ERR_CUDA
 *     reports a failed CUDA call (e.g. a launch error from
 *     cudaGetLastError right after a launch); faults that happen later on the
 *     device are not converted.  Bounded device-side waits that give up set a
 *     device error word readable with h3b_device_error().
 *   - The token sequence holds the video grid F x H x W in the order
 *     (f*H + r)*W + c, followed by the A audio tokens.  After token reduction
 *     the grid is F x H x W/2, the merged video index is (f*H + r)*(W/2) + c',
 *     and the audio tokens follow.
 */
#ifndef H3B_H
#define H3B_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status */
#define H3B_OK              0
#define H3B_ERR_NULL       -1  /* a required pointer is NULL                 */
#define H3B_ERR_ALIGN      -2  /* a pointer is not 16-byte aligned           */
#define H3B_ERR_DIMS       -3  /* unsupported or inconsistent sizes          */
#define H3B_ERR_DTYPE      -4  /* unknown dtype / epilogue code              */
#define H3B_ERR_WORKSPACE  -5  /* workspace smaller than required            */
#define H3B_ERR_CUDA       -6  /* a CUDA runtime/driver call failed          */
#define H3B_ERR_DEVICE     -7  /* no usable sm_100 device                    */
#define H3B_ERR_TIMEOUT    -8  /* a bounded device-side wait gave up         */

/* weight dtypes */
#define H3B_BF16 0
#define H3B_INT8 1

/* Sizes of one DiT block.  d = n_heads * head_dim; head_dim is 64 or 128;
 * ffn a multiple of 128 (4 * d in the workloads); d a multiple of 128; eps the RMSNorm epsilon
 * (1e-6 in the workloads), rope_theta the RoPE base (10000). */
typedef struct h3b_dims {
  int frames, rows, cols, n_audio;   /* video grid F x H x W, audio tokens A */
  int d, n_heads, head_dim, ffn;
  float eps, rope_theta;
} h3b_dims;

/* Weights of one block, all device pointers.
 *   BF16: w_* are bf16 [out, in] row-major: w_qkv [3d, d] (rows = Q heads,
 *         then K heads, then V heads, head_dim rows each), w_o [d, d],
 *         w_fc1 [ffn, d], w_fc2 [d, ffn]; s_* unused (may be NULL).
 *   INT8: w_* are int8 [out, in] with per-output-channel fp32 scales s_*
 *         (as written by h3b_quantize_weights).
 *   g_attn, g_mlp: fp32 [d] RMSNorm gains. */
typedef struct h3b_block_weights {
  int dtype;
  const void *w_qkv, *w_o, *w_fc1, *w_fc2;
  const float *s_qkv, *s_o, *s_fc1, *s_fc2;
  const float *g_attn, *g_mlp;
} h3b_block_weights;

/* Human-readable text of a status code (static storage). */
const char* h3b_status_string(int status);

/* Number of tokens: S = F*H*W + A, or F*H*(W/2) + A when merged != 0. */
int h3b_seq_len(const h3b_dims* dims, int merged);

/* Workspace bytes needed by h3b_block_forward, h3b_stack_forward and
 * h3b_denoise for these dims and dtype.  `token_reduction` != 0 adds the
 * merged-sequence buffer and the second RoPE table.  The activation arenas
 * inside are aliased across the block's lifetime: the QKV arena is reused
 * for the normalised MLP input, and the FC1 hidden overlays the dead QKV,
 * attention-output and norm arenas [arena].  Returns 0 for invalid dims. */
size_t h3b_workspace_bytes(const h3b_dims* dims, int dtype, int token_reduction);

/* Bytes the arena aliasing saves against one buffer per intermediate. */
size_t h3b_workspace_saved_bytes(const h3b_dims* dims, int dtype);

/* One DiT block, in place on the fp32 residual stream x [S, d]
 * (S from h3b_seq_len(dims, merged)) [model]:
 *   u  = RMSNorm(x; g_attn)                 (norm kernel -> bf16 / int8+scale)
 *   qkv = u W_qkv^T, RoPE on Q and K        (GEMM, RoPE fused in the epilogue)
 *   o  = softmax(q k^T / sqrt(head_dim)) v  (flash attention, all S keys)
 *   x += o W_o^T                            (GEMM, residual in the epilogue)
 *   x += GELU(RMSNorm(x; g_mlp) W_fc1^T) W_fc2^T  (GEMMs, GELU / residual
 *                                             fused in the epilogues)
 * INT8 weights use per-token dynamic activation quantisation at each GEMM
 * input and int32 accumulation [int8].  `merged` selects the reduced
 * geometry for positions (merged token c' sits at column 2c'+0.5).
 * ws: device workspace of at least h3b_workspace_bytes(dims, dtype, 0). */
int h3b_block_forward(const h3b_dims* dims, const h3b_block_weights* w, float* x, int merged,
                      void* ws, size_t ws_bytes, void* stream);

/* Blocks 0..n_blocks-1 in order on x [S, d] fp32 in place.  When
 * merge_first >= 0, the sequence is merged (h3b_token_merge) before block
 * merge_first and unmerged after block merge_last (inclusive, 0-indexed)
 * [control].  ws: at least h3b_workspace_bytes(dims, dtype, merge_first >= 0).
 * All blocks must share one dtype.  Between consecutive bf16 blocks outside
 * the reduction window's edges, RMSNorm is folded into the neighbouring
 * GEMMs (the residual epilogue writes bf16(x * g) and per-row sums of x^2,
 * the next GEMM scales its rows by 1/sqrt(mean x^2 + eps)) [fusion]; the
 * result then equals a sequence of h3b_block_forward calls within rounding
 * (the bf16 rounding falls on x * g instead of on the normalised row), not
 * bit for bit.  INT8 stacks match the block sequence bit for bit. */
int h3b_stack_forward(const h3b_dims* dims, const h3b_block_weights* blocks, int n_blocks,
                      int merge_first, int merge_last, float* x,
                      void* ws, size_t ws_bytes, void* stream);

/* Flow-matching denoising loop with whole-velocity reuse [control]:
 * sigma_i = 1 - i/n_steps; step i is fresh iff i % reuse == 0 or
 * i == n_steps-1; on a fresh step v = stack(x) (copy of x run through
 * h3b_stack_forward), otherwise the last fresh v is reused; then
 * x <- x + (sigma_{i+1} - sigma_i) v.
 * x: latent [S, d] fp32, in/out.  v: caller buffer [S, d] fp32 that holds
 * the evaluation input and then the velocity.  n_fresh (host, may be NULL)
 * receives the number of fresh evaluations. */
int h3b_denoise(const h3b_dims* dims, const h3b_block_weights* blocks, int n_blocks,
                int merge_first, int merge_last, int n_steps, int reuse,
                float* x, float* v, void* ws, size_t ws_bytes, int* n_fresh, void* stream);

/* Options of the extended stack / loop entry points: a delta-broadcast
 * unmerge, core residual reuse, fixed condition rows and timestep
 * modulation.  The siami.tw article's control table names the core-reuse knob
 * (--core-reuse 1/4/6, exclusive with whole-velocity reuse) but not its
 * arithmetic, its file list names a 0.999 condition augmentation and fixed
 * condition rows without a form, and no page gives an unmerge rule; the
 * forms below are the plainest readings.  Zero-initialise the struct: every
 * field's zero (with merge_first = core_first = -1) is "off".
 *   merge_first, merge_last: token-reduction window (inclusive, 0-indexed),
 *     merge_first = -1 turns it off.
 *   unmerge_delta: 0 = broadcast each merged token back to both columns;
 *     1 = pre-merge tokens plus the merged blocks' update broadcast:
 *     x(f,r,c) = x_pre(f,r,c) + (y - m)(f,r,c/2); the rows after the
 *     video rows (audio, condition) take y.
 *   core_first, core_last: core window for h3b_denoise_ex (-1 = off); the
 *     reduction window must lie inside it or outside it.  Ignored by
 *     h3b_stack_forward_ex.
 *   n_cond: condition rows appended after the audio tokens (0 = none).  They
 *     take part in every block (joint attention) without rotary embedding.
 *     h3b_stack_forward_ex: x is [S + n_cond, d] (S = h3b_seq_len).
 *     h3b_denoise_ex: x is [S, d] (the generated rows), v is [S + n_cond, d],
 *     and cond_rows [n_cond, d] fp32 (device, 16-byte aligned; already
 *     augmented) are copied into v before every evaluation; the Euler update
 *     covers the S generated rows only.
 *   modulation (NULL = none): fp32 device array, 16-byte aligned, of
 *     mod_steps slices of [n_blocks][2][6][d]: per block, per row class
 *     (0 = generated rows, 1 = condition rows), the vectors shift_attn,
 *     scale_attn, gate_attn, shift_mlp, scale_mlp, gate_mlp.  The block becomes
 *       u  = RMSNorm(x) * (1 + scale_attn) + shift_attn  (QKV GEMM input)
 *       x += gate_attn * (O-proj output)
 *       u2 = RMSNorm(x) * (1 + scale_mlp) + shift_mlp    (FC1 GEMM input)
 *       x += gate_mlp * (FC2 output).
 *     h3b_stack_forward_ex reads slice 0; h3b_denoise_ex reads slice i at
 *     step i when mod_steps == n_steps, slice 0 at every step when it is 1
 *     (any other value: H3B_ERR_DIMS). */
typedef struct h3b_stack_opts {
  int merge_first, merge_last;
  int unmerge_delta;
  int core_first, core_last;
  int n_cond;
  int mod_steps;
  const float* cond_rows;
  const float* modulation;
} h3b_stack_opts;

/* Workspace bytes for the extended entry points (sized for S + n_cond rows;
 * adds the saved merged input for unmerge_delta and the cached core update
 * [S + n_cond, d] fp32 for core reuse). */
size_t h3b_workspace_bytes_ex(const h3b_dims* dims, int dtype, const h3b_stack_opts* opts);

/* h3b_stack_forward with the options above. */
int h3b_stack_forward_ex(const h3b_dims* dims, const h3b_block_weights* blocks, int n_blocks,
                         const h3b_stack_opts* opts, float* x, void* ws, size_t ws_bytes, void* stream);

/* h3b_denoise with the options above and core residual reuse: with
 * core_first >= 0 (then reuse must be 1) every step evaluates the stack, but
 * the core blocks run only on steps i with i % core_reuse == 0 or
 * i == n_steps-1, where their update (core output - core input) is cached in
 * the workspace; on the other steps that update is added instead of running
 * them.  n_fresh / n_core_fresh (host, may be NULL) receive the numbers of
 * stack evaluations and of core evaluations. */
int h3b_denoise_ex(const h3b_dims* dims, const h3b_block_weights* blocks, int n_blocks,
                   const h3b_stack_opts* opts, int n_steps, int reuse, int core_reuse, float* x, float* v,
                   void* ws, size_t ws_bytes, int* n_fresh, int* n_core_fresh, void* stream);

/* Per-row symmetric int8 quantisation [int8]: s[r] = max_k |w[r,k]| / 127
 * (fp32), q[r,k] = rint(w[r,k] / s[r]) (IEEE fp32 divide, half-even),
 * clamped to [-127, 127]; an all-zero row gives s = 0, q = 0.
 * w: bf16 [rows, k]; q: int8 [rows, k]; scale: fp32 [rows].  Used once per
 * weight matrix (per output channel) and, inside the block, per token on
 * activations.  k must be a multiple of 8.  rows == 0 launches nothing (the
 * pointers may then be NULL; k is still checked). */
int h3b_quantize_weights(const void* w, int rows, int k, int8_t* q, float* scale, void* stream);

/* Token reduction [fusion], [control]: xm[(f*H+r)*(W/2)+c'] =
 * (x[(f*H+r)*W+2c'] + x[(f*H+r)*W+2c'+1]) * 0.5 in fp32; audio rows are
 * copied.  x: fp32 [S, d]; xm: fp32 [S', d]; W must be even. */
int h3b_token_merge(const h3b_dims* dims, const float* x, float* xm, void* stream);

/* Inverse broadcast: x[(f*H+r)*W+c] = xm[(f*H+r)*(W/2)+c/2]; audio rows
 * copied.  xm: fp32 [S', d]; x: fp32 [S, d]. */
int h3b_token_unmerge(const h3b_dims* dims, const float* xm, float* x, void* stream);

/* Delta-broadcast unmerge, the unit form of h3b_stack_opts.unmerge_delta
 * [control]: x holds the pre-merge tokens [S, d] fp32 and is updated in
 * place, video row (f*H+r)*W + c += ym[m] - xm0[m] with
 * m = (f*H+r)*(W/2) + c/2 (one fp32 subtraction, then one fp32 addition);
 * the audio rows take ym's rows after the merged video rows.  ym: what the
 * merged blocks returned, xm0: what entered them, both fp32 [S', d] with
 * S' = h3b_seq_len(dims, 1).  W must be even. */
int h3b_token_unmerge_delta(const h3b_dims* dims, float* x, const float* ym, const float* xm0, void* stream);

/* Euler update x[i] <- x[i] + (sigma_next - sigma_cur) * v[i] for i < n
 * (fp32, fused multiply-add); when x_copy is not NULL the updated value is
 * also written to x_copy[i] (the next fresh evaluation's input) [control].
 * n == 0 is a no-op (the pointers may then be NULL). */
int h3b_flow_step(float* x, const float* v, float sigma_cur, float sigma_next, size_t n,
                  float* x_copy, void* stream);

/* Allocation-free block forward (no counterpart on the pages; added for
 * callers that may not allocate device memory -- e.g. code hosted in an
 * application that owns and accounts for all device memory through its own
 * pool, or a latency-critical thread that must not call cudaMalloc, which can
 * synchronise the device).  Same computation, arguments and results as
 * h3b_block_forward, without the workspace: the scratch is a fixed array of
 * H3B_NOALLOC_MAX_BYTES inside the library's device image, held on every GPU
 * that loads the library until the process exits.
 *   - Sizes whose workspace (h3b_workspace_bytes(dims, dtype, 0)) exceeds
 *     H3B_NOALLOC_MAX_BYTES are rejected with H3B_ERR_WORKSPACE; nothing is
 *     enqueued.  32 MiB covers e.g. d = 256 at S = 288 and d = 1024 at
 *     S ~ 3000 tokens.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.  The address is kept for the life of the
 *     process: after cudaDeviceReset on a device it is stale, and this entry
 *     point (like the rest of the library) must not be called on that device
 *     again.
 *   - Calls allocate nothing (no cudaMalloc/cudaFree, no allocating library
 *     routine).
 *   - Every call shares the one array per device, which keeps the previous
 *     call's contents; what must start at zero is cleared inside each call.
 *     Calls whose work overlaps on the GPU (other streams, other host
 *     threads) race on that array: order them on one stream. */
#define H3B_NOALLOC_MAX_BYTES (32u << 20)
int h3b_block_forward_noalloc(const h3b_dims* dims, const h3b_block_weights* w, float* x, int merged,
                              void* stream);

/* ---------------------------------------------------------------------------
 * Unit-level entry points: the individual kernels the block is made of, for
 * kernel-by-kernel parity tests and timing.  Same conventions as above.
 * ------------------------------------------------------------------------- */

/* RoPE table of the (merged) geometry: float2 [S', head_dim/2] holding
 * (cos, sin) of p * theta^(-2j/n) for pair j of the section of width n that
 * carries position p.  Video head dims split [frame D/4 | row 3D/8 |
 * col 3D/8]; audio tokens use one section of width D at position a. */
int h3b_rope_table(const h3b_dims* dims, int merged, float* table, void* stream);

/* RMSNorm of x fp32 [rows, d]: u = x * rsqrt(mean(x^2) + eps) * g.
 * out_dtype H3B_BF16: out is bf16 [rows, d], out_scale unused.
 * out_dtype H3B_INT8: out is int8 [rows, d] quantised per row (rule of
 * h3b_quantize_weights applied to the fp32 u) with scales in out_scale.
 * rows == 0 launches nothing (the pointers may then be NULL). */
int h3b_rmsnorm(const float* x, const float* g, int rows, int d, float eps,
                void* out, float* out_scale, int out_dtype, void* stream);

/* GEMM epilogues (C = A B^T, A [M,K], B [N,K], both K-major). */
#define H3B_EPI_F32       0  /* C fp32 [M,N]  = acc                            */
#define H3B_EPI_BF16      1  /* C bf16 [M,N]  = acc                            */
#define H3B_EPI_QKV_ROPE  2  /* C bf16 [M,N]  = acc, RoPE on columns < 2*d     */
#define H3B_EPI_RESID     3  /* C fp32 [M,N] += acc (residual add, in place)   */
#define H3B_EPI_GELU      4  /* C bf16 [M,N]  = GELU(acc); INT8: also row |max| */
#define H3B_EPI_I32       5  /* C int32 [M,N] = raw integer accumulator (INT8)  */

/* Tensor-core GEMM.  ab_dtype H3B_BF16: A, B bf16, fp32 accumulate;
 * H3B_INT8: A, B int8, int32 accumulate, and (except H3B_EPI_I32) the
 * accumulator is dequantised as float(acc) * scale_a[m] * scale_b[n] before
 * the epilogue.  K must be a multiple of 64 (bf16) / 128 (int8), N a
 * multiple of 32.  H3B_EPI_QKV_ROPE needs rope_table (h3b_rope_table of the
 * same sequence) and dims (for d, head_dim).  H3B_EPI_GELU with INT8 needs
 * row_absmax fp32 [M], zeroed by the caller, which receives max |GELU| of
 * each row (after bf16 rounding).  scratch (optional, device, scratch_bytes
 * long): with H3B_EPI_RESID, when the last wave of output tiles would leave
 * most SMs idle, those tail tiles are split along K over the idle SMs; their
 * fp32 partials go to scratch (up to 148 tiles x 128 KB) and are added into C
 * in a fixed order by a second kernel (deterministic).  NULL disables it.
 * M == 0 launches nothing (A and C may then be NULL; the other arguments are
 * still checked). */
int h3b_gemm(const void* A, const void* B, int M, int N, int K, int ab_dtype, int epilogue,
             void* C, const float* scale_a, const float* scale_b, const float* rope_table,
             const h3b_dims* dims, float* row_absmax, void* scratch, size_t scratch_bytes,
             void* stream);

/* Quantise bf16 rows with a known max |row| (e.g. from H3B_EPI_GELU):
 * s[r] = absmax[r] / 127, q = rint(a / s) clamped, as h3b_quantize_weights.
 * rows == 0 launches nothing (the pointers may then be NULL). */
int h3b_quantize_rows_absmax(const void* a, const float* absmax, int rows, int k,
                             int8_t* q, float* scale, void* stream);

/* Bidirectional attention over the whole sequence, per head:
 * o = softmax(q k^T / sqrt(head_dim)) v.  qkv: bf16 [S, 3*n_heads*head_dim]
 * (Q heads, then K heads, then V heads); o: bf16 [S, n_heads*head_dim].
 * scratch (optional, device): when the work items (256 query rows x head)
 * leave a last wave at most half full, those items are split along the keys
 * over the idle SMs; each part writes its unnormalised O, running max and sum
 * to scratch (up to 148 x 130 KB) and a second kernel merges the parts in a
 * fixed order.  NULL disables it.  S == 0 launches nothing (qkv and o may
 * then be NULL). */
int h3b_attention(const void* qkv, int S, int n_heads, int head_dim, void* o, void* scratch,
                  size_t scratch_bytes, void* stream);

/* The FMA-pipe exp2 that the attention kernel can take for a share of its key
 * pairs (a compile-time option, off by default: on B200 it slowed the kernel):
 * y = 2^n * p(x - n), n = rint(x), p a degree-3 polynomial fitted to 2^f on
 * [-1/2, 1/2] (max relative error 7.5e-5); x is clamped to >= -126.
 * x, y: fp32 [n] device buffers.  For accuracy tests of that approximation. */
int h3b_exp2_poly(const float* x, float* y, int n, void* stream);

/* The FC1 epilogue's GELU, y[i] = x[i] * Phi(x[i]) in fp32 for i < n, for
 * accuracy tests: Phi from the complementary error function of Abramowitz &
 * Stegun formula 7.1.26 (absolute error <= 1.5e-7), never forming 1 + erf on
 * the negative side.  x, y: fp32 device buffers (any alignment); n == 0 is a
 * no-op. */
int h3b_gelu(const float* x, float* y, size_t n, void* stream);

/* ---------------------------------------------------------------------------
 * Device error word and tracing
 * ------------------------------------------------------------------------- */

/* Failure-path self-test: one small kernel waits, with a limit of
 * timeout_us microseconds (1..1000000), on an mbarrier that nothing
 * completes.  The bounded wait gives up, records code (3 << 8) | 1 in the
 * device error word and the kernel exits normally; the context stays usable.
 * Read the code with h3b_device_error. */
int h3b_selftest_wait_timeout(int timeout_us, void* stream);

/* Index-checked build.  libh3b_check.so is the same library compiled with
 * -DH3B_CHECK=1: every hand-indexed global load and store first checks its
 * element range against the extent of its buffer as the kernel's own shape
 * arguments define it (rows x columns of a GEMM output, tokens x width of a
 * norm, the caller's scratch bytes for split partials).  A range outside the
 * extent records (4 << 8) | site in the device error word (the first record
 * wins) and the access is skipped: no trap, no fault.  TMA tile loads are
 * bounded by their tensor maps and are not checked.  h3b_index_checked
 * returns 1 in that build and 0 in the default one.
 * h3b_selftest_index_check(i, n) runs one thread that passes index i of
 * extent n (n > 0) through the same check without touching memory: in the
 * checked build an i outside [0, n) records (4 << 8) | 99; the default build
 * records nothing. */
int h3b_index_checked(void);
int h3b_selftest_index_check(long long i, long long n, void* stream);

/* Reads and clears the device error word of the current device
 * (synchronises the stream).  0 = no error; otherwise a code naming the
 * kernel and wait that gave up. */
int h3b_device_error(void* stream);

/* Per-launch tracing: while enabled, every kernel the library launches is
 * bracketed by CUDA events on its stream.  h3b_trace_start(capacity) clears
 * the record; h3b_trace_stop() synchronises and makes the records readable
 * with h3b_trace_read (kernel ids, milliseconds).  Kernel ids name kernels
 * through h3b_kernel_name. */
int h3b_trace_start(int capacity);
int h3b_trace_stop(int* n_records);
int h3b_trace_read(int* kernel_ids, float* ms, int max_records);
const char* h3b_kernel_name(int kernel_id);

#ifdef __cplusplus
}
#endif
#endif /* H3B_H */
