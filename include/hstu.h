/*
 * hstu.h -- C ABI of libhstu: HSTU jagged causal pointwise attention and the
 * HSTU layer forward on NVIDIA B200 (sm_100a).
 *
 * The operation (HSTU, "Actions Speak Louder than Words: Trillion-Parameter
 * Sequential Transducers for Generative Recommendations", arXiv 2402.17152,
 * abstract; the generative-recommenders README, sections "Efficiency
 * experiments" and "HSTU Ultra attention benchmark", for the layer order):
 * a batch of B user-action sequences is packed back to back ("jagged") into
 * T = seq_offsets[B] tokens. For sequence b with tokens o = seq_offsets[b] ..
 * seq_offsets[b+1]-1, head h and positions j <= i inside the sequence:
 *
 *   s_ij = <q[o+i,h,:], k[o+j,h,:]>
 *        + pos_bias[h][min(i-j, num_pos-1)]
 *        + time_bias[h][clamp(floor(log2(max(1, ts[o+i]-ts[o+j]))), 0, NB-1)]
 *   out[o+i,h,:] = (1/max_seqlen) * sum_{j<=i} silu(s_ij) * v[o+j,h,:]
 *
 * with silu(x) = x * sigmoid(x). No softmax, no 1/sqrt(d) score scale.
 * Sections below: the attention; the layer around it (projections, the
 * input and output LayerNorms, the whole layer); row-wise E4M3 (FP8)
 * projections; the attention backward (bf16 on tensor cores, and fp32).
 *
 * Conventions for every entry point:
 *  - Pointers marked "device" must be device memory of the current CUDA device
 *    (or managed memory); they are owned by the caller, and the library keeps
 *    no reference after the call returns. The library never allocates: scratch
 *    lives in a caller-provided workspace sized by the *_workspace_bytes query.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every call is asynchronous on that stream and never synchronises, except
 *    hstu_device_status(). Calls may be captured in a CUDA graph.
 *  - Argument errors are detected on the host before anything is launched and
 *    return HSTU_ERR_INVALID_ARG or HSTU_ERR_UNSUPPORTED. A failed launch
 *    returns HSTU_ERR_CUDA. Conditions only visible on the device (a sequence
 *    longer than max_seqlen, decreasing offsets, a pipeline wait that ran out)
 *    set a per-device error word that hstu_device_status() reports; outputs
 *    are then unspecified.
 *  - Token strides are in elements. bf16 tensors need 16-byte aligned bases and
 *    token strides that are multiples of 8 elements.
 */
#ifndef HSTU_H_
#define HSTU_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HSTU_ABI_VERSION 2

typedef enum hstu_status {
    HSTU_OK = 0,
    HSTU_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad stride or alignment */
    HSTU_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels implement */
    HSTU_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    HSTU_ERR_TIMEOUT = 4,       /* device: a bounded pipeline wait ran out */
    HSTU_ERR_BAD_INPUT = 5      /* device: offsets decrease or a sequence exceeds max_seqlen */
} hstu_status_t;

typedef enum hstu_dtype {
    HSTU_DTYPE_F32 = 0,         /* fp32 in/out, fp32 arithmetic on CUDA cores */
    HSTU_DTYPE_BF16 = 1         /* bf16 in/out, fp32 accumulation on tcgen05 tensor cores */
} hstu_dtype_t;

typedef enum hstu_epilogue {
    HSTU_EPI_NONE = 0,          /* y = x W^T + b                */
    HSTU_EPI_SILU = 1,          /* y = silu(x W^T + b)          */
    HSTU_EPI_RESIDUAL = 2       /* y = r + x W^T + b            */
} hstu_epilogue_t;

int32_t hstu_abi_version(void);
const char* hstu_status_string(hstu_status_t status);

/* Synchronises `stream`, then returns and clears the device error word of the
 * current device: HSTU_ERR_TIMEOUT, HSTU_ERR_BAD_INPUT, HSTU_ERR_CUDA if the
 * synchronisation itself failed, else HSTU_OK. */
hstu_status_t hstu_device_status(void* stream);

/* ---------------------------------------------------------------- attention */

/* Workspace bytes that hstu_attn_plan + hstu_attn_run (or hstu_attn_fwd)
 * need for a batch of B sequences, total_tokens tokens, the given
 * max_seqlen, H heads and a position table of num_pos entries per head
 * (pass the same num_pos as the run, or 1 when it has no position term; bf16
 * path, the fp32 path needs none). Layout:
 *  - the plan's part: a 256-byte header and 32 bytes per work unit (its
 *    descriptor and the sequence-start mask of a packed tile; at most
 *    U = min(total_tokens/128 + B + 1, B * ceil(max_seqlen/128)) units, each
 *    array rounded up to 256 bytes);
 *  - the run's bias tables: 3968 bytes per head and distinct 128-token
 *    diagonal offset of the position window (min(ceil(max_seqlen/128),
 *    ceil((num_pos + 126)/128) + 1) offsets), and 576 bytes per unit for the
 *    key-timestamp summary of its tile.
 * hstu_attn_plan needs only the plan's part. Returns 0 for invalid sizes. */
size_t hstu_attn_workspace_bytes(int32_t B, int64_t total_tokens, int32_t max_seqlen, int32_t H,
                                 int32_t num_pos);

/* Builds the work list of the bf16 attention in `workspace` (device):
 * one entry per (sequence, 128-query tile), ordered longest-first (a query
 * tile t of a sequence needs t+1 key tiles under the causal mask, so tiles are
 * listed by descending t). Reads seq_offsets (device, int64 [B+1], offsets[0]
 * = 0, non-decreasing, offsets[B] = total_tokens). max_seqlen >= every
 * sequence length, 1 <= max_seqlen <= 131072. One kernel launch. */
hstu_status_t hstu_attn_plan(const int64_t* seq_offsets, int32_t B, int64_t total_tokens,
                             int32_t max_seqlen, void* workspace, size_t workspace_bytes,
                             void* stream);

/* Runs the attention for a batch planned by hstu_attn_plan with the same
 * seq_offsets, B, total_tokens and max_seqlen (bf16 path), or directly (fp32
 * path, workspace ignored).
 *   q, k : device [T, H, d_qk] of `dtype`, token strides q_tok_stride,
 *          k_tok_stride (head stride is d_qk: heads are contiguous in a token)
 *   v    : device [T, H, d_v], token stride v_tok_stride
 *   timestamps : device int64 [T], or NULL to drop the time-bucket term
 *   pos_bias   : device fp32 [H, num_pos], or NULL to drop the position term
 *   time_bias  : device fp32 [H, num_time_buckets] (1..1024 buckets), or NULL
 *   max_seqlen : N of the 1/N scale
 *   out  : device [T, H, d_v] of `dtype`, token stride out_tok_stride; every row
 *          of every sequence is written, nothing else is touched
 *   workspace : the plan's workspace, hstu_attn_workspace_bytes(B, total_tokens,
 *          max_seqlen, H, num_pos or 1) bytes; the run reads the plan's part
 *          and rewrites the bias tables behind it (two launches: the tables,
 *          then the attention)
 * Supported: bf16 with d_qk == d_v in {32, 64, 128} (d = 32 is staged as
 * 64-column tiles); fp32 with d_qk, d_v <= 128. */
hstu_status_t hstu_attn_run(hstu_dtype_t dtype,
                            const void* q, int64_t q_tok_stride,
                            const void* k, int64_t k_tok_stride,
                            const void* v, int64_t v_tok_stride,
                            const int64_t* seq_offsets, int32_t B, int64_t total_tokens,
                            int32_t H, int32_t d_qk, int32_t d_v,
                            const int64_t* timestamps,
                            const float* pos_bias, int32_t num_pos,
                            const float* time_bias, int32_t num_time_buckets,
                            int32_t max_seqlen,
                            void* out, int64_t out_tok_stride,
                            void* workspace, size_t workspace_bytes, void* stream);

/* hstu_attn_plan followed by hstu_attn_run (three launches for bf16, one for fp32). */
hstu_status_t hstu_attn_fwd(hstu_dtype_t dtype,
                            const void* q, int64_t q_tok_stride,
                            const void* k, int64_t k_tok_stride,
                            const void* v, int64_t v_tok_stride,
                            const int64_t* seq_offsets, int32_t B, int64_t total_tokens,
                            int32_t H, int32_t d_qk, int32_t d_v,
                            const int64_t* timestamps,
                            const float* pos_bias, int32_t num_pos,
                            const float* time_bias, int32_t num_time_buckets,
                            int32_t max_seqlen,
                            void* out, int64_t out_tok_stride,
                            void* workspace, size_t workspace_bytes, void* stream);

/* hstu_attn_fwd for callers that cannot allocate device memory when they run
 * the attention, such as an inference-engine plugin whose enqueue step must
 * not call cudaMalloc (it can synchronise the device and fail under memory
 * pressure), or code that has no allocator at hand. The paper has no
 * counterpart: this is an interface convenience of this library.
 *
 * Same arguments, layouts and results as hstu_attn_fwd, minus the workspace:
 * the bf16 path keeps its work list and bias tables in a file-scope device
 * array of HSTU_NOALLOC_SCRATCH_BYTES (16 MiB), which every GPU that loads
 * the library holds until the process exits. A batch needing more than that,
 * i.e. hstu_attn_workspace_bytes(B, total_tokens, max_seqlen, H, num_pos) >
 * 16 MiB (about 600 bytes per work unit, plus 3968 bytes per head and
 * 128-token diagonal offset of the position window), returns
 * HSTU_ERR_UNSUPPORTED before anything is launched; use hstu_attn_fwd then.
 * Nothing is allocated or freed by this call, including by torch or any
 * other library.
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream
 * capture. Every call shares the one array and it keeps the last call's
 * contents; the plan kernel rewrites the unit count and every unit it lists
 * before the attention kernel reads them, so nothing has to be cleared. Calls
 * whose executions overlap on the GPU (other streams, or graphs replayed
 * concurrently) race on the array. */
#define HSTU_NOALLOC_SCRATCH_BYTES 16777216
hstu_status_t hstu_attn_fwd_noalloc(hstu_dtype_t dtype,
                                    const void* q, int64_t q_tok_stride,
                                    const void* k, int64_t k_tok_stride,
                                    const void* v, int64_t v_tok_stride,
                                    const int64_t* seq_offsets, int32_t B, int64_t total_tokens,
                                    int32_t H, int32_t d_qk, int32_t d_v,
                                    const int64_t* timestamps,
                                    const float* pos_bias, int32_t num_pos,
                                    const float* time_bias, int32_t num_time_buckets,
                                    int32_t max_seqlen,
                                    void* out, int64_t out_tok_stride, void* stream);

/* Test hook: for every sequence b, every i and every j <= i (sequence by
 * sequence, row-major in i then j) writes the relative-position index
 * min(i-j, num_pos-1) and the time bucket, computed by the same device
 * functions the bf16 attention kernel uses. Outputs are device int32 arrays of
 * sum_b n_b(n_b+1)/2 entries (either may be NULL). */
hstu_status_t hstu_debug_bias_indices(const int64_t* seq_offsets, int32_t B,
                                      int64_t total_tokens, const int64_t* timestamps,
                                      int32_t num_pos, int32_t num_time_buckets,
                                      int32_t* pos_idx_out, int32_t* bucket_out,
                                      void* stream);

/* Test hook for the bounded-wait machinery: launches one block that waits on a
 * pipeline barrier nothing ever signals, with a limit of about `wait_us`
 * microseconds (1..100000), after which it records HSTU_ERR_TIMEOUT in the
 * device error word and returns. Never hangs, never faults. */
hstu_status_t hstu_debug_wait_timeout(int32_t wait_us, void* stream);

/* ---------------------------------------------------------------- layer */

/* The HSTU layer around the attention, in the order the generative-
 * recommenders README gives for HSTU Ultra ("HSTU Ultra attention
 * benchmark": input normalization, the UVQK projection, attention, output
 * normalization with gating and the output projection, residual). The pages
 * name the pieces (hstu_compute_uqvk, hstu_compute_output) but print no
 * formula; the readings taken are: SiLU on all of U|V|Q|K, LayerNorm over a
 * token's features with biased variance and eps inside the square root,
 * gating by U after the output LayerNorm, residual x + Y W2^T. */

/* y[M, N] = epilogue(x[M, K] W[N, K]^T + bias[N]) on tcgen05 tensor cores.
 * x, W, y, residual: device bf16, row strides ldx, ldw (=K typically), ldy, ldr.
 * bias: device fp32 [N] or NULL. residual: [M, N] bf16, required for
 * HSTU_EPI_RESIDUAL, else ignored. K % 64 == 0, N % 128 == 0.
 * The UVQK projection (f1, SiLU epilogue) and the output projection (f2,
 * residual epilogue) of the layer (README, "HSTU Ultra attention
 * benchmark": UVQK and output projection). */
hstu_status_t hstu_linear_fwd(const void* x, int64_t ldx, int64_t M, int32_t K,
                              const void* W, int64_t ldw, int32_t N, const float* bias,
                              hstu_epilogue_t epilogue, const void* residual, int64_t ldr,
                              void* y, int64_t ldy, void* stream);

/* y[m, :] = LayerNorm(a[m, :]) * u[m, :] over F features (biased variance, eps
 * inside the square root, then gamma, beta; NULL = 1, 0). a, u, y: device bf16
 * with row strides lda, ldu, ldy; gamma, beta: device fp32 [F] or NULL.
 * F % 256 == 0 and F <= 2048. The output normalization and gating step of
 * the layer (README, "HSTU Ultra attention benchmark": fused output
 * normalization and gating). */
hstu_status_t hstu_layernorm_gate_fwd(const void* a, int64_t lda, const void* u, int64_t ldu,
                                      int64_t M, int32_t F, const float* gamma,
                                      const float* beta, float eps, void* y, int64_t ldy,
                                      void* stream);

/* y[m, :] = LayerNorm(a[m, :]) over F features (as hstu_layernorm_gate_fwd
 * without the gate). The layer's input normalization before the UVQK
 * projection (README, "HSTU Ultra attention benchmark": input norm). */
hstu_status_t hstu_layernorm_fwd(const void* a, int64_t lda, int64_t M, int32_t F,
                                 const float* gamma, const float* beta, float eps, void* y,
                                 int64_t ldy, void* stream);

/* Workspace bytes of hstu_layer_fwd (D: the model width of x). */
size_t hstu_layer_workspace_bytes(int64_t total_tokens, int32_t B, int32_t D, int32_t H,
                                  int32_t d, int32_t max_seqlen);

/* One HSTU layer forward (bf16, fp32 accumulation) on `stream`:
 *   0. xn = LayerNorm(x)             over the D features, when input_norm != 0
 *                                    (affine in_gamma, in_beta [D] or NULL;
 *                                    eps ln_eps); else xn = x
 *   1. UVQK = silu(xn W1^T + b1)     x [T, D], W1 [4*H*d, D]; columns U|V|Q|K
 *   2. A = attention(Q, K, V)        as hstu_attn_fwd, d_qk = d_v = d
 *   3. Y = LayerNorm(A) * U          over the H*d features of each token
 *   4. out = x + Y W2^T + b2         W2 [D, H*d]; the residual adds x itself
 * x, W1, W2, out: device bf16 row-major; b1 [4Hd], b2 [D], ln_gamma, ln_beta
 * [Hd]: device fp32 or NULL. Other arguments as hstu_attn_run. D % 128 == 0
 * (D % 256 == 0 and D <= 2048 with the input norm), d in {64, 128},
 * H*d % 256 == 0. README, "HSTU Ultra attention benchmark". */
hstu_status_t hstu_layer_fwd(const void* x, int64_t total_tokens, int32_t D,
                             const void* W1, const float* b1,
                             const void* W2, const float* b2,
                             const float* ln_gamma, const float* ln_beta, float ln_eps,
                             int32_t input_norm, const float* in_gamma, const float* in_beta,
                             const int64_t* seq_offsets, int32_t B, int32_t H, int32_t d,
                             const int64_t* timestamps,
                             const float* pos_bias, int32_t num_pos,
                             const float* time_bias, int32_t num_time_buckets,
                             int32_t max_seqlen, void* out,
                             void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------- FP8 projections */

/* Row-wise E4M3 quantization (generative-recommenders README, "FP8 linear
 * reference and benchmark": row-wise E4M3 quantization of the projection
 * operands). For each row r of x (device bf16 [M, K], row stride ldx):
 *   amax = max |x[r, :]|, inv = 448 / amax, scales[r] = amax / 448 (fp32,
 *   rounded to nearest), codes[r, c] = E4M3(fp32(x[r, c] * inv)), rounding
 *   to nearest (ties to an even mantissa) and saturating finite overflow at
 *   +-448, so that x[r, c] ~ value(codes[r, c]) * scales[r]. A row whose inv
 *   is not a finite fp32 number (all zeros, or amax below 448 / FLT_MAX) gets
 *   inv = 0 and scales[r] = 1: zero codes.
 * codes: device uint8 [M, K], row stride ldq (multiple of 16); scales: device
 * fp32 [M]. K % 16 == 0, ldx % 8 == 0, x and codes 16-byte aligned. One
 * launch, one warp per row. */
hstu_status_t hstu_quant_rows_e4m3(const void* x, int64_t ldx, int64_t M, int32_t K, void* codes,
                                   int64_t ldq, float* scales, void* stream);

/* FP8 addmm on tcgen05 (kind::f8f6f4): y[M, N] = epilogue(
 *   (value(xq) value(wq)^T)[m, n] * x_scales[m] * w_scales[n] + bias[n])
 * with xq [M, K] and wq [N, K] E4M3 codes from hstu_quant_rows_e4m3 (row
 * strides ldx, ldw, multiples of 16), fp32 accumulation, and the epilogues,
 * residual, bias and output of hstu_linear_fwd (y, residual bf16). K % 128 ==
 * 0, N % 128 == 0. */
hstu_status_t hstu_linear_fp8_fwd(const void* xq, int64_t ldx, const float* x_scales, int64_t M,
                                  int32_t K, const void* wq, int64_t ldw, const float* w_scales,
                                  int32_t N, const float* bias, hstu_epilogue_t epilogue,
                                  const void* residual, int64_t ldr, void* y, int64_t ldy,
                                  void* stream);

/* hstu_layernorm_gate_fwd with the bf16 result row quantized row-wise to E4M3
 * in the same kernel (as hstu_quant_rows_e4m3 would quantize it) instead of
 * stored: codes device uint8 [M, F] (row stride ldq, multiple of 16), scales
 * device fp32 [M]. The fused output-normalization-to-FP8 step before f2. */
hstu_status_t hstu_layernorm_gate_fp8_fwd(const void* a, int64_t lda, const void* u, int64_t ldu,
                                          int64_t M, int32_t F, const float* gamma,
                                          const float* beta, float eps, void* codes,
                                          int64_t ldq, float* scales, void* stream);

/* hstu_layernorm_fwd with the bf16 result row quantized row-wise to E4M3 in
 * the same kernel (codes and scales as hstu_layernorm_gate_fp8_fwd): the
 * fused input-LayerNorm-to-FP8 step before the UVQK projection (README,
 * "HSTU Ultra attention benchmark": fused LayerNorm-to-FP8 quantization for
 * the UVQK projection). */
hstu_status_t hstu_layernorm_fp8_fwd(const void* a, int64_t lda, int64_t M, int32_t F,
                                     const float* gamma, const float* beta, float eps,
                                     void* codes, int64_t ldq, float* scales, void* stream);

/* Workspace bytes of hstu_layer_fp8_fwd (D: the model width of x). */
size_t hstu_layer_fp8_workspace_bytes(int64_t total_tokens, int32_t B, int32_t D, int32_t H,
                                      int32_t d, int32_t max_seqlen);

/* hstu_layer_fwd with both projections in FP8: x (or, with input_norm,
 * LayerNorm(x) in the same pass) is quantized row-wise to E4M3, f1 runs on
 * E4M3 codes (SiLU epilogue), the attention in bf16, the LayerNorm gate writes
 * E4M3 codes of its bf16 result, and f2 runs on E4M3 codes with the bf16
 * residual x. W1q [4*H*d, D] / w1_scales [4*H*d] and W2q [D, H*d] / w2_scales
 * [D] are the weights quantized once by hstu_quant_rows_e4m3 (device uint8 /
 * fp32). D % 128 == 0 (D % 256 == 0 and D <= 2048 with the input norm),
 * H*d % 256 == 0 (so both K are multiples of 128), d in {64, 128}; other
 * arguments as hstu_layer_fwd. Seven launches: quantize (or LayerNorm and
 * quantize), f1, plan, bias tables, attention, LayerNorm gate, f2. */
hstu_status_t hstu_layer_fp8_fwd(const void* x, int64_t total_tokens, int32_t D, const void* W1q,
                                 const float* w1_scales, const float* b1, const void* W2q,
                                 const float* w2_scales, const float* b2, const float* ln_gamma,
                                 const float* ln_beta, float ln_eps, int32_t input_norm,
                                 const float* in_gamma, const float* in_beta,
                                 const int64_t* seq_offsets,
                                 int32_t B, int32_t H, int32_t d, const int64_t* timestamps,
                                 const float* pos_bias, int32_t num_pos, const float* time_bias,
                                 int32_t num_time_buckets, int32_t max_seqlen, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------- backward */

/* Gradients of the attention (fp32 path, CUDA cores; the pages' reference
 * implementation has forward and backward attention kernels,
 * generative-recommenders README, "HSTU Ultra attention benchmark") for an
 * upstream gradient dout of hstu_attn_fwd's output. With s_ij = q_i.k_j +
 * pos + time, p_ij = silu(s_ij)/N:
 *   dv_j = sum_{i>=j} p_ij dout_i;  ds_ij = (dout_i.v_j) silu'(s_ij) / N
 *   dq_i = sum_{j<=i} ds_ij k_j;    dk_j = sum_{i>=j} ds_ij q_i
 *   dpos[h][min(i-j, P-1)] and dtime[h][bucket] sum the ds_ij of their pairs.
 * q, k, dq, dk: device fp32 [T, H, d_qk] contiguous; v, dout, dv: [T, H,
 * d_v]; dpos [H, num_pos] required when pos_bias is given, dtime [H,
 * num_time_buckets] when timestamps and time_bias are (both overwritten);
 * d_qk, d_v <= 128; num_pos + num_time_buckets <= 12288. Other arguments as
 * hstu_attn_run. Two kernel launches (a query pass and a key pass) plus the
 * table clears. */
hstu_status_t hstu_attn_bwd_f32(const float* q, const float* k, const float* v, const float* dout,
                                const int64_t* seq_offsets, int32_t B, int64_t total_tokens,
                                int32_t H, int32_t d_qk, int32_t d_v, const int64_t* timestamps,
                                const float* pos_bias, int32_t num_pos, const float* time_bias,
                                int32_t num_time_buckets, int32_t max_seqlen, float* dq, float* dk,
                                float* dv, float* dpos, float* dtime, void* stream);

/* Gradients of the attention on tensor cores (tcgen05), bf16 inputs, same
 * formulas as hstu_attn_bwd_f32. q, k, v, dout: device bf16 [T, H, d] with
 * per-token strides q_stride .. dout_stride in elements (multiples of 8, at
 * least H*d; heads contiguous in a token), d = d_qk = d_v in {64, 128}
 * (HSTU_ERR_UNSUPPORTED otherwise, and for dtype HSTU_DTYPE_F32: use
 * hstu_attn_bwd_f32). Outputs are fp32, contiguous [T, H, d] and 16-byte
 * aligned: dq is zeroed and accumulated; dk and dv rows are written for
 * every token of a sequence (rows of tokens outside every sequence are left
 * as they are); dpos [H, num_pos] (required when pos_bias is given) and dtime
 * [H, num_time_buckets] (required when timestamps and time_bias are) are
 * zeroed and accumulated. Products are rounded as in the forward: p and ds
 * in bf16, sums in fp32; table gradients and dq are accumulated with
 * atomics, so their last bits may differ between runs. `workspace` (device,
 * 16-byte aligned, hstu_attn_bwd_workspace_bytes(B, T, max_seqlen) bytes)
 * holds the work list and the order in which the CTAs take its items (most
 * query tiles first, dealt in a snake so every CTA gets about the same
 * number of steps); one plan launch, one backward launch, and the clears.
 * Other arguments as hstu_attn_fwd. Asynchronous on `stream`. */
size_t hstu_attn_bwd_workspace_bytes(int32_t B, int64_t total_tokens, int32_t max_seqlen);
hstu_status_t hstu_attn_bwd(hstu_dtype_t dtype, const void* q, int64_t q_stride, const void* k,
                            int64_t k_stride, const void* v, int64_t v_stride, const void* dout,
                            int64_t dout_stride, const int64_t* seq_offsets, int32_t B,
                            int64_t total_tokens, int32_t H, int32_t d, const int64_t* timestamps,
                            const float* pos_bias, int32_t num_pos, const float* time_bias,
                            int32_t num_time_buckets, int32_t max_seqlen, float* dq, float* dk,
                            float* dv, float* dpos, float* dtime, void* workspace,
                            size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_H_ */
