/*
 * moe_lowbit.h -- C ABI of the routed low-bit MoE FFN layer (sm_100a).
 *
 * The layer (DeepSeek-V4-style routed MoE over packed expert weights):
 *   1. route: fp32 router logits, sqrtsoftplus scores, top-k with the
 *      selection bias, renormalised weights -- or, in hash mode, the
 *      token-id -> expert table tid2eid;
 *   2. permute: group the T*k (token, slot) pairs by expert;
 *   3. expert FFN: per routed pair y = W2 . (silu(W1 . x) * (W3 . x)) with
 *      W1/W3/W2 dequantised in registers from affine or mxfp4 packs;
 *   4. combine: out[t] = sum_j w[t,j] * y[t,j] (+ shared expert), rounded
 *      once to bf16.
 *
 * Sources, by page title and section:
 *   [PR1192]  mlx-lm PR "Add DeepSeek-v4 (Flash/Pro)": sqrtsoftplus numerical
 *             stability note (softplus = logaddexp(x, 0)); cross-reference
 *             table row "MoE gate dtype" (logits in fp32 for both the top-k
 *             and the hash router); weight-key notes (pre-stacked experts
 *             w1/w2/w3 = gate/down/up of the switch MLP).
 *   [CARD-4BIT]  model card "mlx-community / DeepSeek-V4-Flash-4bit",
 *             Architecture ("Hash-routed MoE", "sqrtsoftplus scoring") and
 *             Conversion (affine 4-bit, group 64).
 *   [CARD-MLX4]  model card "DeepSeek-V4-Flash-MLX-4bit", "REAP-pruned builds"
 *             (router renormalises over the experts it keeps; hash layers use
 *             tid2eid) and "What this port implements" (tid2eid keyed on
 *             token id; FP4 e2m1 packed two per byte).
 *   [PR1190]  mlx-lm PR "Add DeepSeek-V4 model and safetensors/tokenizer
 *             fallback handling": E8M0 scale = 2^(b-127).
 *   [CARD-MIXED] model card "DeepSeek-V4-Flash-0731-MLX-Serve-mixed-2-3-8bit",
 *             precision table (2/3/4/8-bit affine, group 64/128; shared
 *             experts 8-bit) and conversion notes (affine w = scale*q + bias
 *             in MLX's layout; e2m1 + e8m0 decode losslessly to bf16).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are caller-owned DEVICE pointers (cudaMalloc /
 *     torch), unless an entry point says otherwise.  The library never
 *     allocates device memory: scratch comes from a caller workspace of at
 *     least moe_workspace_size() bytes, 256-byte aligned.  The workspace also
 *     holds the device error word; it must be zeroed once before first use
 *     (e.g. cudaMemset) and not be shared by calls that overlap on the GPU.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; no entry point synchronises
 *     except moe_read_device_error.
 *   - Host-side validation happens before any launch and returns
 *     MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED / MOE_ERR_WORKSPACE
 *     synchronously; moe_last_error_detail() then describes the problem.
 *   - Bad *data* (token id outside [0, vocab), tid2eid entry outside [0, E))
 *     never traps: the kernel records MOE_ERR_DEVICE_INPUT in the workspace
 *     error word, routes that slot to expert 0 with weight 0, and continues.
 *     The tensor-core FFN path (step 3) records the same code when an
 *     activation, hidden value or dequantised weight leaves the fp16 range
 *     (|v| > 65504) that its tensor-core operands use.
 *   - A failed launch returns MOE_ERR_CUDA (the CUDA error is consumed and
 *     reported by moe_last_error_detail()).
 *   - Layouts are row-major.  Weights are stored [out, in] per expert and
 *     stacked over experts (F.linear / QuantizedLinear convention).
 */
#ifndef MOE_LOWBIT_H
#define MOE_LOWBIT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null/host pointer, bad dims, misalignment */
  MOE_ERR_UNSUPPORTED = 2,   /* valid but not implemented (format, size)   */
  MOE_ERR_WORKSPACE = 3,     /* workspace smaller than moe_workspace_size */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed       */
  MOE_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up         */
  MOE_ERR_DEVICE_INPUT = 6   /* out-of-range token id / table entry, or a
                                value outside fp16 range on the tensor-core
                                FFN path                                    */
} moe_status_t;

typedef enum { MOE_FMT_AFFINE = 0, MOE_FMT_MXFP4 = 1 } moe_fmt_t;

/*
 * One stacked expert matrix, logical shape [E, out, in] (device pointers).
 *
 * affine [CARD-MIXED precision table; CARD-4BIT Conversion]:
 *   bits in {2,3,4,8}, group in {32,64,128}; W = scale*q + bias per group
 *   of `group` consecutive inputs.
 *   q      : uint32 [E, out, in*bits/32], LSB-first bitstream along `in`
 *            (code i at bits [i*bits, (i+1)*bits) of the row's words; 3-bit
 *            codes straddle words).
 *   scales : bf16   [E, out, in/group]
 *   biases : bf16   [E, out, in/group]
 * mxfp4 [CARD-MLX4; PR1190; CARD-MIXED conversion notes]:
 *   bits = 4, group = 32; W = e2m1(code) * 2^(e - 127).
 *   q      : uint32 [E, out, in/8], low nibble = even element; code bit 3 is
 *            the sign, bits 2..1 the exponent (bias 1), bit 0 the mantissa.
 *   scales : uint8  [E, out, in/32] e8m0 exponents (255 is not supported).
 *   biases : NULL
 * Alignment: q, scales, biases 16-byte aligned.
 */
typedef struct {
  int32_t fmt;      /* moe_fmt_t */
  int32_t bits;
  int32_t group;
  int32_t reserved; /* set to 0 */
  const uint32_t* q;
  const void* scales;
  const void* biases;
} moe_qmat_t;

/*
 * Layer dimensions.  T tokens, d_model inputs/outputs, d_ff hidden width per
 * routed expert, n_experts routed experts, top_k experts per token.
 * hash_mode != 0 selects tid2eid routing (top_k = table width).  vocab is
 * the number of tid2eid rows (hash mode only).  d_ff_shared > 0 declares
 * one always-on shared expert of that hidden width (0: none).
 * n_experts is the layer's own routed expert count: a REAP-pruned layer
 * [CARD-MLX4 "REAP-pruned builds"] passes the number of experts it kept and
 * the survivors' router rows and packs, so routing renormalises over them.
 * router_dtype selects the router weight's storage type: fp32 (0) or bf16
 * (1), the gate's storage in the released checkpoints [CARD-MIXED precision
 * table]; either way each logit is an fp32 dot product of x with the widened
 * row [PR1192 "MoE gate dtype"].
 * Limits: 1 <= T, 32 <= d_model, d_ff, d_ff_shared <= 8192 and multiples of
 * 32 and of every group size used; 1 <= top_k <= min(n_experts, 32);
 * n_experts <= 1024.
 */
typedef struct {
  int32_t T;
  int32_t d_model;
  int32_t d_ff;
  int32_t n_experts;
  int32_t top_k;
  int32_t hash_mode;
  int32_t vocab;
  int32_t d_ff_shared;
  int32_t router_dtype; /* router_w storage: 0 = fp32, 1 = bf16 (logits are fp32 either way) */
} moe_dims_t;

/* Bytes of scratch the calls below need for these dims (0 if dims invalid). */
size_t moe_workspace_size(const moe_dims_t* dims);

/*
 * Step 1 -- routing [PR1192 gate dtype + sqrtsoftplus notes; CARD-4BIT
 * Architecture; CARD-MLX4 REAP section].
 *   learned (hash_mode == 0):
 *     L = x . router_w^T in fp32; s = sqrt(logaddexp(L, 0));
 *     ids = top_k of (s + router_b) per token, ties to the lower expert id,
 *     listed in descending key order; w = s[ids] / sum(s[ids]).
 *     router_b may be NULL (no selection bias).
 *   hash (hash_mode != 0):
 *     ids[t, :] = tid2eid[token_ids[t], :] in table order;
 *     w = renormalised s of those experts' fp32 logits, or 1/k when
 *     router_w is NULL.
 *   x        : bf16 [T, d_model]
 *   router_w : fp32 or bf16 (dims->router_dtype) [n_experts, d_model]
 *              (NULL only in hash mode)
 *   router_b : fp32 [n_experts] or NULL    (learned mode only)
 *   token_ids: int32 [T]                   (hash mode only)
 *   tid2eid  : int32 [vocab, top_k]        (hash mode only)
 *   topk_ids : int32 [T, top_k] (out);  topk_w : fp32 [T, top_k] (out)
 */
moe_status_t moe_route(const moe_dims_t* dims, const void* x, const void* router_w,
                       const float* router_b, const int32_t* token_ids, const int32_t* tid2eid,
                       int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes, void* stream);

/*
 * Step 2 -- permutation: stable counting sort of the flat pairs i = t*k+j by
 * expert id.
 *   topk_ids       : int32 [T*k] (in; every id must be in [0, n_experts))
 *   expert_offsets : int32 [n_experts+1] (out) -- expert e owns sorted
 *                    positions [off[e], off[e+1])
 *   sorted_rows    : int32 [T*k] (out) flat indices, ascending within expert
 *   inv            : int32 [T*k] (out) inv[sorted_rows[p]] = p
 */
moe_status_t moe_permute(const moe_dims_t* dims, const int32_t* topk_ids, int32_t* expert_offsets,
                         int32_t* sorted_rows, int32_t* inv, void* ws, size_t ws_bytes, void* stream);

/*
 * Step 3 -- grouped SwiGLU expert FFN over packed weights [PR1192 weight-key
 * notes: w1 = gate, w3 = up, w2 = down].  For every sorted position p of
 * expert e (token t = sorted_rows[p] / k):
 *   y[p] = W2[e] . (silu(W1[e] . x[t]) * (W3[e] . x[t])),  silu(a) = a/(1+e^-a)
 * with fp32 accumulation.  w1 and w3 must share one format.
 *   x : bf16 [T, d_model];  w1, w3 : [E, d_ff, d_model];  w2 : [E, d_model, d_ff]
 *   expert_offsets : int32 [n_experts+1], sorted_rows : int32 [T*k] as
 *            moe_permute writes them.  They are checked on the device before
 *            use: offsets[0] = 0, offsets[n_experts] = T*k, non-decreasing,
 *            every sorted row in [0, T*k).  A violation records
 *            MOE_ERR_DEVICE_INPUT in the error word and no expert runs (y is
 *            left unwritten); nothing is read or written out of bounds.
 *   y : fp32 [T*k, d_model] (out) in sorted order.
 * Two implementations (moe_set_ffn_path): a weight-streaming GEMV that
 * dequantises in registers and keeps x and h in fp32, for small batches; and
 * a tcgen05 grouped GEMM for large batches, whose operands are fp16 (x, the
 * dequantised weights and h are each rounded once to fp16, 11-bit
 * significand) with fp32 accumulation.  The tensor-core path needs d_ff and
 * d_model to be multiples of 128; values beyond the fp16 range are reported
 * as MOE_ERR_DEVICE_INPUT.
 */
moe_status_t moe_expert_ffn(const moe_dims_t* dims, const void* x, const int32_t* expert_offsets,
                            const int32_t* sorted_rows, const moe_qmat_t* w1, const moe_qmat_t* w3,
                            const moe_qmat_t* w2, float* y, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_expert_ffn without a workspace (no counterpart on the pages; it exists
 * for callers of this library that cannot allocate device memory: a host
 * framework that owns the whole device pool and forbids foreign allocations,
 * a plug-in that is only given its input and output buffers, or code that
 * must not call cudaMalloc/cudaFree because those calls can synchronise the
 * device).  Same arguments and results as moe_expert_ffn, minus ws/ws_bytes.
 *
 * Its scratch (error word, active-expert list, hidden rows h) is one static
 * device array of 4 MiB that every GPU loading this library holds until the
 * process exits.  Limit: 256 + 256-aligned 4*(n_experts+1) + 4*T*top_k*d_ff
 * bytes must fit in 4 MiB (e.g. T*top_k <= 510 at d_ff = 2048); larger
 * problems return MOE_ERR_UNSUPPORTED before any launch.  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress) and
 * caches it, so make that first call before any stream capture.  Every call
 * on a device shares the same array and leaves its contents behind: calls
 * that overlap on the GPU (different streams without ordering, or several
 * host threads) race and corrupt each other's results.  The library itself
 * allocates nothing on this path.  Device-side errors (a permutation that
 * fails its check, a bounded wait that gave up) are kept in the array's
 * error word, the first one since the last read; moe_read_noalloc_error
 * reports and clears it.
 */
moe_status_t moe_expert_ffn_noalloc(const moe_dims_t* dims, const void* x, const int32_t* expert_offsets,
                                    const int32_t* sorted_rows, const moe_qmat_t* w1, const moe_qmat_t* w3,
                                    const moe_qmat_t* w2, float* y, void* stream);

/*
 * The device error word of moe_expert_ffn_noalloc's static scratch on the
 * current device (the counterpart of moe_read_device_error for that entry
 * point; no counterpart on the pages).  Synchronises `stream`, stores
 * MOE_OK, MOE_ERR_DEVICE_INPUT or MOE_ERR_TIMEOUT in *code_out and clears
 * the word.  Allocates nothing.
 */
moe_status_t moe_read_noalloc_error(int32_t* code_out, void* stream);

/*
 * Step 4 -- weighted combine:
 *   out[t] = bf16_rne( sum_{j<k} topk_w[t,j] * y[inv[t*k+j]] + y_shared[t] )
 * summed in ascending j, then the shared term.
 *   y : fp32 [T*k, d_model] sorted order;  inv : int32 [T*k];
 *   topk_w : fp32 [T*k];  y_shared : fp32 [T, d_model] or NULL;
 *   out : bf16 [T, d_model] (out)
 */
moe_status_t moe_combine(const moe_dims_t* dims, const float* y, const int32_t* inv,
                         const float* topk_w, const float* y_shared, void* out, void* stream);

/*
 * The whole layer: steps 1-4 plus, when dims->d_ff_shared > 0, the shared
 * expert (shared[0..2] = w1, w3, w2 with E = 1, added with weight 1
 * [CARD-MIXED precision table; CARD-MLX4 "Why mixed-4_8bit"]).
 * token_ids/tid2eid are used in hash mode, router_b in learned mode.
 * topk_ids_out / topk_w_out are optional copies of the routing (may be NULL).
 *   out : bf16 [T, d_model]
 * Prefill-sized T use the tensor-core grouped GEMM; small T the streaming
 * GEMV path.  Results agree within the stated output tolerance.
 */
moe_status_t moe_forward(const moe_dims_t* dims, const void* x, const int32_t* token_ids,
                         const void* router_w, const float* router_b, const int32_t* tid2eid,
                         const moe_qmat_t* w1, const moe_qmat_t* w3, const moe_qmat_t* w2,
                         const moe_qmat_t* shared, void* out, int32_t* topk_ids_out,
                         float* topk_w_out, void* ws, size_t ws_bytes, void* stream);

/*
 * One expert slice of the layer, for expert parallelism (no counterpart on
 * the pages; the layer's combine is a sum over (token, slot) terms, so it
 * splits by expert): routing runs over all n_experts as in moe_forward, but
 * only experts expert_begin <= e < expert_end run, only their slots enter
 * the combine, and the shared expert is added when include_shared is 1.
 *   out_partial : fp32 [T, d_model], 16-byte aligned:
 *     out_partial[t] = sum_{j<k, e(t,j) in range} topk_w[t,j] * y[t,j]
 *                      (+ y_shared[t]), ascending j, fp32, no rounding to bf16
 * Ranks owning a partition of [0, n_experts), the shared expert on exactly
 * one of them, add (all-reduce) their partials to the layer's output before
 * its bf16 rounding.  Runs on the fused single-launch path: T <= 32 and the
 * shapes that path admits; otherwise MOE_ERR_UNSUPPORTED.  A range outside
 * [0, n_experts] or include_shared not 0/1: MOE_ERR_INVALID_ARG.  Other
 * arguments as in moe_forward.
 */
moe_status_t moe_forward_partial(const moe_dims_t* dims, int32_t expert_begin, int32_t expert_end,
                                 int32_t include_shared, const void* x, const int32_t* token_ids,
                                 const void* router_w, const float* router_b, const int32_t* tid2eid,
                                 const moe_qmat_t* w1, const moe_qmat_t* w3, const moe_qmat_t* w2,
                                 const moe_qmat_t* shared, float* out_partial, int32_t* topk_ids_out,
                                 float* topk_w_out, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_forward with HOST activations: x_host (bf16 [T, d_model]) and, in hash
 * mode, token_ids_host (int32 [T]) are copied to the workspace, the layer
 * runs, and the bf16 result reaches out_host: written there directly by the
 * layer's last kernel when out_host is page-locked host memory mapped into
 * the device's address space (cudaHostAlloc, or a pinned torch tensor) and
 * the output is at most 1 MiB, else copied back from the workspace.
 * Weights, router and table stay device pointers.  Copies are
 * cudaMemcpyAsync on `stream`; use pinned host memory for asynchrony and
 * synchronise the stream before reading out_host.
 */
moe_status_t moe_forward_host(const moe_dims_t* dims, const void* x_host, const int32_t* token_ids_host,
                              const void* router_w, const float* router_b, const int32_t* tid2eid,
                              const moe_qmat_t* w1, const moe_qmat_t* w3, const moe_qmat_t* w2,
                              const moe_qmat_t* shared, void* out_host, void* ws, size_t ws_bytes,
                              void* stream);

/*
 * mxfp8 weight rows to bf16 [PR1192 FP8 re-quantisation thread: fp8 e4m3
 * weight bytes, one e8m0 scale byte per 32 consecutive elements of a row]:
 *   out[r, i] = bf16( e4m3(codes[r, i]) * 2^(scales[r, i/32] - 127) )
 *   codes : bytes [rows, n_in] (byte i of a row is element i), 16-byte aligned
 *   scales: bytes [rows, n_in/32];  out : bf16 [rows, n_in], 16-byte aligned
 * Exact (each value has 4 significant bits times a power of two) while the
 * product lies within bf16's range: every normal e4m3 code for any scale
 * byte from 1 to 254 whose result is finite, subnormal codes for scale
 * bytes >= 5.  Scale byte 255 (the format's NaN) gives +-inf.  n_in a
 * positive multiple of 32, rows >= 0 (0: nothing to do); otherwise
 * MOE_ERR_INVALID_ARG.  One launch, no workspace; the 128x128 block scales of
 * FP8 checkpoints map to these per-32-group bytes on the host (each row's
 * group g takes block (row / 128, g / 4)).
 */
moe_status_t moe_dequant_mxfp8(const void* codes, const uint8_t* scales, int64_t rows, int32_t n_in, void* out,
                               void* stream);

/*
 * mHC residual mixing, fused (the block next to the MoE layer in each
 * DeepSeek-V4 layer) [CARD-4BIT Architecture "mHC": hc_mult parallel copies
 * of the hidden state recombined by a doubly-stochastic, Sinkhorn-normalised
 * mixing matrix; PR1192 review note "Sinkhorn normalization": softmax then
 * sum-and-divide iterations, fused into one pass].  Per token t:
 *   P = row-wise softmax of logits[t];
 *   iters times: every column of P divided by (its sum + eps), then every
 *                row divided by (its sum + eps);
 *   out[t, i, :] = bf16_rne( sum_j P[i, j] * h[t, j, :] )   (fp32 sums)
 *   logits : fp32 [T, n, n];  h : bf16 [T, n, d];  out : bf16 [T, n, d]
 *            (must not alias h);  P_out : fp32 [T, n, n] or NULL.
 * Limits: 1 <= n <= 8, d a positive multiple of 8, 0 <= iters <= 10000,
 * 0 <= eps <= 1; h and out 16-byte aligned.  One launch, no workspace.
 */
moe_status_t moe_hc_sinkhorn_mix(int32_t T, int32_t n, int32_t d, int32_t iters, float eps,
                                 const float* logits, const void* h, float* P_out, void* out, void* stream);

/*
 * Synchronises `stream`, reads the workspace error word into *code_out
 * (MOE_OK or MOE_ERR_DEVICE_INPUT / MOE_ERR_TIMEOUT) and clears it.
 */
moe_status_t moe_read_device_error(void* ws, int32_t* code_out, void* stream);

/*
 * Benchmark timing hooks (calling thread only).  When `events` is non-NULL,
 * the next moe_forward / moe_forward_host call on this thread records
 * events[0] (a cudaEvent_t) before its first kernel and events[i+1] after its
 * i-th kernel, for at most n_events events, on the call's stream; the hook is
 * consumed by that call.  moe_timing_count() then returns how many events
 * were recorded and moe_timing_label(i) names the kernel between events[i]
 * and events[i+1].  Pass NULL to clear.
 */
moe_status_t moe_set_timing_events(void* const* events, int32_t n_events);
int32_t moe_timing_count(void);
const char* moe_timing_label(int32_t i);

/*
 * Expert-FFN implementation used by the calling thread's moe_expert_ffn /
 * moe_forward / moe_forward_host calls (a per-thread setting: other
 * threads' calls are not affected; not for the allocation-free entry point,
 * which always streams).  For moe_forward / moe_forward_host, AUTO (default)
 * runs the whole layer as ONE fused launch for small batches when the shapes
 * allow it (T <= 32, T*top_k <= 256, d_model a multiple of 256, d_model and
 * d_ff multiples of 64 and of the formats' stage widths -- 1024 inputs for
 * 2-bit, 512 for 3/4-bit and mxfp4, 256 for 8-bit -- and not 2-bit with
 * 32-input groups): routing,
 * both FFN stages on the integer tensor-core MMA, and the combine (whose k
 * slots are summed in ascending j, then the shared expert, one bf16
 * rounding).  Otherwise AUTO takes the tcgen05 grouped GEMM from T >= 4
 * (d_ff, d_model multiples of 128) and the weight-streaming GEMV below.
 * DECODE_FUSED forces the fused launch (MOE_ERR_UNSUPPORTED when the shapes
 * do not allow it); GEMV and TENSOR_CORE force the step-by-step kernels.
 * Returns the previous setting, or -1 (setting unchanged) for an unknown
 * value.
 */
typedef enum {
  MOE_FFN_AUTO = 0,
  MOE_FFN_GEMV = 1,
  MOE_FFN_TENSOR_CORE = 2,
  MOE_FFN_DECODE_FUSED = 3
} moe_ffn_path_t;
int32_t moe_set_ffn_path(int32_t path);

/*
 * Testing aid for the bounded device-side waits (no counterpart on the
 * pages).  While enabled on the calling thread, the fused small-batch launch
 * makes its W2 stages wait on a dependency count that nothing completes,
 * with a ~1 ms limit instead of ~2 s: the launch then records
 * MOE_ERR_TIMEOUT in the workspace error word, lets its in-flight copies
 * land, resets its counters and returns; the output is not valid.  A later
 * call with the hook disabled runs normally on the same workspace.  Returns
 * the previous setting.  Not for production use.
 */
int32_t moe_test_stall_fused_wait(int32_t enable);

/* Static description of a status code. */
const char* moe_status_string(moe_status_t status);

/* Detail of the last host-side failure on the calling thread ("" if none). */
const char* moe_last_error_detail(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_LOWBIT_H */
