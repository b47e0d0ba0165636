/*
 * w4a16.h -- C ABI of libw4a16: weight-only int4 (Q4_0 grid, group 32) matmul for one B200.
 *
 * The operations follow "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8
 * throughput" (deniz.in):
 *   - section "A repack, not a re-quantization": every group of 32 weights along the input
 *     dimension sits on a 16-level grid with levels -8..7; the per-group step is recovered by
 *     trying max|w|/m for m = 1..8, keeping the first that reproduces the group, refining it by
 *     least squares, and storing it at bf16;
 *   - section "What changed in vLLM's TPU backend": W4A16 linear layers, and a fused-MoE method
 *     whose grouped matmul takes a scale per 32-wide group and dequantises each weight tile on
 *     chip before the multiply, with bf16 activations;
 *   - section "The gap at 26B": 128 experts per layer, 8 active per token.
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is DEVICE memory owned by the caller, except where a comment says
 *     otherwise.  The library never allocates or frees memory and keeps no pointer after return.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*; NULL = the legacy
 *     default stream).  Nothing synchronises the host and nothing is copied to the host.
 *   - bf16 values are passed as their uint16 bit patterns.  Arrays are dense and row-major.
 *   - Packed codes ("layout L1"): a row of K weights is K/8 uint32 words holding u = q + 8 (q is
 *     the int4 code in -8..7) of elements 8w..8w+7 in k order: bits 4j..4j+3 of word w hold
 *     element 8w + j, j = 0..7 (the lowest nibble is the lowest k).  Four consecutive words
 *     (16 bytes) hold exactly one group of 32, so one 16-byte load is one group.  The kernels
 *     read this layout as it is; any reordering they need happens on the activation side.
 *     Scales are one bf16 per group: scales[r][g] scales elements 32g..32g+31 of row r.
 *     Dequantised weight = s * q.
 *   - The returned status reports host-side checks (null pointers, sizes, alignment) and launch
 *     failures (W4_ERR_CUDA; the CUDA error is available from w4_last_cuda_error()).  Conditions
 *     found on the device are written to the optional `dev_status` word, which the caller reads
 *     after synchronising.
 *   - Pointers to codes, activations, outputs and workspaces must be 16-byte aligned.
 */
#ifndef W4A16_H
#define W4A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  W4_OK = 0,
  W4_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad alignment */
  W4_ERR_UNSUPPORTED = 2,   /* a valid request this build does not handle */
  W4_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed */
  W4_ERR_TIMEOUT = 4,       /* (device status) a bounded wait gave up */
  W4_ERR_WORKSPACE = 5      /* workspace missing or smaller than w4_workspace_bytes() */
} w4_status;

typedef enum {
  W4_EPI_NONE = 0,          /* out[r, n] = bf16(sum_k a[r, k] * W[n, k]) */
  W4_EPI_GELU_GATE = 1      /* out[r, j] = bf16(gelu_tanh(g_j) * u_j), g = rows [0, N/2) of W,
                               u = rows [N/2, N); out has N/2 columns */
} w4_epilogue;

typedef enum {
  W4_OP_LINEAR = 1,
  W4_OP_ROUTE = 2,
  W4_OP_GMM = 3,
  W4_OP_LINEAR_G = 4,       /* w4a16_linear_g (zero-points assumed present: an upper bound) */
  W4_OP_GMM_G = 5,          /* moe_w4a16_gmm_g (likewise) */
  W4_OP_LAYER = 6,          /* moe_w4a16_layer: M_or_T = T, N = H, K = I, E, k */
  W4_OP_LAYER_CTL = 7       /* its control area at the front of that workspace (T ignored) */
} w4_op;

/*
 * w4_repack -- recover int4 codes and bf16 scales from bf16 weights that sit on the Q4_0 grid.
 * ("A repack, not a re-quantization", the m-search and least-squares refinement.)
 *
 *   w        [rows, K] bf16 weights (input).
 *   rows, K  K % 32 == 0, rows >= 0.  Groups are the rows * K / 32 runs of 32 along K.
 *   codes    [rows, K/8] uint32, layout L1 (output).
 *   scales   [rows, K/32] bf16 (output).
 *   group_m  [rows, K/32] uint8 (output, may be NULL): the first m in 1..8 whose step max|w|/m
 *            reproduces the group, or 0 when no m does ("off the grid").
 *   off_grid_count  one unsigned 64-bit device word (output, may be NULL): set to the number of
 *            off-grid groups of this call.
 *
 * Per group, with all arithmetic in float64 on the bf16 values:
 *   a = max|w_i|; for m = 1..8: step = a/m, r_i = w_i/step, q_i = rint(r_i) (half to even); the
 *   group reproduces when every q_i is in -8..7 and |r_i - q_i| <= 1/16.  The first such m
 *   wins.  Off the grid: q_i = clamp(rint(w_i / (a/8)), -8, 7).  Refinement:
 *   s* = sum_i w_i q_i / sum_i q_i^2 (index order), scale = bf16(s*) rounded to nearest even.
 *   An all-zero group gives scale 0, codes 0, m = 1.  A group holding NaN or infinity is off
 *   the grid with codes 0 and a NaN scale (0x7FC0).
 * The result is bit-identical to that definition (codes, scales, group_m and the count).
 */
w4_status w4_repack(const uint16_t* w, int64_t rows, int64_t K, uint32_t* codes,
                    uint16_t* scales, uint8_t* group_m, unsigned long long* off_grid_count,
                    void* stream);

/*
 * w4a16_linear -- y = x W^T with W dequantised on chip from int4 codes and bf16 scales.
 * ("What changed in vLLM's TPU backend": W4A16 for linear layers.)
 *
 *   x        [M, K] bf16 activations.       codes  [N, K/8] uint32 (layout L1).
 *   scales   [N, K/32] bf16.                 y      [M, N] bf16 (output).
 *   M >= 0, N >= 1, K >= 32 with K % 32 == 0.
 *   workspace, workspace_bytes: device scratch of at least
 *            w4_workspace_bytes(W4_OP_LINEAR, M, N, K, 1, 1) bytes (may be NULL when that is 0;
 *            W4_ERR_WORKSPACE when smaller).  Its contents need no preparation (the call clears
 *            or overwrites the part it relies on, on `stream`).  Calls sharing one workspace must
 *            not overlap on the GPU.
 * y[m, n] = bf16(sum_k x[m, k] * s[n, k/32] * q[n, k]) with float32 accumulation.  Both
 * kernels first write x once in fp16 with a power-of-two exponent per row (exact for every
 * element within a factor 2^27 of its row's largest), and every tensor-core product is exact;
 * the float32 sums and the final rounding are inexact.
 * Two kernels serve the call: for M < 64 (or N % 128 != 0, or K > 4096, or K % 64 != 0) a
 * weight-streaming kernel (workspace: the prepared rows -- fp16 values, row multipliers and
 * per-group bias corrections, in records of 8 or 16 rows per 512- or 256-k stage, about
 * ceil(M/16) * ceil(K/256) * 10.3 KB -- and split-K partials), otherwise the tensor-core kernel (workspace: M * K * 2 bytes and 4 per row, each rounded up to 256, plus one
 * byte per weight row).  In the streaming kernel each
 * group's sum also carries a float32 rounding of a bias term that its correction cancels: about
 * 2^-13 of the group's mean |x| times 32 per group, far below the bf16 output rounding.
 */
w4_status w4a16_linear(const uint16_t* x, const uint32_t* codes, const uint16_t* scales,
                       uint16_t* y, int64_t M, int64_t N, int64_t K, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * moe_route_permute -- top-k expert selection, softmax weights and the expert-major permutation.
 * (128 experts, 8 active per token: "The gap at 26B".)
 *
 *   logits          [T, E] float32 router logits (must not hold NaN).
 *   T >= 0, 1 <= E <= 1024, 1 <= k <= min(E, 32).
 *   topk_ids        [T, k] int32 (output): the k largest logits, descending; equal logits are
 *                   ordered by the lower expert index first.
 *   topk_w          [T, k] float32 (output): softmax over the k selected logits.
 *   expert_offsets  [E + 1] int32 (output): exclusive prefix sum of per-expert pair counts.
 *   sorted_pair     [T * k] int32 (output): pair ids p = t*k + j ordered by (expert, p).
 *   pair_pos        [T * k] int32 (output): inverse of sorted_pair (pair_pos[sorted_pair[r]] = r).
 *   workspace       at least w4_workspace_bytes(W4_OP_ROUTE, T, 0, 0, E, k) bytes.
 * Ids, offsets and both permutations are exact; weights are float32.
 */
w4_status moe_route_permute(const float* logits, int32_t T, int32_t E, int32_t k,
                            int32_t* topk_ids, float* topk_w, int32_t* expert_offsets,
                            int32_t* sorted_pair, int32_t* pair_pos, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * moe_w4a16_gmm -- grouped W4A16 GEMM over experts, one output row per routed (token, expert)
 * pair in expert-major order.  ("What changed in vLLM's TPU backend": the grouped matmul over
 * the experts' packed int4 weights and 32-wide scales, each tile dequantised before the
 * multiply.)
 *
 *   a               activations, bf16, K columns.  When a_row_of_pair is given, a has rows/k
 *                   rows (tokens) and sorted row r reads a[a_row_of_pair[r] / k]; when NULL, a
 *                   has `rows` rows and sorted row r reads a[r].
 *   a_row_of_pair   [rows] int32 or NULL (usually sorted_pair from moe_route_permute).
 *   k               pairs per token (divisor applied to a_row_of_pair).
 *   codes           [E, N, K/8] uint32 (layout L1).    scales  [E, N, K/32] bf16.
 *   expert_offsets  [E + 1] int32: rows of expert e are [off[e], off[e+1]); off[E] == rows.
 *   rows            total sorted rows (T * k).  N >= 1 (even for W4_EPI_GELU_GATE), K % 32 == 0.
 *   epilogue        W4_EPI_NONE: out [rows, N]; W4_EPI_GELU_GATE: out [rows, N/2].
 *   workspace       at least w4_workspace_bytes(W4_OP_GMM, rows, N, K, E, k) bytes
 *                   (W4_ERR_WORKSPACE when smaller; nonzero whenever rows > 0): every sorted row
 *                   of `a` written once, in sorted order, in fp16 with a power-of-two exponent.
 *                   The tensor-core kernel (rows >= 32 * E, K <= 4096, K % 64 == 0, N % 128 == 0
 *                   or (N/2) % 64 == 0 with W4_EPI_GELU_GATE) needs rows * K * 2 bytes and 4
 *                   per row (each rounded up to 256) plus E * N bytes (a power-of-two exponent per
 *                   weight row); the weight-streaming kernel one record per token block of 8
 *                   or 16 rows of an expert and per 512- or 256-k stage (about 10 KB: fp16
 *                   values, row multipliers and per-group bias corrections), for at most
 *                   min(rows, rows / 8 + E) blocks, plus split-K partials for a few rows.
 *   dev_status      one int32 device word or NULL: set to a w4_status code if the device finds a
 *                   problem (offsets out of range: W4_ERR_INVALID_ARG; a pair naming a row past
 *                   the end of `a`: W4_ERR_INVALID_ARG, that row read as row 0); left unchanged
 *                   otherwise.
 * Accumulation is float32 and every tensor-core product is exact; out is rounded to bf16 (the
 * accuracy statement of w4a16_linear applies).
 */
w4_status moe_w4a16_gmm(const uint16_t* a, const int32_t* a_row_of_pair, int32_t k,
                        const uint32_t* codes, const uint16_t* scales,
                        const int32_t* expert_offsets, int32_t E, int64_t rows, int32_t N,
                        int32_t K, int32_t epilogue, uint16_t* out, void* workspace,
                        size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * moe_combine -- y[t] = sum_{j=0..k-1} w[t, j] * o[pair_pos[t*k + j]], float32 in slot order,
 * rounded to bf16.
 *
 *   o         [T * k, H] bf16 expert outputs in sorted order.   topk_w  [T, k] float32.
 *   pair_pos  [T * k] int32.   y  [T, H] bf16 (output).   H % 8 == 0.
 */
w4_status moe_combine(const uint16_t* o, const float* topk_w, const int32_t* pair_pos,
                      int32_t T, int32_t k, int32_t H, uint16_t* y, void* stream);

/*
 * moe_w4a16_layer -- one MoE decode layer in ONE kernel launch:
 *   y = moe_combine(down(gelu_gate(gate_up(x routed by logits)))),
 * i.e. moe_route_permute, moe_w4a16_gmm (gate/up, W4_EPI_GELU_GATE), moe_w4a16_gmm (down) and
 * moe_combine fused into a persistent kernel whose phases hand over through counters in the
 * workspace.  ("What changed in vLLM's TPU backend": the fused-MoE layer over the experts' packed
 * int4 weights; "The gap at 26B": 128 experts, 8 active.)  For the sizes it accepts it computes
 * exactly what those four calls compute on the weight-streaming kernel, in the same order, so y is
 * bit-identical to theirs.
 *
 *   x          [T, H] bf16, 16-byte aligned.       logits  [T, E] float32.
 *   gu_codes   [E, 2I, H/8] uint32 (layout L1), gu_scales [E, 2I, H/32] bf16: gate rows 0..I-1
 *              and up rows I..2I-1 of each expert.   dn_codes [E, H, I/8], dn_scales [E, H, I/32].
 *   y          [T, H] bf16 (output, 16-byte aligned).
 *   workspace  at least w4_workspace_bytes(W4_OP_LAYER, T, H, I, E, k) bytes, 256-byte aligned.
 *              Its first w4_workspace_bytes(W4_OP_LAYER_CTL, 0, H, I, E, k) bytes are the
 *              kernel's counters: zero them once before the first call (every call leaves them
 *              zero, whatever T).  The rest holds the routing, h and the expert outputs.  Calls
 *              sharing a workspace must not overlap on the GPU.
 *   dev_status one int32 device word or NULL: W4_ERR_TIMEOUT if a phase's wait for another ran
 *              out (the kernel then still ends; y is not valid), W4_ERR_INVALID_ARG as for
 *              moe_w4a16_gmm.
 * Accepts 1 <= T <= 128 with T * k <= 6 E (decode: the routed rows form blocks of 8 per expert),
 * E <= 576, 1 <= k <= min(32, E), H and I multiples of 32 (T = 0: nothing to do);
 * W4_ERR_UNSUPPORTED otherwise, W4_ERR_INVALID_ARG for malformed arguments.  The launch is
 * cooperative (one CTA per SM, all resident); it may be captured in a CUDA graph.
 */
w4_status moe_w4a16_layer(const uint16_t* x, const float* logits, int32_t T, int32_t E, int32_t k,
                          const uint32_t* gu_codes, const uint16_t* gu_scales, const uint32_t* dn_codes,
                          const uint16_t* dn_scales, int32_t H, int32_t I, uint16_t* y, void* workspace,
                          size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * w4a16_linear_g, moe_w4a16_gmm_g -- the same linear and grouped GEMM on the weight-format
 * variants: other group sizes along the input dimension and an asymmetric zero-point.
 * ("What quantization really is", section "How the ruler works": a scale and an optional
 * zero-point, asymmetric quantisation when values are not centred on zero, and group-wise
 * granularity.  The page's formulas are lost in extraction; this is the standard uniform form.)
 *
 *   codes    as in layout L1, read as unsigned codes u in 0..15.
 *   scales   [rows, K/group] bf16 (2-byte aligned): one scale per group of `group` elements.
 *   zeros    [rows, K/group] uint8 zero-points z in 0..15, or NULL for the symmetric grid z = 8.
 *   group    32, 64, 128, ... (32 times a power of two) dividing K.
 *   Dequantised weight W = s * (u - z); group = 32 with zeros NULL is exactly the symmetric
 *   format of w4a16_linear / moe_w4a16_gmm.  Every other argument, the workspace (sized with
 *   W4_OP_LINEAR_G / W4_OP_GMM_G) and the accuracy statement are those of w4a16_linear /
 *   moe_w4a16_gmm; both calls always take the weight-streaming kernel, scales and zero-points
 *   loaded directly per stage (the zero-point's term (8 - z) * sum over the group of x enters
 *   each group's MMA as part of its C operand, in float32).
 */
w4_status w4a16_linear_g(const uint16_t* x, const uint32_t* codes, const uint16_t* scales,
                         const uint8_t* zeros, int32_t group, uint16_t* y, int64_t M, int64_t N,
                         int64_t K, void* workspace, size_t workspace_bytes, void* stream);
w4_status moe_w4a16_gmm_g(const uint16_t* a, const int32_t* a_row_of_pair, int32_t k,
                          const uint32_t* codes, const uint16_t* scales, const uint8_t* zeros,
                          int32_t group, const int32_t* expert_offsets, int32_t E, int64_t rows,
                          int32_t N, int32_t K, int32_t epilogue, uint16_t* out, void* workspace,
                          size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * moe_rms_chain -- the input of the next layer of a stack of MoE layers from this layer's output:
 *   x_next[t, h] = bf16(y[t, h] / sqrt(mean_h y[t, h]^2 + eps)), rounded to nearest even.
 * (No counterpart on the pages, which give no blocks between the MoE layers of a model; this is
 * the plainest chaining that keeps a stack of gated expert MLPs -- quadratic in their input --
 * bounded: a root-mean-square normalisation without a learned weight, eps = 1e-6 in this
 * library's stack.)
 *
 *   y       [T, H] bf16 (input).    x_next  [T, H] bf16 (output; may not alias y).
 *   T >= 0, H % 8 == 0, eps >= 0.  Both pointers 16-byte aligned.
 * The sum of squares is float32 in a fixed order; the root and the division are correctly
 * rounded float32, so an element can differ from the float64 definition by one bf16 unit where
 * the quotient sits within float32 rounding of a bf16 midpoint.
 */
w4_status moe_rms_chain(const uint16_t* y, int64_t T, int32_t H, float eps, uint16_t* x_next,
                        void* stream);

/*
 * w4a16_linear_noalloc -- w4a16_linear for callers that cannot allocate device memory.
 * (No counterpart on the pages: an interface addition of this library.)
 *
 * Same arguments, result and accuracy as w4a16_linear, without a workspace: the prepared
 * activation rows and, when K is split across CTAs, the float32 partials and arrival counters
 * live in a file-scope device array of 8 MiB (8388608 bytes) that every GPU loading the library
 * keeps until process exit.  Callers
 * that are handed only their input and output buffers (a plugin inside a framework that owns all
 * device memory through its own pool, or a runtime held to a fixed memory budget) can call it
 * without cudaMalloc, which would bypass the pool and synchronise the device.
 *   - Always takes the weight-streaming kernel, over the rows in as many chunks as keep each
 *     chunk's scratch within 8 MiB.  Returns W4_ERR_WORKSPACE, launching nothing, when a single
 *     row's scratch exceeds 8 MiB (8388608 bytes).
 *   - The first call on a device looks up the array's device address (once per device); make
 *     that first call before any stream capture.
 *   - Every call reuses the same array (its kernels clear the arrival counters they use, on
 *     `stream`): calls that overlap on the GPU race and must be ordered by the caller (one
 *     stream, or events).
 *   - Allocates nothing: no cudaMalloc/cudaFree, no allocating library routine.
 */
w4_status w4a16_linear_noalloc(const uint16_t* x, const uint32_t* codes, const uint16_t* scales,
                               uint16_t* y, int64_t M, int64_t N, int64_t K, void* stream);

/* Workspace bytes an entry point needs for the given sizes (0 when it needs none). */
size_t w4_workspace_bytes(int32_t op, int64_t M_or_T, int64_t N, int64_t K, int32_t E, int32_t k);

/* Human-readable name of a status code (static storage). */
const char* w4_status_str(int32_t status);

/* The CUDA error code behind the last W4_ERR_CUDA returned on this host thread (0 if none). */
int32_t w4_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H */
