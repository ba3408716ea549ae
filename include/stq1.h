/*
 * stq1.h -- C ABI of the STQ1_0 quantized-matmul library (libstq1.so), sm_100a.
 *
 * STQ1_0 stores weights in groups of four lanes whose values are {-d, 0, +d}
 * with exactly one zero lane; the 32 possible patterns are a 5-bit code, and
 * one fp16 scale d is shared by 256 weights (lemmy.durstig.online post 66506,
 * "Four weights, five bits").  Each group's code is a 4-bit code plus a 1-bit
 * table-select into a 32-entry codebook; a 256-weight block is 42 bytes,
 * 1.3125 bits per weight ("AngelSlim Shrinks Tencent's 1.5TB Hy4-Preview to
 * 214 GiB at 6x Compression", "How STQ1_0 works").
 *
 * Block layout (the pages fix the semantics, not the bits; this library fixes
 * them as follows), little-endian, 42 bytes, no padding:
 *   bytes  0..1   d, IEEE binary16
 *   bytes  2..33  qs[32]: the 4-bit code n of group g is
 *                 (qs[g >> 1] >> (4 * (g & 1))) & 0xF
 *   bytes 34..41  qh[8]:  the select bit t of group g is
 *                 (qh[g >> 3] >> (g & 7)) & 1
 * Group g (0..63) holds columns 256*b + 4*g + l, l = 0..3.  Codebook: the zero
 * lane is z = n >> 2; the other lanes, in ascending order a < b < c, carry
 * +1, (bit 1 of n ? -1 : +1), (bit 0 of n ? -1 : +1); t = 1 negates all
 * three.  Decoded weight = pattern value * d.
 * Matrix layout: an [N, K] matrix (K % 256 == 0) is N*K/256 blocks stored
 * row-major; block (j, b) starts at byte (j * K/256 + b) * 42.
 *
 * Conventions for every call:
 *   - Return value: STQ1_OK (0) or a negative STQ1_ERR_* code.  Nothing
 *     throws across this boundary; arguments are checked on the host before
 *     any work is enqueued, and a failed check enqueues nothing.
 *   - Device pointers are raw CUDA device addresses owned by the caller; the
 *     library never allocates, frees or retains them after the call returns
 *     (work enqueued on the stream still reads them until it completes).
 *   - Device calls are asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  Errors found on the device (for example an
 *     expert id outside [0, E)) do not trap: the kernel records a code in a
 *     device error word, skips the bad item and finishes; stq1_status()
 *     reads and clears that word.
 *   - bf16 and fp16 values are passed as uint16_t bit patterns.
 *   - Host threads: every call may be made from any thread.  The library's
 *     process-wide state (per-device configuration, cached device
 *     attributes and tensor maps, the path setting) is set up under locks or
 *     atomics.  What a caller passes in is not: two calls that share a
 *     workspace must not overlap.  The device error word is one per device
 *     and process, so a stq1_status() read reports errors of every thread's
 *     calls on that device.
 *   - Each entry point opens an NVTX range named after it, so a profiler's
 *     timeline shows which call enqueued which kernels.
 */
#ifndef STQ1_H
#define STQ1_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define STQ1_OK 0
#define STQ1_ERR_SHAPE (-1)       /* K % 256 != 0, a non-positive size, too large a size */
#define STQ1_ERR_NULL (-2)        /* a required pointer is NULL */
#define STQ1_ERR_CUDA (-3)        /* a CUDA runtime call failed (launch error etc.) */
#define STQ1_ERR_DEVICE (-4)      /* (stq1_status) the device error word was set */
#define STQ1_ERR_VALUE (-5)       /* NaN/Inf weight, negative or non-finite importance */
#define STQ1_ERR_ALIGN (-6)       /* a pointer is not 16-byte aligned */
#define STQ1_ERR_WORKSPACE (-7)   /* workspace NULL or smaller than the query says */
#define STQ1_ERR_ARG (-8)         /* an invalid mode, flag or option */
#define STQ1_ERR_SCRATCH (-9)     /* (stq1_gemv_noalloc) the shape needs more than the built-in scratch */

/* Device error word bits (reported through stq1_status). */
#define STQ1_DEV_BAD_EXPERT 1     /* a topk id was outside [0, E); its slot was skipped */
#define STQ1_DEV_WAIT_LIMIT 2     /* a bounded wait inside a kernel gave up */
#define STQ1_DEV_BAD_VALUE 4      /* (stq1_quantize) NaN/Inf weight or negative/non-finite importance */
#define STQ1_DEV_BOUNDS 8         /* (debug build) an index failed a bounds check; its access was skipped */

/* Encoder modes for stq1_quantize_ref and stq1_quantize. */
#define STQ1_ENC_PLAIN 0          /* amax scale, smallest-|w| lane zeroed */
#define STQ1_ENC_SHERRY 1         /* alternating WLS scale / weighted zero placement */

/* stq1_moe_gateup flags. */
#define STQ1_MOE_WEIGHT_UP 1      /* multiply rows N/2..N-1 (the up half) by the routing weight */
#define STQ1_MOE_FP8 2            /* tile path: E4M3 activations (per-token fp32 scale), fp8 MMAs */
#define STQ1_MOE_SKIP_FOREIGN 4   /* ids outside [0, E) give y = 0 without an error (expert parallelism) */

/* Weight formats for stq1_hessian_error. */
#define STQ1_FMT_STQ1_0 0         /* 42 bytes per 256 weights (1.3125 bpw) */
#define STQ1_FMT_STQ2 1           /* 66 bytes per 256 weights (2.0625 bpw), see stq1_quantize_stq2 */

/* Library version (major * 10000 + minor * 100 + patch). */
int stq1_version(void);

/*
 * stq1_quantize_ref -- host encoder (CPU only, deterministic, multi-threaded).
 *
 * Plain mode (amax encoder: "AngelSlim Shrinks ...", bullet list): per block
 * d = fp16(max |w|) rounded to nearest-even and saturated at 65504; in each
 * group the lane of least |w| is zero (ties: lowest lane) and the others take
 * the sign of w (-0.0 counts as positive).
 * Sherry mode (lemmy.durstig.online post 66506, "Scale and zero position are
 * fit together"): start from the plain zero lanes; `rounds` times fit
 * d = sum h|w| / sum h over the non-zero lanes (weighted least squares), then
 * re-pick each group's zero lane as the one minimising h_l*d*(2|w_l| - d), the
 * extra weighted error of zeroing it (ties: lowest lane); finally refit d for
 * the final lanes and round it to fp16.  Arithmetic is IEEE fp64 with sums in
 * ascending column order; a block whose importance is all zero uses h = 1, a
 * fit whose denominator is zero uses h = 1.
 *
 *   W       [N, K] fp32, row-major, host memory (read only).
 *   h       [K] fp32 per-column importance (diagonal imatrix), host memory;
 *           NULL means h = 1.  Ignored in plain mode.
 *   mode    STQ1_ENC_PLAIN or STQ1_ENC_SHERRY.
 *   rounds  number of alternating rounds for Sherry mode (>= 0; the pages use 3).
 *   out     host buffer of N*K/256*42 bytes, written completely.
 *   threads worker threads (<= 0: use the hardware concurrency).
 * Errors: STQ1_ERR_NULL, STQ1_ERR_SHAPE (K % 256, N <= 0), STQ1_ERR_VALUE
 * (non-finite weight, negative or non-finite h), STQ1_ERR_ARG (mode, rounds).
 * On error `out` may be partly written.
 */
int stq1_quantize_ref(const float* W, const float* h, int64_t N, int64_t K, int mode,
                      int rounds, uint8_t* out, int threads);

/*
 * stq1_quantize -- the same encoders on the GPU, byte-identical to
 * stq1_quantize_ref for every input that function accepts (one thread per
 * 256-weight block, fp64 in the same order, no fused multiply-add).
 *   W      device, [N, K] fp32 row-major, 16-byte aligned.
 *   h      device, [K] fp32 importance, 16-byte aligned (Sherry mode;
 *          NULL means h = 1; ignored in plain mode).
 *   out    device, N*K/256*42 bytes, 2-byte aligned (fully overwritten).
 *   rounds Sherry rounds (0..1000; the pages use 3).
 * Asynchronous on `stream`.  A NaN/Inf weight, or a negative or non-finite
 * importance, sets STQ1_DEV_BAD_VALUE in the device error word (read it with
 * stq1_status) and the affected blocks are written as zeros.
 * Errors: STQ1_ERR_NULL, STQ1_ERR_SHAPE, STQ1_ERR_ARG, STQ1_ERR_ALIGN,
 * STQ1_ERR_CUDA.
 */
int stq1_quantize(const float* W, const float* h, int64_t N, int64_t K, int mode, int rounds,
                  uint8_t* out, void* stream);

/*
 * stq1_dequant -- decoded weights as bf16 (device).
 * W_bf16[j, k] = bf16_rne(fp32(d)) with the pattern's sign, zero lanes +0.0.
 *   W_packed  device, N*K/256*42 bytes, 16-byte aligned.
 *   W_bf16    device, [N, K] uint16 (bf16 bits), 16-byte aligned.
 * Errors: STQ1_ERR_NULL, STQ1_ERR_SHAPE, STQ1_ERR_ALIGN, STQ1_ERR_CUDA.
 */
int stq1_dequant(const void* W_packed, uint16_t* W_bf16, int64_t N, int64_t K, void* stream);

/*
 * stq1_gemv_workspace -- bytes of device workspace stq1_gemv needs for this
 * shape (0 if none).  Layout: the first 2048 bytes hold split-K arrival
 * counters, the rest partial sums.  The counter bytes must be zero before the
 * first call; every call that completes leaves them zero again, whatever the
 * shape, so one workspace can serve calls of different shapes (not
 * concurrently).  Do not share it with stq1_moe_gateup.
 */
size_t stq1_gemv_workspace(int64_t N, int64_t K, int batch);

/*
 * stq1_gemv -- y[t, j] = sum_k W^[j, k] x[t, k], fp32 accumulation.
 * The decoded weight is never materialised in memory ("Runtime" section of
 * the lemmy post: STQ1_0 CUDA kernels).  1 or 2 tokens use the lookup-table
 * kernel: codes index per-group tables of the activation sums, so the weight
 * side has no multiplies (one table load per token and group).  3 to 15
 * tokens use the tensor-core decode kernel:
 * each group's code is expanded once in registers to bf16 +/-1 and 0 and
 * contracted against up to 8 tokens per MMA (fp32 accumulation, d applied
 * per 256-weight block in fp32).  Larger batches use the tensor-core tile
 * kernel when it is expected to be faster (see stq1_set_path).
 *   W_packed   device, [N, K] STQ1_0 blocks, 16-byte aligned.
 *   x          device, [batch, K] bf16 bits, row-major, 16-byte aligned.
 *   y          device, [batch, N] fp32, row-major (fully overwritten).
 *   batch      1 .. 65535.
 *   workspace  device, at least stq1_gemv_workspace(N, K, batch) bytes,
 *              16-byte aligned (may be NULL when that is 0).
 * Accuracy: |y - y_exact| <= 1e-3 * sum_k |W^[j,k] x[t,k]| + 1e-6.
 * Calls that share a workspace must not run concurrently.
 * Errors: STQ1_ERR_NULL, STQ1_ERR_SHAPE, STQ1_ERR_ALIGN, STQ1_ERR_WORKSPACE,
 * STQ1_ERR_CUDA.
 */
int stq1_gemv(const void* W_packed, const uint16_t* x, float* y, int64_t N, int64_t K,
              int batch, void* workspace, size_t ws_bytes, void* stream);

/*
 * stq1_moe_workspace -- bytes of device workspace stq1_moe_gateup needs
 * (routing tables; no zero-fill needed).  Calls sharing it must not overlap.
 */
size_t stq1_moe_workspace(int T, int topk, int E, int64_t N, int64_t K, int flags);

/*
 * stq1_moe_gateup -- routed expert gate/up projections for top-k MoE.
 * y[t, s, :] = W^_{e} x[t, :] with e = topk_ids[t, s] (unweighted), for the
 * fused gate (rows 0..N/2-1) + up (rows N/2..N-1) matrix of each expert.
 * Token-slot pairs are grouped by expert on the device and only the routed
 * experts' blocks are read (256 routed experts, top-8: lemmy post,
 * "Precision follows weight sensitivity").
 *   expert_blocks  device, E consecutive [N, K] STQ1_0 matrices, 16-byte aligned.
 *   x              device, [T, K] bf16 bits, 16-byte aligned.
 *   topk_ids       device, [T, topk] int32.
 *   topk_weights   device, [T, topk] fp32; read only with STQ1_MOE_WEIGHT_UP
 *                  (may be NULL otherwise).
 *   y              device, [T, topk, N] fp32 (fully overwritten; a slot whose
 *                  id is out of range is set to 0 and flagged in the error word).
 *   flags          STQ1_MOE_WEIGHT_UP | STQ1_MOE_FP8 | STQ1_MOE_SKIP_FOREIGN.
 *   ws, ws_bytes   device workspace, at least stq1_moe_workspace(...) bytes
 *                  (computed with the same flags).
 * Requires N even, K % 256 == 0, 1 <= topk <= E (any topk with STQ1_MOE_SKIP_FOREIGN).
 * Paths: with few token-slot pairs per routed expert (decode), experts with
 * one or two pairs run on the lookup-table kernel and the others on the
 * tensor-core decode kernel (units of up to 8 pairs of one expert); with many
 * (prefill) the tensor-core tile kernel.
 * Streams: when a decode call splits its experts this way, the tensor-core
 * part runs on a second stream that the library keeps per device and host
 * thread.  It forks from `stream` with an event after the routing kernel and
 * joins back before the call returns, so work enqueued on `stream` later
 * waits for both parts.  Under stream capture the fork and the join become
 * graph edges; the first such call of a thread creates the stream and its two
 * events, so make it before capturing.  If they cannot be created, both parts
 * run on `stream`.
 * STQ1_MOE_FP8 applies to the tile kernel only: each token row of x is
 * quantized to E4M3 as by stq1_quantize_x_e4m3, the +/-1 weight patterns are
 * E4M3 too, the MMAs run in fp8 with fp32 accumulation and y is multiplied by
 * the row's scale.  The weights stay exact; the activations carry E4M3's
 * relative error (up to 2^-4), so this variant is outside the accuracy bound
 * below and its error is measured, not bounded.  The decode kernels (table
 * and tensor-core decode) ignore the flag.
 * Accuracy (without STQ1_MOE_FP8): as stq1_gemv, per output.
 * Errors: STQ1_ERR_NULL, STQ1_ERR_SHAPE, STQ1_ERR_ALIGN, STQ1_ERR_WORKSPACE,
 * STQ1_ERR_ARG, STQ1_ERR_CUDA.
 */
int stq1_moe_gateup(const void* expert_blocks, const uint16_t* x, const int32_t* topk_ids,
                    const float* topk_weights, float* y, int T, int topk, int E, int64_t N,
                    int64_t K, int flags, void* ws, size_t ws_bytes, void* stream);

/*
 * stq1_swiglu -- the gated activation after a fused gate/up projection (the
 * pages stop at gate/up; this is the plain reading of a gated MoE FFN):
 * act[p, j] = bf16(SiLU(y[p, j]) * y[p, N/2 + j]), SiLU(v) = v / (1 + e^-v),
 * evaluated in fp64 and rounded once to bf16 (nearest, ties to even), ready to
 * be the bf16 input of the down projection.
 *   y    device, [P, N] fp32 (gate rows 0..N/2-1, then up rows), e.g. the
 *        [T, topk, N] output of stq1_moe_gateup with P = T * topk.
 *   act  device, [P, N/2] bf16 bits (fully overwritten).
 * Requires N even.  Asynchronous on `stream`.
 * Errors: STQ1_ERR_NULL, STQ1_ERR_SHAPE, STQ1_ERR_CUDA.
 */
int stq1_swiglu(const float* y, uint16_t* act, int64_t P, int64_t N, void* stream);

/*
 * stq1_moe_combine -- out[t, h] = sum_s w[t, s] * y[t, s, h] in fp32, slots in
 * order (the plain sum when w is NULL, e.g. when the routing weight was
 * applied to the up half with STQ1_MOE_WEIGHT_UP).
 *   y    device, [T, topk, H] fp32;  w  device, [T, topk] fp32 or NULL;
 *   out  device, [T, H] fp32 (fully overwritten).
 * Errors: STQ1_ERR_NULL, STQ1_ERR_SHAPE, STQ1_ERR_CUDA.
 */
int stq1_moe_combine(const float* y, const float* w, float* out, int64_t T, int topk, int64_t H,
                     void* stream);

/*
 * stq1_moe_ffn_workspace / stq1_moe_ffn -- a routed MoE feed-forward layer:
 * gate/up (stq1_moe_gateup) -> SwiGLU (stq1_swiglu) -> down projection per
 * routed (token, slot) pair (stq1_moe_gateup with each pair as its own token)
 * -> combine (stq1_moe_combine), all on `stream`.
 *   gateup_blocks  device, E consecutive [N, H] STQ1_0 matrices (gate rows
 *                  0..N/2-1, up rows N/2..N-1).
 *   down_blocks    device, E consecutive [H, N/2] STQ1_0 matrices.
 *   x              device, [T, H] bf16 bits.  topk_ids [T, topk] int32.
 *   topk_weights   device, [T, topk] fp32; with STQ1_MOE_WEIGHT_UP applied to
 *                  the up half (combine = plain sum), otherwise in the combine;
 *                  NULL (without that flag) gives the unweighted sum.
 *   out            device, [T, H] fp32 (fully overwritten).
 *   flags          STQ1_MOE_WEIGHT_UP | STQ1_MOE_FP8 (fp8 applies to the tile
 *                  path of both projections).
 *   ws, ws_bytes   at least stq1_moe_ffn_workspace(...) bytes, 16-byte aligned.
 * Requires N even, H and N/2 multiples of 256.
 * Errors: as stq1_moe_gateup.
 */
size_t stq1_moe_ffn_workspace(int T, int topk, int E, int64_t N, int64_t H, int flags);
int stq1_moe_ffn(const void* gateup_blocks, const void* down_blocks, const uint16_t* x,
                 const int32_t* topk_ids, const float* topk_weights, float* out, int T, int topk, int E,
                 int64_t N, int64_t H, int flags, void* ws, size_t ws_bytes, void* stream);

/*
 * stq1_moe_ffn_local_workspace / stq1_moe_ffn_local -- one rank's share of an
 * expert-parallel MoE feed-forward layer: the experts [expert_begin,
 * expert_begin + E_local) of E, held in gateup_local / down_local (E_local
 * matrices each, as stq1_moe_ffn), applied to every (token, slot) pair routed
 * to them; pairs routed to other ranks' experts contribute 0.  `out` [T, H]
 * is this rank's partial sum; the layer's output is the sum of all ranks'
 * partials (an all-reduce).  topk_ids hold global expert ids.  Other
 * arguments as stq1_moe_ffn; ws at least stq1_moe_ffn_local_workspace(...).
 * Only this rank's pairs are computed and stored: they are grouped by expert
 * on the device, gate/up writes one row per local pair, SwiGLU and the down
 * projection run over those rows only (the down projection reuses the
 * grouping), and the combine gathers each token's local rows; nothing is
 * written for pairs of other ranks.  (Shapes whose H / 256 or N / 512 is odd
 * run the whole-layer chain with foreign pairs zeroed instead.)
 * All pointers 16-byte aligned.
 * Errors: as stq1_moe_ffn.
 */
size_t stq1_moe_ffn_local_workspace(int T, int topk, int E_local, int64_t N, int64_t H, int flags);
int stq1_moe_ffn_local(const void* gateup_local, const void* down_local, const uint16_t* x,
                       const int32_t* topk_ids, const float* topk_weights, float* out, int T, int topk,
                       int E_local, int expert_begin, int64_t N, int64_t H, int flags, void* ws,
                       size_t ws_bytes, void* stream);

/*
 * stq1_ep_dispatch / stq1_ep_combine -- the token exchange of an
 * expert-parallel MoE layer whose tokens are spread over the ranks as well
 * (prefill).  The pages ran the model on eight GPUs without describing the
 * split ("Tencent's 200GB Hy4-preview ...", "The catch: not a drop-in GGUF");
 * this is the plain expert-parallel reading: each rank sends every (token,
 * slot) pair to the rank that holds its expert, that rank runs the pair
 * through its experts (stq1_moe_ffn_local with the received rows as tokens,
 * topk = 1), and the results come back to be summed per token.  The exchange
 * itself (an all-to-all over NCCL) is the caller's.
 * Ownership: the E experts are split into `world` contiguous ranges, the first
 * E % world ranks holding one expert more.
 *
 * stq1_ep_dispatch groups this rank's pairs p = t * topk + s by owner rank:
 *   topk_ids  device, [T, topk] int32 global expert ids.
 *   x         device, [T, K] bf16 bits, 16-byte aligned, K % 8 == 0.
 *   topk_weights  device, [T, topk] fp32, read only when w_send is not NULL.
 *   order     device, [T * topk] int32: order[i] = the pair sent i-th.
 *   inv       device, [T * topk] int32: inv[p] = i (or -1 for an id outside
 *             [0, E), which is sent nowhere and sets STQ1_DEV_BAD_EXPERT).
 *   counts    device, [world + 1] int32: pairs sent to each rank, in rank
 *             order (rank r's rows are the counts[r] rows after those of
 *             ranks < r), then the total.
 *   local_ids device, [T * topk] int32: local_ids[i] = the expert of pair
 *             order[i] within its owner's range.
 *   x_send    device, [T * topk, K] bf16: x_send[i] = x[order[i] / topk]
 *             (rows past counts[world] are left untouched), 16-byte aligned.
 *   w_send    device, [T * topk] fp32: w_send[i] = topk_weights[order[i]], or
 *             NULL.
 * Rows of one rank are in no particular order (the order changes no result).
 *
 * stq1_ep_combine: out[t, h] = sum over slots s with inv[t * topk + s] >= 0
 * of rows[inv[t * topk + s], h], fp32 in slot order (0 without such a slot);
 * rows = [T * topk, H] fp32, the results returned in send order.
 * Both are asynchronous on `stream`.
 * Errors: STQ1_ERR_NULL, STQ1_ERR_SHAPE, STQ1_ERR_ALIGN, STQ1_ERR_CUDA.
 */
int stq1_ep_dispatch(const int32_t* topk_ids, const uint16_t* x, const float* topk_weights, int T, int topk, int E,
                     int world, int64_t K, int32_t* order, int32_t* inv, int32_t* counts, int32_t* local_ids,
                     uint16_t* x_send, float* w_send, void* stream);
int stq1_ep_combine(const float* rows, const int32_t* inv, float* out, int64_t T, int topk, int64_t H,
                    void* stream);

/*
 * stq1_quantize_x_e4m3 -- the activation quantization of the fp8 tile variant
 * (the pages have no fp8 step; this is the library's choice).  Per row t of
 * x: amax = max |x[t, k]|, inv = 448 / amax and scales[t] = amax / 448 (IEEE
 * fp32 divisions; both 0 for an all-zero row), q[t, k] = the OCP FP8 E4M3 code
 * of the fp32 product x[t, k] * inv, rounded to nearest with ties to even and
 * saturated at +/-448 (the sign of zero is kept).  x[t, k] ~= scales[t] *
 * value(q[t, k]).
 *   x       device, [T, K] bf16 bits (finite), 16-byte aligned.
 *   q       device, [T, K] bytes, 16-byte aligned (fully overwritten).
 *   scales  device, [T] fp32.
 * Requires K % 16 == 0.  Asynchronous on `stream`.
 * Errors: STQ1_ERR_NULL, STQ1_ERR_SHAPE, STQ1_ERR_ALIGN, STQ1_ERR_CUDA.
 */
int stq1_quantize_x_e4m3(const uint16_t* x, int64_t T, int64_t K, uint8_t* q, float* scales,
                         void* stream);

/*
 * stq1_gemv_prefetch -- stq1_gemv, and while it runs its CTAs ask the GPU to
 * bring the next_bytes bytes at W_next into L2 (cp.async.bulk.prefetch; no
 * completion is awaited and nothing waits for it), so that a following call
 * whose weights are W_next finds them in L2 instead of waiting for HBM.  For
 * a chain of matmuls over known matrices (the layers of a decode step).
 * Results are those of stq1_gemv.  Only the lookup-table path (batch below
 * the tile path's threshold) issues the prefetch.
 *   W_next      device pointer, 16-byte aligned, only read; NULL: no prefetch.
 *   next_bytes  bytes to prefetch (rounded down to a multiple of 16); >= 0.
 * Errors: those of stq1_gemv; STQ1_ERR_SHAPE (next_bytes < 0), STQ1_ERR_ALIGN
 * (W_next not 16-byte aligned).
 */
int stq1_gemv_prefetch(const void* W_packed, const uint16_t* x, float* y, int64_t N, int64_t K, int batch,
                       void* workspace, size_t ws_bytes, const void* W_next, int64_t next_bytes, void* stream);

/*
 * stq1_gemv_noalloc -- stq1_gemv without a caller workspace and without any
 * allocation.  The source pages have no counterpart; this entry point exists
 * for callers that cannot allocate device memory or keep a workspace: hosts
 * and plugin frameworks that own all device memory and pass only input and
 * output buffers, and latency-critical code that must not call cudaMalloc
 * (it can synchronize the device).
 *   Same arguments, layouts and accuracy as stq1_gemv, minus the workspace.
 *   Always uses the lookup-table kernel.  Its split-K scratch (2 KiB of
 *   arrival counters plus the partial sums) lives in a 1 MiB buffer compiled
 *   into the library, which every GPU that loads the library holds until the
 *   process exits.  A shape needing more (2048 + S*batch*N*4 bytes, with S the
 *   split count; [4096, 7168] at batch 8 needs 919,552) returns
 *   STQ1_ERR_SCRATCH and enqueues nothing.
 *   The first call on a device looks up that buffer's device address (with
 *   that device current); make that first call before any stream capture.
 *   Each call clears the counters on `stream` before its kernel.  All calls
 *   in the process share the one buffer and it keeps the last call's contents:
 *   calls that may overlap on the GPU (different streams, or concurrent host
 *   threads) race on it and must be serialized by the caller.
 * Errors: STQ1_ERR_NULL, STQ1_ERR_SHAPE, STQ1_ERR_ALIGN, STQ1_ERR_SCRATCH,
 * STQ1_ERR_CUDA.
 */
int stq1_gemv_noalloc(const void* W_packed, const uint16_t* x, float* y, int64_t N, int64_t K,
                      int batch, void* stream);

/*
 * stq1_set_path -- process-wide choice between the matmul kernels, for testing
 * and crossover measurements: 0 = by size (default: 1 or 2 tokens use the
 * lookup-table kernel and 3 to 15 the tensor-core decode kernel; MoE calls
 * averaging fewer than 16 pairs per routed expert send experts with one or
 * two pairs to the lookup-table kernel and the others to the tensor-core
 * decode kernel; 16 or more tokens, and MoE calls averaging 16 or more pairs
 * per routed expert, use the tensor-core tile kernel when it is expected to
 * be faster), 1 = always the lookup-table
 * kernel, 2 = the tile kernel whenever the shape allows it, 3 = the
 * tensor-core decode kernel (up to 8 tokens per unit) whenever the shape
 * allows it.  "Allows" means K / 256 even; other shapes use a generic kernel.
 * The value is read atomically by each call: a call that overlaps a change
 * on another host thread uses either the old or the new choice.
 * Errors: STQ1_ERR_ARG.
 */
int stq1_set_path(int path);

/*
 * stq1_selftest_wait -- exercises the failure-detection path without a fault:
 * one thread waits, through the bounded wait every kernel of this library
 * uses, on a barrier phase that is completed first (arrive = 1) or that
 * nothing completes (arrive = 0).  With arrive = 0 the wait gives up after
 * its bound (2^14 suspended tries of at most 100 us each, so under two
 * seconds), records STQ1_DEV_WAIT_LIMIT in the device error word and the
 * kernel returns; the context stays usable.  Read the outcome with
 * stq1_status.  Asynchronous on `stream`.
 * Errors: STQ1_ERR_ARG (arrive not 0 or 1), STQ1_ERR_CUDA.
 */
int stq1_selftest_wait(int arrive, void* stream);

/*
 * Debug build.  The library also builds as libstq1_debug.so, compiled with
 * STQ1_DEBUG.  That build bounds-checks the indices its kernels take from
 * device memory and from the call's geometry before using them:
 *   - the routing tables: tile counts against the table's size; each tile's
 *     expert, pair range and token count; each pair id and activation row;
 *   - the shared-memory windows a row is read from;
 *   - the shared-memory destinations of every tensor copy;
 *   - the output and routing-weight rows of the tile kernel;
 *   - the rows the gathers, the dispatch and the combines touch.
 * A failed check records STQ1_DEV_BOUNDS in the device error word and skips
 * the access (a unit leaves, a row is zeroed or not stored, a copy is not
 * issued), so results are wrong but nothing reads or writes out of bounds.
 * It is the stand-in for a memory checker; the release build has no checks
 * and the same results.
 *
 * stq1_build_flags -- STQ1_BUILD_DEBUG if this library is the debug build,
 * else 0.
 */
#define STQ1_BUILD_DEBUG 1
int stq1_build_flags(void);

/*
 * stq1_selftest_bounds -- exercises the debug build's bounds check without an
 * out-of-bounds access: one thread stores into a 32-entry shared array at
 * `index` if 0 <= index < bound passes the check.  The address is masked
 * into the array, so any arguments are safe.  In the debug build an index
 * outside [0, bound) records STQ1_DEV_BOUNDS and skips the store; the release
 * build does not check.  Read the outcome with stq1_status.  Asynchronous on
 * `stream`.
 * Errors: STQ1_ERR_CUDA.
 */
int stq1_selftest_bounds(int index, int bound, void* stream);

/*
 * stq1_status -- synchronise `stream`, return STQ1_OK if no device error was
 * recorded since the last call, else STQ1_ERR_DEVICE with the bits in
 * *device_err (may be NULL).  Clears the word.  STQ1_ERR_CUDA if the
 * synchronisation itself fails.
 */
int stq1_status(void* stream, int* device_err);

/*
 * ---- Mixed-precision allocation ----
 * The pages let calibration data choose each layer's bit width: sensitivity is
 * the layer's error under the full Hessian H = X^T X of its calibration
 * inputs, and layers move from STQ1_0 to a 2.06-bpw format greedily by error
 * reduction per added byte ("AngelSlim Shrinks ..." bullet list;
 * lemmy.durstig.online post 66506, "Full-Hessian scoring").  The pages'
 * partner format is third-party; the partner here is STQ2, defined below.
 */

/*
 * stq1_quantize_stq2 -- STQ2 encoder (GPU).  Per 256 weights (66 bytes): bytes
 * 0-1 the fp16 scale d, then 64 code bytes: weight k of the block at bits
 * 2 (k mod 4) of code byte k / 4; code q means the level (d (2q - 3)) / 3.
 * rounds = 0: d = fp16(max |w|) (round to nearest even, saturating at 65504)
 * and each weight takes the nearest level, ties to the lower code.
 * rounds > 0: the pages fit the partner format with the importance matrix
 * (lemmy.durstig.online post 66506, "Full-Hessian scoring"), and STQ2 is fit
 * the way the Sherry scale is: starting from those codes, `rounds` times
 * d = 3 sum h w m / sum h m^2 (m = 2q - 3, k ascending; the weighted
 * least-squares scale for fixed codes), then the nearest levels at that d;
 * the stored scale is fp16 of one more fit.  All in fp64 with a fixed order,
 * so the bytes are those of the oracle's encoder.
 *   W       device, [N, K] fp32 row-major, 16-byte aligned.
 *   h       device, [K] fp32 importance per column, 16-byte aligned, or NULL
 *           (h = 1).  A block whose h is all zero uses h = 1.
 *   rounds  0..1000.
 *   out     device, N*K/256*66 bytes, 2-byte aligned (fully overwritten).
 * Asynchronous on `stream`.  A NaN/Inf weight, or a negative or non-finite
 * importance, sets STQ1_DEV_BAD_VALUE in the device error word and the block
 * is written as zeros.
 * Errors: STQ1_ERR_NULL, STQ1_ERR_SHAPE (K % 256, non-positive sizes),
 * STQ1_ERR_ARG (rounds), STQ1_ERR_ALIGN, STQ1_ERR_CUDA.
 */
int stq1_quantize_stq2(const float* W, const float* h, int64_t N, int64_t K, int rounds, uint8_t* out,
                       void* stream);

/*
 * stq1_hessian_diag -- diagonal of each layer's calibration Hessian (GPU):
 * h[l][k] = sum over r of x[l][r][k]^2, summed in fp64 and rounded once to
 * fp32.  This is the per-column importance (imatrix) the Sherry encoder and
 * the diagonal score use.
 *   x  device, [L][rows][K] bf16 bits, 2-byte aligned.
 *   h  device, [L][K] fp32, 4-byte aligned (fully overwritten).
 * Errors: STQ1_ERR_NULL, STQ1_ERR_SHAPE (non-positive sizes, L > 65535),
 * STQ1_ERR_ALIGN, STQ1_ERR_CUDA.
 */
int stq1_hessian_diag(const uint16_t* x, int64_t L, int64_t rows, int64_t K, float* h, void* stream);

/*
 * stq1_hessian_error -- per-layer quantisation error under the full and the
 * diagonal Hessian (GPU, tensor cores).  For each layer l, with
 * D = W[l] - decode(packed[l]) [N, K] and X = x[l] [n_cal, K]:
 *   out[2l]     = tr(D X^T X D^T) = sum over calibration rows c and output
 *                 rows j of (sum_k D[j,k] X[c,k])^2   (the full score)
 *   out[2l + 1] = sum over j, k of h[l][k] D[j,k]^2   (the diagonal score;
 *                 with h from stq1_hessian_diag it is the imatrix score)
 * D is formed in fp32 and rounded to bf16 for the contraction (fp32
 * accumulation), so the full score carries a relative error of the order of
 * 2^-9 per element of D; the diagonal score is formed from the fp32 D.
 *   format  STQ1_FMT_STQ1_0 or STQ1_FMT_STQ2.
 *   packed  device, [L][N][K/256 * bytes per block], 2-byte aligned.
 *   W       device, [L][N][K] fp32, 16-byte aligned (the unquantised weights).
 *   x       device, [L][n_cal][K] bf16 bits, 16-byte aligned.
 *   h       device, [L][K] fp32, 16-byte aligned.
 *   out     device, [L][2] fp64, 8-byte aligned (zeroed on `stream`, then
 *           accumulated by the kernel; the order of the additions is not fixed).
 * Asynchronous on `stream`.  A wait that runs out sets STQ1_DEV_WAIT_LIMIT.
 * Errors: STQ1_ERR_NULL, STQ1_ERR_ARG (format), STQ1_ERR_SHAPE (K % 256,
 * non-positive sizes), STQ1_ERR_ALIGN, STQ1_ERR_CUDA.
 */
int stq1_hessian_error(int format, const void* packed, const float* W, const uint16_t* x, const float* h,
                       int64_t L, int64_t N, int64_t K, int64_t n_cal, double* out, void* stream);

/*
 * stq1_mix_allocate -- greedy layer allocation (host, deterministic).  Start
 * with every layer in the lower format; visit layers in decreasing order of
 * gain = (err_low - err_high) / (bytes_high - bytes_low) (ties: lower index);
 * stop at the first gain <= 0; upgrade a layer when total + cost <= budget,
 * where total starts as the sum of bytes_low in layer order and grows by each
 * upgrade's cost = bytes_high - bytes_low (a layer that does not fit is
 * skipped and later ones are still tried).  All arithmetic is IEEE fp64.
 *   err_low, err_high, bytes_low, bytes_high  host, [n_layers] fp64.
 *   pick  host, [n_layers]: 1 = the higher format, 0 = the lower.
 * Errors: STQ1_ERR_NULL, STQ1_ERR_SHAPE (n_layers <= 0), STQ1_ERR_VALUE
 * (a non-finite input, or bytes_high <= bytes_low).
 */
int stq1_mix_allocate(const double* err_low, const double* err_high, const double* bytes_low,
                      const double* bytes_high, int64_t n_layers, double budget, uint8_t* pick);

#ifdef __cplusplus
}
#endif

#endif /* STQ1_H */
