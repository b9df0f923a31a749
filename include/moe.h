/*
 * moe.h -- C ABI of the routed-MoE FFN layer for NVIDIA B200 (sm_100a).
 *
 * The layer (Hy3 routed experts; "Tencent Hy3-295B 架构深度拆解",
 * pillumina.github.io, §2.3 parameter breakdown and §4.1 routing flow;
 * "DeepSeek V4-Flash 架构 QA", cctoctofx.netlify.app, Q4.5 and Q8.4; Hy3
 * commentary, wmrh.cn/news/24252, §2.3 fp32 combine):
 *
 *   logits = x W_gate^T (+ gate_bias)          fp32 accumulate
 *   s      = sigmoid(logits)
 *   top-k  = k largest s per token, equal scores -> lower expert index
 *   w_j    = scale * s_j / sum_{i in top-k} s_i
 *   y_j    = W_down[e_j] ( SiLU(W_gate_rows[e_j] x) * (W_up_rows[e_j] x) )
 *   out    = bf16( sum_j w_j * float(y_j) )     fp32 sum, one final cast
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are DEVICE pointers, row-major and contiguous, 16-byte
 *   aligned. bf16 tensors are passed as void* (IEEE bfloat16 bit patterns).
 * - Layouts: x [T, d]; w_gate [E, d]; w_gate_up [E, 2*d_ff, d] with rows
 *   [0, d_ff) the gate projection and [d_ff, 2*d_ff) the up projection;
 *   w_down [E, d, d_ff]; topk_idx [T, k] int32; topk_w [T, k] fp32 (both in
 *   descending score order); out [T, d].
 * - FP8 weights (MOE_FLAG_FP8_WEIGHTS): w_gate_up / w_down hold e4m3 codes
 *   (one byte each) in the same layouts, and s_gate_up [E, 2*d_ff] /
 *   s_down [E, d] hold fp32 per-output-row scales; the weight value is
 *   code * scale. Without the FP8 or FP4 flag both scale pointers must be
 *   NULL (the scale pointers are void* because their element type follows
 *   the weight format).
 * - FP4 weights (MOE_FLAG_FP4_WEIGHTS; the V4-Flash column of "Tencent
 *   Hy3-295B 架构深度拆解" §2.2, OCP MX E2M1 with block-32 scales):
 *   w_gate_up [E, 2*d_ff, d/2] / w_down [E, d, d_ff/2] hold E2M1 codes two to
 *   a byte, the even column in the low nibble (bit 3 the sign, bits 2-1 the
 *   exponent, bit 0 the mantissa: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), and
 *   s_gate_up [E, 2*d_ff, d/32] / s_down [E, d, d_ff/32] hold one E8M0 byte b
 *   per 32 consecutive columns of a row, the block's scale 2^(b - 127)
 *   (b = 255 is not a scale: unspecified output). The weight value is
 *   code value * block scale. With neither path flag the experts run on the
 *   weight-streaming kernels at up to one mean row per expert (T*k <= E) and
 *   on the tensor-core SM-pair kernels above that (d, d_ff multiples of 256;
 *   the streaming kernels otherwise). MOE_FLAG_FP8_WEIGHTS,
 *   MOE_FLAG_PACKED_WEIGHTS or MOE_FLAG_SHARED_EXPERT with it:
 *   MOE_ERR_INVALID_ARG.
 * - Packed bf16 weights (MOE_FLAG_PACKED_WEIGHTS): w_gate_up and w_down hold
 *   the same values rearranged by moe_pack_weights into 16 KB blocks of 128
 *   rows x 64 columns (block (e, rb, kb) = rows [128 rb, 128 rb + 128) and
 *   columns [64 kb, 64 kb + 64) of expert e, row-major inside the block;
 *   blocks ordered by e, then rb, then kb), so that every weight tile the
 *   tensor-core kernels load is one contiguous span of memory (measured on
 *   B200: gate_up 4-6% faster). Needs bf16 weights, d and d_ff multiples of
 *   256 and the tensor-core path: with MOE_FLAG_FP8_WEIGHTS or
 *   MOE_FLAG_STREAM_PATH it is MOE_ERR_INVALID_ARG, with other shapes
 *   MOE_ERR_UNSUPPORTED_SHAPE.
 * - Shared expert (MOE_FLAG_SHARED_EXPERT; "Tencent Hy3-Flash QA" Q4.7, the
 *   complete Hy3 block): w_gate_up / w_down (and s_gate_up / s_down) hold
 *   E + 1 experts, and expert E is a shared expert that every token uses with
 *   weight 1 on top of its k routed experts:
 *     out = bf16( sum_j w_j * float(y_j) + float(y_shared) )   (shared last).
 *   The routing arrays stay [T, k]; the grouping, the expert GEMMs and the
 *   combine work on k + 1 slots per token (slot k of every token is expert E)
 *   and E + 1 experts: row_of has T*(k+1) entries, counts E+1, offsets E+2,
 *   x_perm / h / y T*(k+1) rows. Needs E <= 255.
 * - Grouping ("permuted rows"): token-slot s = t*k + j goes to row
 *   row_of[s] = offsets[e] + (number of earlier slots s' < s with the same
 *   expert e = topk_idx[s]); offsets[e] = sum_{e' < e} counts[e'],
 *   offsets[E] = T*k. Rows of one expert are contiguous and keep slot order.
 * - Supported shapes: T >= 1; d and d_ff multiples of 128; 1 <= E <= 256;
 *   1 <= k <= min(E, 32); T*k*max(d, d_ff) < 2^31. Anything else returns
 *   MOE_ERR_UNSUPPORTED_SHAPE before any launch.
 * - ws is a caller-owned device workspace of at least moe_workspace_size(cfg)
 *   bytes, 256-byte aligned, initialised once with moe_workspace_init. The
 *   library allocates no memory and keeps no state between calls other than
 *   per-device kernel attributes and a driver entry point looked up once.
 * - stream is a cudaStream_t (NULL = legacy default stream). Every call is
 *   asynchronous on it; no call synchronises, except moe_read_status.
 * - Return value: MOE_OK (0) or a negative MOE_ERR_* code. Argument errors are
 *   reported before any work is queued. MOE_ERR_CUDA means a launch failed
 *   (cudaGetLastError). Faults inside kernels are not converted; kernels
 *   whose waits are bounded record MOE_ERR_TIMEOUT in the workspace status
 *   word instead of hanging (read it with moe_read_status).
 * - Values: NaN/Inf inputs give unspecified outputs. Results are
 *   deterministic: the same inputs give bitwise-identical outputs.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1)       /* NULL pointer, misalignment, bad flag mix */
#define MOE_ERR_UNSUPPORTED_SHAPE (-2) /* shape outside the supported set above */
#define MOE_ERR_WORKSPACE (-3)         /* ws_bytes < moe_workspace_size(cfg) */
#define MOE_ERR_CUDA (-4)              /* a CUDA launch or runtime call failed */
#define MOE_ERR_TIMEOUT (-5)           /* a bounded device wait gave up */

#define MOE_FLAG_FP8_WEIGHTS 0x1u /* expert weights are e4m3 codes + fp32 row scales */
#define MOE_FLAG_STREAM_PATH 0x2u /* experts on the weight-streaming (decode) kernels */
#define MOE_FLAG_GEMM_PATH 0x4u   /* experts on the tensor-core grouped GEMMs */
#define MOE_FLAG_PACKED_WEIGHTS 0x8u /* bf16 expert weights in moe_pack_weights' layout */
#define MOE_FLAG_SHARED_EXPERT 0x10u /* expert E of the weights is a shared expert (below) */
#define MOE_FLAG_FP4_WEIGHTS 0x20u /* expert weights are E2M1 codes + E8M0 block-32 scales */

/* Which expert weight moe_pack_weights rearranges. */
#define MOE_WEIGHTS_GATE_UP 0 /* w_gate_up [E, 2*d_ff, d] */
#define MOE_WEIGHTS_DOWN 1    /* w_down [E, d, d_ff] */
/* With neither path flag the library picks by the mean rows per expert T*k/E. */

typedef struct moe_config {
    int32_t T;      /* tokens */
    int32_t d;      /* hidden size (4096 for Hy3) */
    int32_t E;      /* routed experts (192) */
    int32_t k;      /* experts per token (8) */
    int32_t d_ff;   /* expert intermediate size (1536) */
    float scale;    /* router_scaling_factor (2.826) */
    uint32_t flags; /* MOE_FLAG_* */
} moe_config;

/* Bytes of workspace every entry point below needs for cfg (0 if cfg is
 * invalid). Covers the routing scratch, the grouping, the permuted activations
 * [T*k, d], the intermediate h [T*k, d_ff] and the expert outputs [T*k, d]. */
MOE_API size_t moe_workspace_size(const moe_config* cfg);

/* Zero the workspace's control words (status word and routing counters) for
 * cfg. Call once after allocating ws, before any other call that uses it. */
MOE_API int moe_workspace_init(const moe_config* cfg, void* ws, size_t ws_bytes, void* stream);

/* Router: logits = x w_gate^T (+ gate_bias, nullable [E] fp32, added before the
 * sigmoid), sigmoid, top-k (ties -> lower index), renormalise over the k
 * selected scores and multiply by cfg->scale. Writes topk_idx [T, k] int32 and
 * topk_w [T, k] fp32 in descending score order.
 * Pages: "Tencent Hy3-295B 架构深度拆解" §4.1 (router lines and steps 1-5);
 * Hy3 commentary §3.3 for a logit bias added before the sigmoid. */
MOE_API int moe_route(const moe_config* cfg, const void* x, const void* w_gate, const float* gate_bias,
              int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes, void* stream);

/* moe_route with the complete Hy3 block's e_score_correction_bias: score_bias
 * (nullable [E] fp32) is added to the sigmoid scores for the choice of the k
 * experts only; topk_w still renormalises the unbiased sigmoid scores of the
 * chosen experts ("Tencent Hy3-295B 架构深度拆解" §4.1 steps 2-4; "Tencent
 * Hy3-Flash QA" Q4.3). NULL gives moe_route exactly. */
MOE_API int moe_route2(const moe_config* cfg, const void* x, const void* w_gate,
               const float* gate_bias, const float* score_bias, int32_t* topk_idx, float* topk_w,
               void* ws, size_t ws_bytes, void* stream);

/* Router score functions (moe_route_options.score_fn). Both are increasing in
 * the logit, so the choice is the k largest logits either way. */
#define MOE_SCORE_SIGMOID 0       /* s = 1 / (1 + e^-z) (Hy3) */
#define MOE_SCORE_SQRT_SOFTPLUS 1 /* s = sqrt(log(1 + e^z)) (the V4-Flash router,
                                     "Tencent Hy3-295B 架构深度拆解" §2.2) */

/* Optional router inputs, for moe_route3 / moe_forward3 (every pointer
 * nullable: NULL turns the piece off).
 *   score_bias   [E] fp32 e_score_correction_bias, as in moe_route2;
 *   norm_weight  [d] fp32 route_norm weight ("Tencent Hy3-Flash QA" Q4.9):
 *                the router scores xn = x / sqrt(mean(x^2) + norm_eps) * g
 *                (the experts still take x); norm_eps > 0 (1e-6 is the
 *                RMSNorm epsilon the pages give);
 *   score_fn     MOE_SCORE_SIGMOID or MOE_SCORE_SQRT_SOFTPLUS: the score s
 *                that is ranked (plus score_bias, if given) and renormalised,
 *                w_j = scale * s_j / sum_{i in top-k} s_i; any other value is
 *                MOE_ERR_INVALID_ARG. */
typedef struct moe_route_options {
    const float* score_bias;
    const float* norm_weight;
    float norm_eps;
    int32_t score_fn;
} moe_route_options;

/* moe_route with the options above (opt NULL: moe_route). With a norm weight
 * the routing runs on the CUDA-core router at every batch size. */
MOE_API int moe_route3(const moe_config* cfg, const void* x, const void* w_gate,
               const float* gate_bias, const moe_route_options* opt, int32_t* topk_idx,
               float* topk_w, void* ws, size_t ws_bytes, void* stream);

/* Group token-slots by expert (the grouping defined above): writes counts [E],
 * offsets [E+1], row_of [T*k] (int32) and x_perm [T*k, d] bf16 with
 * x_perm[row_of[t*k+j]] = x[t]. Pages: the per-expert loop with index_add_ of
 * "DeepSeek V4-Flash 架构 QA" Q8.4, re-expressed as a grouping for batched
 * expert GEMMs ("Tencent Hy3-Flash QA" Q6.4, grouped MM). */
MOE_API int moe_permute(const moe_config* cfg, const int32_t* topk_idx, const void* x, int32_t* counts,
                int32_t* offsets, int32_t* row_of, void* x_perm, void* ws, size_t ws_bytes,
                void* stream);

/* The grouping of moe_permute without the activation copy: writes counts,
 * offsets and row_of exactly as moe_permute does, and token_of_row [T*k]
 * int32 with token_of_row[row_of[t*k+j]] = t for every kept slot (rows at or
 * beyond offsets[E] are not written). For moe_expert_gate_up_gather, which
 * reads the token rows of x by these indices. Same pages as moe_permute. */
MOE_API int moe_permute_index(const moe_config* cfg, const int32_t* topk_idx, int32_t* counts,
                      int32_t* offsets, int32_t* row_of, int32_t* token_of_row, void* ws,
                      size_t ws_bytes, void* stream);

/* gate_up step of the SwiGLU experts on grouped rows: for each expert e and
 * each of its rows r in [offsets[e], offsets[e+1]):
 *   h[r, f] = bf16( SiLU(g) * u ),  g = <x_perm[r], w_gate_up[e, f]>,
 *   u = <x_perm[r], w_gate_up[e, d_ff + f]>, fp32 accumulate and epilogue.
 * h is [T*k, d_ff] bf16. Pages: "DeepSeek V4-Flash 架构 QA" Q4.5 (SwiGLU);
 * "Tencent Hy3-295B 架构深度拆解" §2.3 (fused gate_up_proj 2*1536 x 4096). */
MOE_API int moe_expert_gate_up(const moe_config* cfg, const void* x_perm, const int32_t* offsets,
                       const void* w_gate_up, const void* s_gate_up, void* h, void* ws,
                       size_t ws_bytes, void* stream);

/* moe_expert_gate_up with the grouped rows read from x by index: the row r
 * of expert e is x[token_of_row[r]] (x [T, d] bf16, token_of_row as written
 * by moe_permute_index, every entry in [0, T) for rows below offsets[E]).
 * Result identical to moe_permute + moe_expert_gate_up. The bf16 tensor-core
 * SM-pair kernel gathers the rows with TMA as it loads them; the other paths
 * first copy them into the workspace. */
MOE_API int moe_expert_gate_up_gather(const moe_config* cfg, const void* x,
                              const int32_t* token_of_row, const int32_t* offsets,
                              const void* w_gate_up, const void* s_gate_up, void* h, void* ws,
                              size_t ws_bytes, void* stream);

/* down step: y[r, i] = bf16( <h[r], w_down[e, i]> ), fp32 accumulate; y is
 * [T*k, d] bf16. Pages: "Tencent Hy3-295B 架构深度拆解" §2.3 (down_proj
 * 4096 x 1536). */
MOE_API int moe_expert_down(const moe_config* cfg, const void* h, const int32_t* offsets,
                    const void* w_down, const void* s_down, void* y, void* ws, size_t ws_bytes,
                    void* stream);

/* Both expert steps (h lives in ws): y [T*k, d] bf16 from x_perm. */
MOE_API int moe_experts(const moe_config* cfg, const void* x_perm, const int32_t* offsets,
                const void* w_gate_up, const void* s_gate_up, const void* w_down,
                const void* s_down, void* y, void* ws, size_t ws_bytes, void* stream);

/* fp32 combine and unpermute: out[t, :] = bf16_rne( sum_{j<k} topk_w[t, j] *
 * float(y[row_of[t*k + j], :]) ), summed in fp32 in j order, one final cast.
 * Pages: Hy3 commentary §2.3 (enable_moe_fp32_combine = true: convert the
 * branch outputs to fp32 before adding, cast back once). */
MOE_API int moe_combine(const moe_config* cfg, const void* y, const int32_t* row_of, const float* topk_w,
                void* out, void* ws, size_t ws_bytes, void* stream);

/* Batches of at most this many token-slots (T*k) are grouped by index
 * (moe_permute_index) and their gate_up GEMM gathers the token rows itself
 * (moe_expert_gate_up_gather); larger batches write the permuted copy
 * (moe_permute + moe_expert_gate_up): once tiles hold many tokens, the
 * one-row TMA gathers cost more than the copy. */
#define MOE_GATHER_MAX_SLOTS 4096

/* The whole layer: route, group, gate_up, down, combine (the grouping and
 * gate_up as MOE_GATHER_MAX_SLOTS says). out [T, d] bf16. The intermediates
 * live in ws. Resets the workspace status word first. */
MOE_API int moe_forward(const moe_config* cfg, const void* x, const void* w_gate, const float* gate_bias,
                const void* w_gate_up, const void* s_gate_up, const void* w_down,
                const void* s_down, void* out, void* ws, size_t ws_bytes, void* stream);

/* Rearrange one bf16 expert weight (which = MOE_WEIGHTS_GATE_UP or
 * MOE_WEIGHTS_DOWN, row-major as above) into the packed layout described
 * under MOE_FLAG_PACKED_WEIGHTS: w_packed has the same size and must not
 * overlap w. A pure permutation of the values (bit-exact), done once when
 * the weights are loaded; the layer's mathematics is unchanged. cfg->flags
 * may carry MOE_FLAG_PACKED_WEIGHTS or not; d and d_ff must be multiples of
 * 256 (else MOE_ERR_UNSUPPORTED_SHAPE) and the FP8 flag must be clear. This
 * storage form is not in the pages; it serves the tensor-core kernels'
 * tile loads. */
MOE_API int moe_pack_weights(const moe_config* cfg, int which, const void* w, void* w_packed,
                     void* stream);

/* moe_forward with the optional score_bias of moe_route2 (NULL gives
 * moe_forward exactly). Together with MOE_FLAG_SHARED_EXPERT this is the
 * complete Hy3 MoE block. */
MOE_API int moe_forward2(const moe_config* cfg, const void* x, const void* w_gate,
                 const float* gate_bias, const float* score_bias, const void* w_gate_up,
                 const void* s_gate_up, const void* w_down, const void* s_down, void* out,
                 void* ws, size_t ws_bytes, void* stream);

/* moe_forward with the router options of moe_route3 (opt NULL: moe_forward). */
MOE_API int moe_forward3(const moe_config* cfg, const void* x, const void* w_gate,
                 const float* gate_bias, const moe_route_options* opt, const void* w_gate_up,
                 const void* s_gate_up, const void* w_down, const void* s_down, void* out,
                 void* ws, size_t ws_bytes, void* stream);

/* Expert parallelism ("DeepSeek V4-Flash 架构 QA" Q4.7, the expert-parallel
 * strategy, and Q4.10, the MoE's all-to-all traffic): P ranks each own
 * E_local = E/P consecutive experts. A rank receives the grouped token rows
 * of its experts from n_src ranks, source by source, each source's rows
 * grouped by local expert: counts [n_src, E_local] int32 (device) holds the
 * rows of local expert e from source p at counts[p * E_local + e]. Writes
 * expert_of_row [n_rows] int32 (device): the local expert of each received
 * row in that arrival order, the routing (k = 1) with which moe_permute
 * regroups the rows by expert for the local grouped GEMMs. Rows at or past
 * the sum of counts get -1. n_src * E_local <= MOE_EP_MAX_SEGMENTS and
 * E_local <= 256, else MOE_ERR_UNSUPPORTED_SHAPE; NULL pointers or
 * n_rows < 1: MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED_SHAPE. Asynchronous on
 * stream; allocates nothing. */
#define MOE_EP_MAX_SEGMENTS 8192
MOE_API int moe_ep_row_experts(const int32_t* counts, int32_t n_src, int32_t E_local,
                               int32_t* expert_of_row, int32_t n_rows, void* stream);

/* Failure-detection self-test: one thread waits, with the library's bounded
 * wait and a limit of limit_ns (1 ns .. 10 s), on an mbarrier that nothing
 * completes, then records MOE_ERR_TIMEOUT in the status word of ws (read it
 * with moe_read_status). Faults, traps and hangs nothing; the context stays
 * usable. Not part of the layer (the pages have no counterpart). */
MOE_API int moe_selftest_bounded_wait(void* ws, unsigned long long limit_ns, void* stream);

/* Bytes of the fixed device array behind moe_route_noalloc. */
#define MOE_NOALLOC_SCRATCH_BYTES (2u << 20)

/* moe_route for callers that cannot allocate device memory (no workspace
 * argument). The pages have no counterpart: this is a deployment convenience.
 * It runs the CUDA-core router with moe_route's K split S (1 <= S <= 16; S = 1
 * for every T > 128 at E = 192): where moe_route runs that router too (T <=
 * 128, or k > 8) the indices and weights are bitwise moe_route's. For
 * T >= 129 with k <= 8, moe_route runs the tensor-core router, whose logits
 * sum in another order: the same experts on every token whose k-th/(k+1)-th
 * score gap is at least ~1e-5, the weights within ~2e-5 relative. Its scratch
 * -- fp32 partial logits [S, T, E] and one counter per 8 tokens -- lives in a
 * device array of MOE_NOALLOC_SCRATCH_BYTES compiled into the library, held
 * on every GPU that loads it until the process exits. Returns
 * MOE_ERR_UNSUPPORTED_SHAPE when 4*S*T*E plus the counters (4*ceil(T/8)
 * bytes, rounded up to 256) exceed that size (T <= 2728 at E = 192), besides
 * the shape checks of moe_route. The first call on a device (that device
 * current) looks up the array's address; make it before any stream capture
 * (later calls outside capture look it up again, so a device reset leaves no
 * stale address). All calls share the array: calls that overlap on the GPU
 * race and must be serialised by the caller. It calls no allocator. */
MOE_API int moe_route_noalloc(const moe_config* cfg, const void* x, const void* w_gate,
                              const float* gate_bias, int32_t* topk_idx, float* topk_w,
                              void* stream);

/* Synchronise stream, then read and clear the workspace status word: MOE_OK,
 * or MOE_ERR_TIMEOUT if a bounded device wait gave up since the last read. */
MOE_API int moe_read_status(void* ws, void* stream);

/* Static text for a status code. */
MOE_API const char* moe_status_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
