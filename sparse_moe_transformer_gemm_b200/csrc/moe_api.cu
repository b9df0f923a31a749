// moe_api.cu -- the C ABI declared in include/moe.h: argument checks, the
// workspace carve-up and the kernel launches. Host code only.
#include <math.h>

#include "internal.h"

using namespace moe;

namespace {

constexpr uint32_t kKnownFlags = MOE_FLAG_FP8_WEIGHTS | MOE_FLAG_STREAM_PATH | MOE_FLAG_GEMM_PATH |
                                 MOE_FLAG_PACKED_WEIGHTS | MOE_FLAG_SHARED_EXPERT |
                                 MOE_FLAG_FP4_WEIGHTS;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_cfg(const moe_config* c) {
    if (!c) return MOE_ERR_INVALID_ARG;
    if ((c->flags & ~kKnownFlags) != 0) return MOE_ERR_INVALID_ARG;
    if ((c->flags & MOE_FLAG_STREAM_PATH) && (c->flags & MOE_FLAG_GEMM_PATH))
        return MOE_ERR_INVALID_ARG;
    if ((c->flags & MOE_FLAG_PACKED_WEIGHTS) &&
        (c->flags & (MOE_FLAG_FP8_WEIGHTS | MOE_FLAG_STREAM_PATH)))
        return MOE_ERR_INVALID_ARG;
    // FP4 experts: routed experts only, in their own code layout
    if ((c->flags & MOE_FLAG_FP4_WEIGHTS) &&
        (c->flags & (MOE_FLAG_FP8_WEIGHTS | MOE_FLAG_PACKED_WEIGHTS | MOE_FLAG_SHARED_EXPERT)))
        return MOE_ERR_INVALID_ARG;
    if (!isfinite(c->scale)) return MOE_ERR_INVALID_ARG;
    if (c->T < 1 || c->E < 1 || c->E > 256 - shared_slots(*c) || c->k < 1 || c->k > c->E ||
        c->k > 32)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->d < 128 || c->d % 128 != 0 || c->d > 8192) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->d_ff < 128 || c->d_ff % 128 != 0 || c->d_ff > 8192) return MOE_ERR_UNSUPPORTED_SHAPE;
    const long long R = (long long)c->T * (c->k + shared_slots(*c));
    const long long wide = c->d > c->d_ff ? c->d : c->d_ff;
    if (R * wide >= (1LL << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if ((c->flags & MOE_FLAG_PACKED_WEIGHTS) && !pair_gemm_supported(*c))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

bool packed(const moe_config* c) { return (c->flags & MOE_FLAG_PACKED_WEIGHTS) != 0; }

// Expert weights: bf16 without a quantised format (no scales); e4m3 codes +
// fp32 row scales, or E2M1 codes + E8M0 block scales, with one.
int check_expert_weights(const moe_config* c, const void* w, const void* s) {
    if (!w || !aligned16(w)) return MOE_ERR_INVALID_ARG;
    if (c->flags & (MOE_FLAG_FP8_WEIGHTS | MOE_FLAG_FP4_WEIGHTS)) {
        if (!s) return MOE_ERR_INVALID_ARG;
    } else if (s) {
        return MOE_ERR_INVALID_ARG;
    }
    return MOE_OK;
}

int check_ws(const moe_config* c, const void* ws, size_t ws_bytes) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < ws_layout(*c).total) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                   \
    do {                                \
        int rc_ = (expr);               \
        if (rc_ != MOE_OK) return rc_;  \
    } while (0)

// Automatic choice: the TMA-fed tensor-core tiles stream bf16 weights faster
// than the register-staged streaming kernels at every batch size measured on
// B200 (decode T=64: 1.07 ms vs 1.45 ms per layer), so they are the default.
// FP8 and FP4 weights have a tensor-core path on SM pairs only (d, d_ff
// multiples of 256); other shapes with those weights use the streaming kernels.
// The tensor-core FP4 path widens every weight tile to bf16 once per token
// tile and issues its MMAs whatever the tile's token count, which below about
// one token per expert costs more than the streaming kernels' direct FMAs:
// FP4 streams up to kFp4StreamRowsPerExpert mean rows per expert (measured at
// the Hy3 shape, top-6, per layer streaming vs tensor cores: T=8 0.28 vs
// 0.38 ms; T=64 1.27 vs 1.22 ms; T=2048 31.2 vs 1.51 ms).
constexpr int kFp4StreamRowsPerExpert = 1;
bool quantised(const moe_config* c) {
    return (c->flags & (MOE_FLAG_FP8_WEIGHTS | MOE_FLAG_FP4_WEIGHTS)) != 0;
}
bool use_stream_path(const moe_config* c) {
    if (c->flags & MOE_FLAG_STREAM_PATH) return true;
    if (c->flags & MOE_FLAG_GEMM_PATH) return false;
    if (quantised(c) && !pair_gemm_supported(*c)) return true;
    return (c->flags & MOE_FLAG_FP4_WEIGHTS) &&
           (long long)c->T * c->k <= (long long)kFp4StreamRowsPerExpert * c->E;
}

// Router: the tensor-core kernel where it applies (k <= 8) and the batch fills
// more than one 128-token tile; small batches (decode) use the K-split CUDA-core
// kernel, whose grid covers the SMs where the tensor-core one runs a handful
// of CTAs.
constexpr int kRouterTcMinTokens = 129;

// route_norm needs the per-token sum of squares next to the logits: the
// CUDA-core router computes both exactly in fp32 (the tensor-core router's bf16
// operands cannot carry x * g unrounded), so it serves every batch size then.
cudaError_t route(const moe_config* c, const void* x, const void* w_gate, const float* gate_bias,
                  const moe_route_options* opt, int32_t* idx, float* w, void* ws,
                  cudaStream_t s) {
    const moe_route_options none = {nullptr, nullptr, 0.f, MOE_SCORE_SIGMOID};
    const moe_route_options& o = opt ? *opt : none;
    const WsLayout L = ws_layout(*c);
    if (!o.norm_weight && router_tc_supported(*c) && c->T >= kRouterTcMinTokens)
        return launch_router_tc(*c, x, w_gate, gate_bias, o.score_bias, o.score_fn, idx, w,
                                at<int>(ws, L.status), s);
    return launch_router(*c, x, w_gate, gate_bias, o.score_bias, o.norm_weight, o.norm_eps,
                         o.score_fn, idx, w, at<float>(ws, L.logits), at<float>(ws, L.sumsq),
                         at<int32_t>(ws, L.counters), router_ksplit(*c), s);
}

int check_route_options(const moe_route_options* opt) {
    if (!opt) return MOE_OK;
    if (opt->norm_weight && !(opt->norm_eps > 0.f && isfinite(opt->norm_eps)))
        return MOE_ERR_INVALID_ARG;
    if (opt->score_fn != MOE_SCORE_SIGMOID && opt->score_fn != MOE_SCORE_SQRT_SOFTPLUS)
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

int experts_gate_up(const moe_config* c, const void* x_perm, const int32_t* offsets,
                    const void* w_gate_up, const void* s_gate_up, void* h, void* ws,
                    cudaStream_t s) {
    const moe_config g = grouped_config(*c);  // the shared expert is expert E
    if (use_stream_path(c))
        return cuda_status(launch_gate_up_stream(g, x_perm, offsets, w_gate_up, s_gate_up, h, s));
    int* status = at<int>(ws, ws_layout(*c).status);
    if (c->flags & MOE_FLAG_FP4_WEIGHTS) {
        if (!pair_gemm_supported(*c)) return MOE_ERR_UNSUPPORTED_SHAPE;
        return cuda_status(
            launch_gate_up_gemm_pair_fp4(g, x_perm, offsets, w_gate_up, s_gate_up, h, status, s));
    }
    if (c->flags & MOE_FLAG_FP8_WEIGHTS) {
        if (!pair_gemm_supported(*c)) return MOE_ERR_UNSUPPORTED_SHAPE;
        return cuda_status(launch_gate_up_gemm_pair_fp8(g, x_perm, offsets, w_gate_up,
                                                        static_cast<const float*>(s_gate_up), h,
                                                        status, s));
    }
    if (pair_gemm_supported(*c))
        return cuda_status(
            launch_gate_up_gemm_pair(g, x_perm, offsets, w_gate_up, packed(c), h, status, s));
    return cuda_status(launch_gate_up_gemm(g, x_perm, offsets, w_gate_up, h, status, s));
}

// gate_up on token rows gathered by index: the bf16 SM-pair GEMM gathers the
// rows of x itself (TMA tile::gather4); every other path first gathers them
// into the workspace's x_perm region with a copy kernel.
int experts_gate_up_gather(const moe_config* c, const void* x, const int32_t* token_of_row,
                           const int32_t* offsets, const void* w_gate_up, const void* s_gate_up,
                           void* h, void* ws, cudaStream_t s) {
    const WsLayout L = ws_layout(*c);
    if (!use_stream_path(c) && !quantised(c) && pair_gemm_supported(*c))
        return cuda_status(launch_gate_up_gemm_pair_gather(grouped_config(*c), x, token_of_row,
                                                           offsets, w_gate_up, packed(c), h,
                                                           at<int>(ws, L.status), s));
    void* xperm = at<void>(ws, L.xperm);
    MOE_TRY(cuda_status(launch_gather_rows(*c, x, token_of_row, offsets, xperm, s)));
    return experts_gate_up(c, xperm, offsets, w_gate_up, s_gate_up, h, ws, s);
}

int experts_down(const moe_config* c, const void* h, const int32_t* offsets, const void* w_down,
                 const void* s_down, void* y, void* ws, cudaStream_t s) {
    const moe_config g = grouped_config(*c);
    if (use_stream_path(c))
        return cuda_status(launch_down_stream(g, h, offsets, w_down, s_down, y, s));
    int* status = at<int>(ws, ws_layout(*c).status);
    if (c->flags & MOE_FLAG_FP4_WEIGHTS) {
        if (!pair_gemm_supported(*c)) return MOE_ERR_UNSUPPORTED_SHAPE;
        return cuda_status(
            launch_down_gemm_pair_fp4(g, h, offsets, w_down, s_down, y, status, s));
    }
    if (c->flags & MOE_FLAG_FP8_WEIGHTS) {
        if (!pair_gemm_supported(*c)) return MOE_ERR_UNSUPPORTED_SHAPE;
        return cuda_status(
            launch_down_gemm_pair_fp8(g, h, offsets, w_down, static_cast<const float*>(s_down),
                                      y, status, s));
    }
    if (pair_gemm_supported(*c))
        return cuda_status(launch_down_gemm_pair(g, h, offsets, w_down, packed(c), y, status, s));
    return cuda_status(launch_down_gemm(g, h, offsets, w_down, y, status, s));
}

// Batches of at most MOE_GATHER_MAX_SLOTS grouped token-slots gather in the GEMM.
bool gather_batch(const moe_config* c) {
    return (long long)c->T * (c->k + shared_slots(*c)) <= MOE_GATHER_MAX_SLOTS;
}

}  // namespace

extern "C" {

size_t moe_workspace_size(const moe_config* cfg) {
    if (check_cfg(cfg) != MOE_OK) return 0;
    return ws_layout(*cfg).total;
}

int moe_workspace_init(const moe_config* cfg, void* ws, size_t ws_bytes, void* stream) {
    MOE_TRY(check_cfg(cfg));
    MOE_TRY(check_ws(cfg, ws, ws_bytes));
    return cuda_status(cudaMemsetAsync(ws, 0, ws_layout(*cfg).control_end,
                                       static_cast<cudaStream_t>(stream)));
}

int moe_route3(const moe_config* cfg, const void* x, const void* w_gate, const float* gate_bias,
               const moe_route_options* opt, int32_t* topk_idx, float* topk_w, void* ws,
               size_t ws_bytes, void* stream) {
    MOE_TRY(check_cfg(cfg));
    if (!x || !w_gate || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_gate)) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_route_options(opt));
    MOE_TRY(check_ws(cfg, ws, ws_bytes));
    return cuda_status(route(cfg, x, w_gate, gate_bias, opt, topk_idx, topk_w, ws,
                             static_cast<cudaStream_t>(stream)));
}

int moe_route2(const moe_config* cfg, const void* x, const void* w_gate, const float* gate_bias,
               const float* score_bias, int32_t* topk_idx, float* topk_w, void* ws,
               size_t ws_bytes, void* stream) {
    const moe_route_options opt = {score_bias, nullptr, 0.f, MOE_SCORE_SIGMOID};
    return moe_route3(cfg, x, w_gate, gate_bias, &opt, topk_idx, topk_w, ws, ws_bytes, stream);
}

int moe_route(const moe_config* cfg, const void* x, const void* w_gate, const float* gate_bias,
              int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes, void* stream) {
    return moe_route2(cfg, x, w_gate, gate_bias, nullptr, topk_idx, topk_w, ws, ws_bytes, stream);
}

int moe_permute(const moe_config* cfg, const int32_t* topk_idx, const void* x, int32_t* counts,
                int32_t* offsets, int32_t* row_of, void* x_perm, void* ws, size_t ws_bytes,
                void* stream) {
    MOE_TRY(check_cfg(cfg));
    if (!topk_idx || !x || !counts || !offsets || !row_of || !x_perm) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_ws(cfg, ws, ws_bytes));
    const WsLayout L = ws_layout(*cfg);
    return cuda_status(launch_permute(*cfg, topk_idx, x, counts, offsets, row_of, x_perm,
                                      at<int32_t>(ws, L.hist), at<int32_t>(ws, L.rank),
                                      static_cast<cudaStream_t>(stream)));
}

int moe_permute_index(const moe_config* cfg, const int32_t* topk_idx, int32_t* counts,
                      int32_t* offsets, int32_t* row_of, int32_t* token_of_row, void* ws,
                      size_t ws_bytes, void* stream) {
    MOE_TRY(check_cfg(cfg));
    if (!topk_idx || !counts || !offsets || !row_of || !token_of_row) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_ws(cfg, ws, ws_bytes));
    const WsLayout L = ws_layout(*cfg);
    return cuda_status(launch_permute_index(*cfg, topk_idx, counts, offsets, row_of, token_of_row,
                                            at<int32_t>(ws, L.hist), at<int32_t>(ws, L.rank),
                                            static_cast<cudaStream_t>(stream)));
}

int moe_expert_gate_up_gather(const moe_config* cfg, const void* x, const int32_t* token_of_row,
                              const int32_t* offsets, const void* w_gate_up,
                              const void* s_gate_up, void* h, void* ws, size_t ws_bytes,
                              void* stream) {
    MOE_TRY(check_cfg(cfg));
    if (!x || !token_of_row || !offsets || !h || !aligned16(x) || !aligned16(h))
        return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_expert_weights(cfg, w_gate_up, s_gate_up));
    MOE_TRY(check_ws(cfg, ws, ws_bytes));
    return experts_gate_up_gather(cfg, x, token_of_row, offsets, w_gate_up, s_gate_up, h, ws,
                                  static_cast<cudaStream_t>(stream));
}

int moe_expert_gate_up(const moe_config* cfg, const void* x_perm, const int32_t* offsets,
                       const void* w_gate_up, const void* s_gate_up, void* h, void* ws,
                       size_t ws_bytes, void* stream) {
    MOE_TRY(check_cfg(cfg));
    if (!x_perm || !offsets || !h || !aligned16(x_perm) || !aligned16(h))
        return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_expert_weights(cfg, w_gate_up, s_gate_up));
    MOE_TRY(check_ws(cfg, ws, ws_bytes));
    return experts_gate_up(cfg, x_perm, offsets, w_gate_up, s_gate_up, h, ws,
                           static_cast<cudaStream_t>(stream));
}

int moe_expert_down(const moe_config* cfg, const void* h, const int32_t* offsets,
                    const void* w_down, const void* s_down, void* y, void* ws, size_t ws_bytes,
                    void* stream) {
    MOE_TRY(check_cfg(cfg));
    if (!h || !offsets || !y || !aligned16(h) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_expert_weights(cfg, w_down, s_down));
    MOE_TRY(check_ws(cfg, ws, ws_bytes));
    return experts_down(cfg, h, offsets, w_down, s_down, y, ws, static_cast<cudaStream_t>(stream));
}

int moe_experts(const moe_config* cfg, const void* x_perm, const int32_t* offsets,
                const void* w_gate_up, const void* s_gate_up, const void* w_down,
                const void* s_down, void* y, void* ws, size_t ws_bytes, void* stream) {
    MOE_TRY(check_cfg(cfg));
    if (!x_perm || !offsets || !y || !aligned16(x_perm) || !aligned16(y))
        return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_expert_weights(cfg, w_gate_up, s_gate_up));
    MOE_TRY(check_expert_weights(cfg, w_down, s_down));
    MOE_TRY(check_ws(cfg, ws, ws_bytes));
    const WsLayout L = ws_layout(*cfg);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    void* h = at<void>(ws, L.h);
    MOE_TRY(experts_gate_up(cfg, x_perm, offsets, w_gate_up, s_gate_up, h, ws, s));
    return experts_down(cfg, h, offsets, w_down, s_down, y, ws, s);
}

int moe_combine(const moe_config* cfg, const void* y, const int32_t* row_of, const float* topk_w,
                void* out, void* ws, size_t ws_bytes, void* stream) {
    MOE_TRY(check_cfg(cfg));
    if (!y || !row_of || !topk_w || !out || !aligned16(y) || !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_ws(cfg, ws, ws_bytes));
    return cuda_status(launch_combine(*cfg, y, row_of, topk_w, out,
                                      static_cast<cudaStream_t>(stream)));
}

int moe_forward3(const moe_config* cfg, const void* x, const void* w_gate, const float* gate_bias,
                 const moe_route_options* opt, const void* w_gate_up, const void* s_gate_up,
                 const void* w_down, const void* s_down, void* out, void* ws, size_t ws_bytes,
                 void* stream) {
    MOE_TRY(check_cfg(cfg));
    MOE_TRY(check_route_options(opt));
    if (!x || !w_gate || !out || !aligned16(x) || !aligned16(w_gate) || !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_expert_weights(cfg, w_gate_up, s_gate_up));
    MOE_TRY(check_expert_weights(cfg, w_down, s_down));
    MOE_TRY(check_ws(cfg, ws, ws_bytes));
    const WsLayout L = ws_layout(*cfg);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* idx = at<int32_t>(ws, L.idx);
    float* w = at<float>(ws, L.w);
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* row_of = at<int32_t>(ws, L.row_of);
    int32_t* counts = at<int32_t>(ws, L.counts);
    int32_t* hist = at<int32_t>(ws, L.hist);
    int32_t* rank = at<int32_t>(ws, L.rank);
    void* h = at<void>(ws, L.h);
    void* y = at<void>(ws, L.y);
    MOE_TRY(cuda_status(cudaMemsetAsync(ws, 0, L.control_end, s)));
    MOE_TRY(cuda_status(route(cfg, x, w_gate, gate_bias, opt, idx, w, ws, s)));
    if (gather_batch(cfg)) {
        int32_t* tok = at<int32_t>(ws, L.tok);
        MOE_TRY(cuda_status(
            launch_permute_index(*cfg, idx, counts, offsets, row_of, tok, hist, rank, s)));
        MOE_TRY(experts_gate_up_gather(cfg, x, tok, offsets, w_gate_up, s_gate_up, h, ws, s));
    } else {
        void* xperm = at<void>(ws, L.xperm);
        MOE_TRY(cuda_status(
            launch_permute(*cfg, idx, x, counts, offsets, row_of, xperm, hist, rank, s)));
        MOE_TRY(experts_gate_up(cfg, xperm, offsets, w_gate_up, s_gate_up, h, ws, s));
    }
    MOE_TRY(experts_down(cfg, h, offsets, w_down, s_down, y, ws, s));
    return cuda_status(launch_combine(*cfg, y, row_of, w, out, s));
}

int moe_forward2(const moe_config* cfg, const void* x, const void* w_gate, const float* gate_bias,
                 const float* score_bias, const void* w_gate_up, const void* s_gate_up,
                 const void* w_down, const void* s_down, void* out, void* ws, size_t ws_bytes,
                 void* stream) {
    const moe_route_options opt = {score_bias, nullptr, 0.f, MOE_SCORE_SIGMOID};
    return moe_forward3(cfg, x, w_gate, gate_bias, &opt, w_gate_up, s_gate_up, w_down, s_down,
                        out, ws, ws_bytes, stream);
}

int moe_forward(const moe_config* cfg, const void* x, const void* w_gate, const float* gate_bias,
                const void* w_gate_up, const void* s_gate_up, const void* w_down,
                const void* s_down, void* out, void* ws, size_t ws_bytes, void* stream) {
    return moe_forward3(cfg, x, w_gate, gate_bias, nullptr, w_gate_up, s_gate_up, w_down, s_down,
                        out, ws, ws_bytes, stream);
}

int moe_pack_weights(const moe_config* cfg, int which, const void* w, void* w_packed,
                     void* stream) {
    MOE_TRY(check_cfg(cfg));
    if (cfg->flags & (MOE_FLAG_FP8_WEIGHTS | MOE_FLAG_FP4_WEIGHTS)) return MOE_ERR_INVALID_ARG;
    if (which != MOE_WEIGHTS_GATE_UP && which != MOE_WEIGHTS_DOWN) return MOE_ERR_INVALID_ARG;
    if (!w || !w_packed || !aligned16(w) || !aligned16(w_packed)) return MOE_ERR_INVALID_ARG;
    if (!pair_gemm_supported(*cfg)) return MOE_ERR_UNSUPPORTED_SHAPE;
    const int rows = which == MOE_WEIGHTS_GATE_UP ? 2 * cfg->d_ff : cfg->d;
    const int cols = which == MOE_WEIGHTS_GATE_UP ? cfg->d : cfg->d_ff;
    const int experts = cfg->E + shared_slots(*cfg);  // the shared expert is packed too
    const size_t bytes = (size_t)experts * rows * cols * 2;
    const char* a = static_cast<const char*>(w);
    const char* b = static_cast<const char*>(w_packed);
    if (a < b + bytes && b < a + bytes) return MOE_ERR_INVALID_ARG;  // overlap
    return cuda_status(launch_pack_weights(experts, rows, cols, w, w_packed,
                                           static_cast<cudaStream_t>(stream)));
}

int moe_read_status(void* ws, void* stream) {
    if (!ws) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t host = 0;
    if (cudaMemcpyAsync(&host, ws, sizeof host, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, sizeof host, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    return host == 0 ? MOE_OK : (host < 0 ? host : MOE_ERR_TIMEOUT);
}

const char* moe_status_string(int code) {
    switch (code) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument (null pointer, misalignment or flags)";
        case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case MOE_ERR_WORKSPACE: return "workspace smaller than moe_workspace_size(cfg)";
        case MOE_ERR_CUDA: return "CUDA launch or runtime error";
        case MOE_ERR_TIMEOUT: return "a bounded device wait gave up";
        default: return "unknown status code";
    }
}

}  // extern "C"
