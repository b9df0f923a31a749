// internal.h -- workspace layout and kernel launchers shared by the library's
// translation units. Not part of the public ABI (that is include/moe.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "../../include/moe.h"

namespace moe {

constexpr int kRouterTokens = 8;        // tokens per router CTA
constexpr int kRouterExperts = 32;      // experts per router CTA (8 warps x 4)
constexpr int kPermuteChunk = 2048;     // token-slots per ranking chunk
constexpr int kStreamMaxTokens = 8;     // rows per pass of the streaming expert kernels

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Launch a kernel of the layer with programmatic stream serialization: it may
// begin launching while the previous kernel on the stream finishes (each
// kernel waits for its predecessor in pdl_launch_and_wait before it touches
// global memory), which hides the launch gap between consecutive kernels.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Byte offsets of every workspace region. The control words (status word and
// router counters) come first so that one memset clears them.
struct WsLayout {
    size_t status;    // int32 status word (+ padding)
    size_t counters;  // int32 [ceil(T / kRouterTokens)] router arrival counters
    size_t control_end;
    size_t logits;    // fp32 [router_ksplit, T, E] partial router logits
    size_t sumsq;     // fp32 [router_ksplit, T] route_norm partial sums of squares
    size_t hist;      // int32 [n_chunks, E]
    size_t rank;      // int32 [T*k]
    size_t idx;       // int32 [T*k]
    size_t w;         // fp32  [T*k]
    size_t counts;    // int32 [E]
    size_t offsets;   // int32 [E+1]
    size_t row_of;    // int32 [T*k]
    size_t tok;       // int32 [T*k] token of each grouped row
    size_t xperm;     // bf16 [T*k, d]
    size_t h;         // bf16 [T*k, d_ff]
    size_t y;         // bf16 [T*k, d]
    size_t sched;     // int32 GEMM tile scheduling scratch
    size_t total;
};

inline int n_router_groups(const moe_config& c) {
    return (c.T + kRouterTokens - 1) / kRouterTokens;
}
constexpr int kRouterCtasPerSm = 2;     // CUDA-core router CTAs resident per SM
constexpr int kRouterMaxSplit = 16;     // K slices of the CUDA-core router at most

// K slices of the CUDA-core router: the largest power of two (at most
// kRouterMaxSplit, keeping d / slices a multiple of 128) whose grid still runs
// in one wave on 148 SMs.
inline int router_ksplit(const moe_config& c) {
    const int base = ((c.E + kRouterExperts - 1) / kRouterExperts) * n_router_groups(c);
    int ks = 1;
    while (2 * ks <= kRouterMaxSplit && base * 2 * ks <= kRouterCtasPerSm * 148 &&
           (c.d / 128) % (2 * ks) == 0)
        ks *= 2;
    return ks;
}
inline int n_permute_chunks(const moe_config& c) {
    long R = (long)c.T * c.k;
    return (int)((R + kPermuteChunk - 1) / kPermuteChunk);
}

// The shared expert (MOE_FLAG_SHARED_EXPERT) is expert E of the weight arrays
// and slot k of every token: the grouping, the expert GEMMs and the combine
// run on the "grouped" configuration with E + 1 experts and k + 1 slots.
inline int shared_slots(const moe_config& c) {
    return (c.flags & MOE_FLAG_SHARED_EXPERT) ? 1 : 0;
}
inline moe_config grouped_config(const moe_config& c) {
    moe_config g = c;
    g.E += shared_slots(c);
    g.k += shared_slots(c);
    return g;
}

inline WsLayout ws_layout(const moe_config& c) {
    WsLayout L{};
    const moe_config g = grouped_config(c);
    size_t R = (size_t)g.T * g.k;
    size_t o = 0;
    L.status = o;   o += 256;
    L.counters = o; o = align256(o + sizeof(int32_t) * n_router_groups(c));
    L.control_end = o;
    L.logits = o;   o = align256(o + sizeof(float) * router_ksplit(c) * (size_t)c.T * c.E);
    L.sumsq = o;    o = align256(o + sizeof(float) * router_ksplit(c) * (size_t)c.T);
    L.hist = o;     o = align256(o + sizeof(int32_t) * (size_t)n_permute_chunks(g) * g.E);
    L.rank = o;     o = align256(o + sizeof(int32_t) * R);
    L.idx = o;      o = align256(o + sizeof(int32_t) * R);
    L.w = o;        o = align256(o + sizeof(float) * R);
    L.counts = o;   o = align256(o + sizeof(int32_t) * g.E);
    L.offsets = o;  o = align256(o + sizeof(int32_t) * (g.E + 1));
    L.row_of = o;   o = align256(o + sizeof(int32_t) * R);
    L.tok = o;      o = align256(o + sizeof(int32_t) * R);
    L.xperm = o;    o = align256(o + 2 * R * c.d);
    L.h = o;        o = align256(o + 2 * R * c.d_ff);
    L.y = o;        o = align256(o + 2 * R * c.d);
    L.sched = o;    o = align256(o + sizeof(int32_t) * 4 * (g.E + 1));
    L.total = o;
    return L;
}

// ---- launchers (each returns cudaError_t of the launch) ----
cudaError_t launch_router(const moe_config& c, const void* x, const void* w_gate,
                          const float* gate_bias, const float* score_bias, const float* norm_w,
                          float norm_eps, int score_fn, int32_t* idx, float* w, float* logits,
                          float* sumsq, int32_t* counters, int ksplit, cudaStream_t s);

bool router_tc_supported(const moe_config& c);
cudaError_t launch_router_tc(const moe_config& c, const void* x, const void* w_gate,
                             const float* gate_bias, const float* score_bias, int score_fn,
                             int32_t* idx, float* w, int* status, cudaStream_t s);

cudaError_t launch_permute(const moe_config& c, const int32_t* idx, const void* x, int32_t* counts,
                           int32_t* offsets, int32_t* row_of, void* x_perm, int32_t* hist,
                           int32_t* rank, cudaStream_t s);

cudaError_t launch_permute_index(const moe_config& c, const int32_t* idx, int32_t* counts,
                                 int32_t* offsets, int32_t* row_of, int32_t* token_of_row,
                                 int32_t* hist, int32_t* rank, cudaStream_t s);
cudaError_t launch_gather_rows(const moe_config& c, const void* x, const int32_t* token_of_row,
                               const int32_t* offsets, void* x_perm, cudaStream_t s);

cudaError_t launch_gate_up_stream(const moe_config& c, const void* x_perm, const int32_t* offsets,
                                  const void* w_gate_up, const void* s_gate_up, void* h,
                                  cudaStream_t s);
cudaError_t launch_down_stream(const moe_config& c, const void* h, const int32_t* offsets,
                               const void* w_down, const void* s_down, void* y, cudaStream_t s);

cudaError_t launch_gate_up_gemm(const moe_config& c, const void* x_perm, const int32_t* offsets,
                                const void* w_gate_up, void* h, int* status, cudaStream_t s);
cudaError_t launch_down_gemm(const moe_config& c, const void* h, const int32_t* offsets,
                             const void* w_down, void* y, int* status, cudaStream_t s);

bool pair_gemm_supported(const moe_config& c);
cudaError_t launch_gate_up_gemm_pair(const moe_config& c, const void* x_perm,
                                     const int32_t* offsets, const void* w_gate_up, bool packed,
                                     void* h, int* status, cudaStream_t s);
cudaError_t launch_down_gemm_pair(const moe_config& c, const void* h, const int32_t* offsets,
                                  const void* w_down, bool packed, void* y, int* status,
                                  cudaStream_t s);
cudaError_t launch_gate_up_gemm_pair_gather(const moe_config& c, const void* x,
                                            const int32_t* token_of_row, const int32_t* offsets,
                                            const void* w_gate_up, bool packed, void* h,
                                            int* status, cudaStream_t s);
// Rearranges E x [rows, cols] bf16 into 128 x 64 blocks (see MOE_FLAG_PACKED_WEIGHTS).
cudaError_t launch_pack_weights(int E, int rows, int cols, const void* w, void* w_packed,
                                cudaStream_t s);

cudaError_t launch_gate_up_gemm_pair_fp8(const moe_config& c, const void* x_perm,
                                         const int32_t* offsets, const void* w_gate_up,
                                         const float* s_gate_up, void* h, int* status,
                                         cudaStream_t s);
cudaError_t launch_down_gemm_pair_fp8(const moe_config& c, const void* h, const int32_t* offsets,
                                      const void* w_down, const float* s_down, void* y,
                                      int* status, cudaStream_t s);

cudaError_t launch_ep_row_experts(const int32_t* counts, int n_src, int e_local,
                                  int32_t* expert_of_row, int n_rows, cudaStream_t s);

// FP4 (E2M1 codes + E8M0 block-32 scales) on the same SM-pair kernels.
cudaError_t launch_gate_up_gemm_pair_fp4(const moe_config& c, const void* x_perm,
                                         const int32_t* offsets, const void* w_gate_up,
                                         const void* s_gate_up, void* h, int* status,
                                         cudaStream_t s);
cudaError_t launch_down_gemm_pair_fp4(const moe_config& c, const void* h, const int32_t* offsets,
                                      const void* w_down, const void* s_down, void* y,
                                      int* status, cudaStream_t s);

cudaError_t launch_combine(const moe_config& c, const void* y, const int32_t* row_of,
                           const float* topk_w, void* out, cudaStream_t s);

}  // namespace moe
