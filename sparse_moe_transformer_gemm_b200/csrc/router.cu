// router.cu -- fused router: logits GEMM (fp32 accumulate), sigmoid, top-k
// with lowest-index tie-break, renormalisation over the selected scores and
// the router scaling factor.
//
// Method: "Tencent Hy3-295B 架构深度拆解" (pillumina.github.io) §4.1 -- the
// router computes fp32 logits F.linear(x.float(), W.float()), scores them with
// an element-wise sigmoid, selects the top-8, renormalises the selected
// sigmoid scores to sum to 1 and multiplies by router_scaling_factor 2.826.
// The optional per-expert bias is added to the logits before the sigmoid
// (Hy3 commentary, wmrh.cn/news/24252, §3.3).
//
// Structure: CTA (expert block b, token group g, K slice z) computes the
// partial logits of kRouterTokens tokens x kRouterExperts experts over the
// z-th of gridDim.z equal slices of d on CUDA cores and writes them to the fp32
// scratch logits[z][T, E]. Small batches split K so that the grid covers the
// SMs (decode: 64 tokens -> 48 CTAs unsplit, 384 with 8 slices). The last CTA
// of a token group to finish (an arrival counter, no waiting) sums the slices
// in z order and runs the selection: one warp per token, k rounds of a
// warp-wide argmax over the (biased) logits -- the sigmoid is increasing, so
// this selects the k largest scores -- and the sigmoid of the k selected. With
// an e_score_correction_bias ("Tencent Hy3-295B 架构深度拆解" §4.1 step 2) the
// choice ranks sigmoid + bias and the weights renormalise the sigmoid scores.
// With score_fn 1 every "sigmoid" above reads sqrt(softplus(logit)) (the
// V4-Flash router of the same page, §2.2), also increasing in the logit.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int RT = kRouterTokens;    // tokens per CTA
constexpr int RE = kRouterExperts;   // experts per CTA
constexpr int RWARPS = 8;
constexpr int EPW = RE / RWARPS;     // experts per warp
constexpr int KC = 1024;             // x columns staged per chunk
static_assert(RT == RWARPS, "selection uses one warp per token");

__device__ __forceinline__ void load_w(uint4 (&u)[EPW], const __nv_bfloat16* __restrict__ wg,
                                       int e_base, int E, int d, int col) {
#pragma unroll
    for (int a = 0; a < EPW; ++a)
        u[a] = (e_base + a < E) ? *reinterpret_cast<const uint4*>(wg + (size_t)(e_base + a) * d + col)
                                : make_uint4(0, 0, 0, 0);
}

__global__ void __launch_bounds__(RWARPS * 32, kRouterCtasPerSm)
router_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wg,
              const float* __restrict__ bias, const float* __restrict__ sbias,
              const float* __restrict__ norm_w, float norm_eps, int score_fn, int T, int d,
              int E, int k, float scale, float* __restrict__ logits, float* __restrict__ sumsq,
              int* __restrict__ counters, int* __restrict__ idx_out, float* __restrict__ w_out) {
    pdl_launch_and_wait();
    __shared__ __align__(16) float xs[RT][KC];
    __shared__ int s_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e_base = blockIdx.x * RE + warp * EPW;
    const int t0 = blockIdx.y * RT;
    const int ks = gridDim.z;
    const int dk = d / ks;  // a multiple of 128
    const int k0 = blockIdx.z * dk;

    float acc[EPW][RT];
#pragma unroll
    for (int a = 0; a < EPW; ++a)
#pragma unroll
        for (int b = 0; b < RT; ++b) acc[a][b] = 0.f;
    float ss_tok = 0.f;  // route_norm: sum of squares of token t0 + warp over this slice

    for (int kc = k0; kc < k0 + dk; kc += KC) {
        const int kw = min(KC, k0 + dk - kc);  // multiple of 128
        const int v8 = kw / 8;
        __syncthreads();
        for (int v = threadIdx.x; v < RT * v8; v += blockDim.x) {
            const int tt = v / v8, c8 = (v - tt * v8) * 8;
            float f[8];
            if (t0 + tt < T) {
                uint4 u = *reinterpret_cast<const uint4*>(x + (size_t)(t0 + tt) * d + kc + c8);
                bf16x8_to_float(u, f);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = 0.f;
            }
            *reinterpret_cast<float4*>(&xs[tt][c8]) = make_float4(f[0], f[1], f[2], f[3]);
            *reinterpret_cast<float4*>(&xs[tt][c8 + 4]) = make_float4(f[4], f[5], f[6], f[7]);
        }
        __syncthreads();
        if (norm_w) {
            // route_norm: warp w sums the squares of token w's chunk (fixed order),
            // then the chunk is multiplied by the norm weight; 1/rms is applied to
            // the finished logit (logit = (1/rms) sum_c x_c g_c W_ec)
            float ss = 0.f;
            for (int c = lane; c < kw; c += 32) ss = fmaf(xs[warp][c], xs[warp][c], ss);
            ss_tok += warp_sum(ss);
            __syncthreads();
            for (int v = threadIdx.x; v < RT * kw; v += blockDim.x) {
                const int tt = v / kw, c = v - tt * kw;
                xs[tt][c] *= norm_w[kc + c];
            }
            __syncthreads();
        }
        // the weight vectors of the next column step are in flight while the
        // current ones are used
        uint4 cur[EPW];
        load_w(cur, wg, e_base, E, d, kc + lane * 8);
        for (int c = lane * 8; c < kw; c += 256) {
            uint4 nxt[EPW];
            if (c + 256 < kw) load_w(nxt, wg, e_base, E, d, kc + c + 256);
            float wv[EPW][8];
#pragma unroll
            for (int a = 0; a < EPW; ++a) bf16x8_to_float(cur[a], wv[a]);
#pragma unroll
            for (int b = 0; b < RT; ++b) {
                const float4 p = *reinterpret_cast<const float4*>(&xs[b][c]);
                const float4 q = *reinterpret_cast<const float4*>(&xs[b][c + 4]);
#pragma unroll
                for (int a = 0; a < EPW; ++a) {
                    float s = acc[a][b];
                    s = fmaf(wv[a][0], p.x, s); s = fmaf(wv[a][1], p.y, s);
                    s = fmaf(wv[a][2], p.z, s); s = fmaf(wv[a][3], p.w, s);
                    s = fmaf(wv[a][4], q.x, s); s = fmaf(wv[a][5], q.y, s);
                    s = fmaf(wv[a][6], q.z, s); s = fmaf(wv[a][7], q.w, s);
                    acc[a][b] = s;
                }
            }
#pragma unroll
            for (int a = 0; a < EPW; ++a) cur[a] = nxt[a];
        }
    }

#pragma unroll
    for (int a = 0; a < EPW; ++a)
#pragma unroll
        for (int b = 0; b < RT; ++b) acc[a][b] = warp_sum(acc[a][b]);
    if (lane == 0) {
#pragma unroll
        for (int a = 0; a < EPW; ++a)
#pragma unroll
            for (int b = 0; b < RT; ++b) {
                const int e = e_base + a, t = t0 + b;
                if (e < E && t < T) logits[((size_t)blockIdx.z * T + t) * E + e] = acc[a][b];
            }
    }

    if (norm_w && blockIdx.x == 0 && lane == 0 && t0 + warp < T)
        sumsq[(size_t)blockIdx.z * T + t0 + warp] = ss_tok;

    // Arrival: the last expert-block CTA of this token group does the selection.
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int ticket = atomicAdd(&counters[blockIdx.y], 1);
        s_last = (ticket == (int)(gridDim.x * gridDim.z) - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    const int t = t0 + warp;
    if (t < T) {
        // The sigmoid is increasing: select on the (biased) logits, evaluate the
        // sigmoid for the selected ones only.
        float sc[8];  // E <= 256: expert lane + 32*q
#pragma unroll
        for (int q = 0; q < 8; ++q) sc[q] = 0.f;
        // slices summed in order 0, 1, ...; all loads of a slice are independent
#pragma unroll
        for (int p = 0; p < kRouterMaxSplit; ++p) {
            if (p < ks) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int e = lane + 32 * q;
                    if (e < E) sc[q] += __ldcg(logits + ((size_t)p * T + t) * E + e);
                }
            }
        }
        if (norm_w) {
            float ms = 0.f;
            for (int p = 0; p < ks; ++p) ms += __ldcg(sumsq + (size_t)p * T + t);
            const float inv = 1.0f / sqrtf(ms / (float)d + norm_eps);
#pragma unroll
            for (int q = 0; q < 8; ++q) sc[q] *= inv;
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int e = lane + 32 * q;
            if (e < E) {
                if (bias) sc[q] += bias[e];
            } else {
                sc[q] = -INFINITY;
            }
        }
        if (sbias) {
            // e_score_correction_bias: the choice ranks sigmoid + bias, the
            // weights renormalise the sigmoid scores of the chosen experts
            float prob[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int e = lane + 32 * q;
                prob[q] = (e < E) ? score_value(sc[q], score_fn) : 0.f;
                sc[q] = (e < E) ? prob[q] + sbias[e] : -INFINITY;
            }
            warp_select_topk(sc, k, scale, idx_out + (size_t)t * k, w_out + (size_t)t * k, prob,
                             score_fn);
        } else {
            warp_select_topk(sc, k, scale, idx_out + (size_t)t * k, w_out + (size_t)t * k,
                             nullptr, score_fn);
        }
    }
    if (threadIdx.x == 0) counters[blockIdx.y] = 0;
}

}  // namespace

cudaError_t launch_router(const moe_config& c, const void* x, const void* w_gate,
                          const float* gate_bias, const float* score_bias, const float* norm_w,
                          float norm_eps, int score_fn, int32_t* idx, float* w, float* logits,
                          float* sumsq, int32_t* counters, int ksplit, cudaStream_t s) {
    dim3 grid((c.E + RE - 1) / RE, n_router_groups(c), ksplit);
    const cudaError_t err = launch_pdl(
        router_kernel, grid, dim3(RWARPS * 32), 0, s, static_cast<const __nv_bfloat16*>(x),
        static_cast<const __nv_bfloat16*>(w_gate), gate_bias, score_bias, norm_w, norm_eps, score_fn,
        c.T, c.d, c.E, c.k, c.scale, logits, sumsq, counters, idx, w);
    return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
