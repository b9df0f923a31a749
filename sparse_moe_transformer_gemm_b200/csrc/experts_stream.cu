// experts_stream.cu -- weight-streaming SwiGLU experts for few rows per expert.
//
// Decode-sized batches route ~2-3 rows to each expert, so the expert step is
// bound by reading the touched experts' weights once ("Tencent Hy3-Flash QA"
// Q3.4: decode reads every active parameter per token). These kernels stream
// each touched expert's weight rows exactly once per pass with 16-byte
// non-allocating loads, keep the expert's (<= kStreamMaxTokens) activation
// rows in shared memory and accumulate in fp32 on the CUDA cores. Experts with
// no rows cost one early-exiting CTA column. More rows than kStreamMaxTokens
// are handled in passes (correct for any count, efficient only for few).
//
// gate_up: h[r, f] = bf16( SiLU(<x_r, W[e, f]>) * <x_r, W[e, F + f]> )
// down:    y[r, i] = bf16( <h_r, Wd[e, i]> )
// SwiGLU as in "DeepSeek V4-Flash 架构 QA" Q4.5; expert tensor shapes as in
// "Tencent Hy3-295B 架构深度拆解" §2.3. FP8 weights: the dot product runs on
// the e4m3 codes and the row's fp32 scale multiplies the finished sum.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int SWARPS = 8;
constexpr int ROWS_PER_WARP = 4;                  // output rows per warp per CTA
constexpr int ROWS_PER_CTA = SWARPS * ROWS_PER_WARP;
constexpr int NTMAX = kStreamMaxTokens;

// acc_a[t] += <wa, xs[t]>, acc_b[t] += <wb, xs[t]> over this lane's share of a
// row of L elements. xs: NT rows of L bf16 in shared memory.
template <int NT, bool FP8>
__device__ __forceinline__ void pair_dots(const uint8_t* __restrict__ wa,
                                          const uint8_t* __restrict__ wb,
                                          const __nv_bfloat16* xs, int L, int lane,
                                          float (&acc_a)[NT], float (&acc_b)[NT]) {
    constexpr int EPV = FP8 ? 16 : 8;   // elements per 16-byte vector
    constexpr int BPE = FP8 ? 1 : 2;    // bytes per element
    constexpr int U = FP8 ? 2 : 4;      // vectors per row in flight per lane
    for (int c0 = lane * EPV; c0 < L; c0 += 32 * EPV * U) {
        uint4 va[U], vb[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + u * 32 * EPV;
            if (c < L) {
                va[u] = ld_stream_u4(wa + (size_t)c * BPE);
                vb[u] = ld_stream_u4(wb + (size_t)c * BPE);
            } else {
                va[u] = make_uint4(0, 0, 0, 0);
                vb[u] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + u * 32 * EPV;
            if (c >= L) break;
            float fa[EPV], fb[EPV];
            if constexpr (FP8) {
                e4m3x16_to_float(va[u], fa);
                e4m3x16_to_float(vb[u], fb);
            } else {
                bf16x8_to_float(va[u], fa);
                bf16x8_to_float(vb[u], fb);
            }
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                float xf[EPV];
                const uint4* xp = reinterpret_cast<const uint4*>(xs + (size_t)t * L + c);
                bf16x8_to_float(xp[0], xf);
                if constexpr (FP8) bf16x8_to_float(xp[1], xf + 8);
                float sa = acc_a[t], sb = acc_b[t];
#pragma unroll
                for (int i = 0; i < EPV; ++i) {
                    sa = fmaf(fa[i], xf[i], sa);
                    sb = fmaf(fb[i], xf[i], sb);
                }
                acc_a[t] = sa;
                acc_b[t] = sb;
            }
        }
    }
}

template <int NT, bool FP8>
__device__ void gate_up_rows(const uint8_t* __restrict__ wexp, const float* __restrict__ s_exp,
                             const __nv_bfloat16* xs, int d, int F, int f_base, int lane,
                             __nv_bfloat16* __restrict__ h, long row0) {
    constexpr int BPE = FP8 ? 1 : 2;
    for (int i = 0; i < ROWS_PER_WARP; ++i) {
        const int f = f_base + i;
        if (f >= F) break;
        float g[NT], u[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) g[t] = u[t] = 0.f;
        pair_dots<NT, FP8>(wexp + (size_t)f * d * BPE, wexp + (size_t)(F + f) * d * BPE, xs, d,
                           lane, g, u);
        const float sg = FP8 ? s_exp[f] : 1.f, su = FP8 ? s_exp[F + f] : 1.f;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const float gt = warp_sum(g[t]) * sg, ut = warp_sum(u[t]) * su;
            if (lane == t) {
                const float hv = silu_mul(gt, ut);
                reinterpret_cast<uint16_t*>(h)[(row0 + t) * F + f] = float_to_bf16_bits(hv);
            }
        }
    }
}

template <int NT, bool FP8>
__device__ void down_rows(const uint8_t* __restrict__ wexp, const float* __restrict__ s_exp,
                          const __nv_bfloat16* hs, int d, int F, int i_base, int lane,
                          __nv_bfloat16* __restrict__ y, long row0) {
    constexpr int BPE = FP8 ? 1 : 2;
    for (int p = 0; p < ROWS_PER_WARP; p += 2) {
        const int i = i_base + p;
        if (i >= d) break;
        float a[NT], b[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) a[t] = b[t] = 0.f;
        pair_dots<NT, FP8>(wexp + (size_t)i * F * BPE, wexp + (size_t)(i + 1) * F * BPE, hs, F,
                           lane, a, b);
        const float sa = FP8 ? s_exp[i] : 1.f, sb = FP8 ? s_exp[i + 1] : 1.f;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const float at = warp_sum(a[t]) * sa, bt = warp_sum(b[t]) * sb;
            if (lane == t) {
                const uint32_t packed = pack_bf16x2(at, bt);
                *reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(y) + (row0 + t) * d + i) =
                    packed;
            }
        }
    }
}

// Copy nt rows of L bf16 starting at src into shared memory.
__device__ __forceinline__ void stage_rows(__nv_bfloat16* dst, const __nv_bfloat16* src, int nt,
                                           int L) {
    const uint4* s = reinterpret_cast<const uint4*>(src);
    uint4* t = reinterpret_cast<uint4*>(dst);
    for (int v = threadIdx.x; v < nt * L / 8; v += blockDim.x) t[v] = s[v];
}

template <bool FP8>
__global__ void __launch_bounds__(SWARPS * 32)
gate_up_stream_kernel(const __nv_bfloat16* __restrict__ xperm, const int* __restrict__ offsets,
                      const uint8_t* __restrict__ wgu, const float* __restrict__ s_gu,
                      __nv_bfloat16* __restrict__ h, int d, int F) {
    extern __shared__ __align__(16) uint8_t smem[];
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem);
    const int e = blockIdx.y;
    const int r0 = offsets[e];
    const int n = offsets[e + 1] - r0;
    if (n <= 0) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int f_base = blockIdx.x * ROWS_PER_CTA + warp * ROWS_PER_WARP;
    constexpr size_t BPE = FP8 ? 1 : 2;
    const uint8_t* wexp = wgu + (size_t)e * 2 * F * d * BPE;
    const float* sexp = FP8 ? s_gu + (size_t)e * 2 * F : nullptr;
    for (int p = 0; p < n; p += NTMAX) {
        const int nt = min(NTMAX, n - p);
        __syncthreads();
        stage_rows(xs, xperm + (size_t)(r0 + p) * d, nt, d);
        __syncthreads();
        const long row0 = (long)r0 + p;
        switch (nt) {
            case 1: gate_up_rows<1, FP8>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
            case 2: gate_up_rows<2, FP8>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
            case 3: gate_up_rows<3, FP8>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
            case 4: gate_up_rows<4, FP8>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
            case 5: gate_up_rows<5, FP8>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
            case 6: gate_up_rows<6, FP8>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
            case 7: gate_up_rows<7, FP8>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
            default: gate_up_rows<8, FP8>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
        }
    }
}

template <bool FP8>
__global__ void __launch_bounds__(SWARPS * 32)
down_stream_kernel(const __nv_bfloat16* __restrict__ h, const int* __restrict__ offsets,
                   const uint8_t* __restrict__ wd, const float* __restrict__ s_d,
                   __nv_bfloat16* __restrict__ y, int d, int F) {
    extern __shared__ __align__(16) uint8_t smem[];
    __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(smem);
    const int e = blockIdx.y;
    const int r0 = offsets[e];
    const int n = offsets[e + 1] - r0;
    if (n <= 0) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i_base = blockIdx.x * ROWS_PER_CTA + warp * ROWS_PER_WARP;
    constexpr size_t BPE = FP8 ? 1 : 2;
    const uint8_t* wexp = wd + (size_t)e * d * F * BPE;
    const float* sexp = FP8 ? s_d + (size_t)e * d : nullptr;
    for (int p = 0; p < n; p += NTMAX) {
        const int nt = min(NTMAX, n - p);
        __syncthreads();
        stage_rows(hs, h + (size_t)(r0 + p) * F, nt, F);
        __syncthreads();
        const long row0 = (long)r0 + p;
        switch (nt) {
            case 1: down_rows<1, FP8>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
            case 2: down_rows<2, FP8>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
            case 3: down_rows<3, FP8>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
            case 4: down_rows<4, FP8>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
            case 5: down_rows<5, FP8>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
            case 6: down_rows<6, FP8>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
            case 7: down_rows<7, FP8>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
            default: down_rows<8, FP8>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
        }
    }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

cudaError_t launch_gate_up_stream(const moe_config& c, const void* x_perm, const int32_t* offsets,
                                  const void* w_gate_up, const float* s_gate_up, void* h,
                                  cudaStream_t s) {
    const bool fp8 = (c.flags & MOE_FLAG_FP8_WEIGHTS) != 0;
    const size_t smem = (size_t)NTMAX * c.d * 2;
    dim3 grid((c.d_ff + ROWS_PER_CTA - 1) / ROWS_PER_CTA, c.E);
    cudaError_t err;
    if (fp8) {
        if ((err = set_smem(gate_up_stream_kernel<true>, smem)) != cudaSuccess) return err;
        gate_up_stream_kernel<true><<<grid, SWARPS * 32, smem, s>>>(
            static_cast<const __nv_bfloat16*>(x_perm), offsets,
            static_cast<const uint8_t*>(w_gate_up), s_gate_up, static_cast<__nv_bfloat16*>(h),
            c.d, c.d_ff);
    } else {
        if ((err = set_smem(gate_up_stream_kernel<false>, smem)) != cudaSuccess) return err;
        gate_up_stream_kernel<false><<<grid, SWARPS * 32, smem, s>>>(
            static_cast<const __nv_bfloat16*>(x_perm), offsets,
            static_cast<const uint8_t*>(w_gate_up), nullptr, static_cast<__nv_bfloat16*>(h), c.d,
            c.d_ff);
    }
    return cudaGetLastError();
}

cudaError_t launch_down_stream(const moe_config& c, const void* h, const int32_t* offsets,
                               const void* w_down, const float* s_down, void* y, cudaStream_t s) {
    const bool fp8 = (c.flags & MOE_FLAG_FP8_WEIGHTS) != 0;
    const size_t smem = (size_t)NTMAX * c.d_ff * 2;
    dim3 grid((c.d + ROWS_PER_CTA - 1) / ROWS_PER_CTA, c.E);
    cudaError_t err;
    if (fp8) {
        if ((err = set_smem(down_stream_kernel<true>, smem)) != cudaSuccess) return err;
        down_stream_kernel<true><<<grid, SWARPS * 32, smem, s>>>(
            static_cast<const __nv_bfloat16*>(h), offsets, static_cast<const uint8_t*>(w_down),
            s_down, static_cast<__nv_bfloat16*>(y), c.d, c.d_ff);
    } else {
        if ((err = set_smem(down_stream_kernel<false>, smem)) != cudaSuccess) return err;
        down_stream_kernel<false><<<grid, SWARPS * 32, smem, s>>>(
            static_cast<const __nv_bfloat16*>(h), offsets, static_cast<const uint8_t*>(w_down),
            nullptr, static_cast<__nv_bfloat16*>(y), c.d, c.d_ff);
    }
    return cudaGetLastError();
}

}  // namespace moe
