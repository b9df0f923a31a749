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
// "Tencent Hy3-295B 架构深度拆解" §2.3. Three weight formats:
//   bf16;
//   FP8: e4m3 codes, and the row's fp32 scale multiplies the finished sum;
//   FP4 (the V4-Flash column of the same page, §2.2): E2M1 codes two to a
//     byte; one E8M0 scale per 32 consecutive elements of a row, so one
//     16-byte vector is one scale block; the block's power-of-two scale
//     multiplies each token's partial sum over the block's codes.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

enum WFmt : int { kBF16 = 0, kFP8 = 1, kFP4 = 2 };

constexpr int SWARPS = 8;
constexpr int ROWS_PER_WARP = 4;                  // output rows per warp per CTA
constexpr int ROWS_PER_CTA = SWARPS * ROWS_PER_WARP;
constexpr int NTMAX = kStreamMaxTokens;

// Bytes of a weight row of L elements.
template <int FMT>
__host__ __device__ constexpr size_t row_bytes(int L) {
    return FMT == kBF16 ? (size_t)L * 2 : FMT == kFP8 ? (size_t)L : (size_t)L / 2;
}

// FP4 half block: acc_a[t] += sa * <fa, xs[t][c, c+16)> and likewise for b,
// with fa / fb the codes' values (the block's power-of-two scale multiplies
// each token's 16-element partial sum: 2 NT multiplies instead of 32).
template <int NT>
__device__ __forceinline__ void dot16_rows(const float (&fa)[16], const float (&fb)[16], float sa,
                                           float sb, const __nv_bfloat16* xs, int L, int c,
                                           float (&acc_a)[NT], float (&acc_b)[NT]) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const uint4* xp = reinterpret_cast<const uint4*>(xs + (size_t)t * L + c);
        float xf[16];
        bf16x8_to_float(xp[0], xf);
        bf16x8_to_float(xp[1], xf + 8);
        float ra = 0.f, rb = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            ra = fmaf(fa[i], xf[i], ra);
            rb = fmaf(fb[i], xf[i], rb);
        }
        acc_a[t] = fmaf(ra, sa, acc_a[t]);
        acc_b[t] = fmaf(rb, sb, acc_b[t]);
    }
}

// acc_a[t] += <wa, xs[t]>, acc_b[t] += <wb, xs[t]> over this lane's share of a
// row of L elements. xs: NT rows of L bf16 in shared memory. FP4: qa / qb are
// the two rows' E8M0 block scales (L / 32 bytes each).
template <int NT, int FMT>
__device__ __forceinline__ void pair_dots(const uint8_t* __restrict__ wa,
                                          const uint8_t* __restrict__ wb,
                                          const uint8_t* __restrict__ qa,
                                          const uint8_t* __restrict__ qb,
                                          const __nv_bfloat16* xs, int L, int lane,
                                          float (&acc_a)[NT], float (&acc_b)[NT]) {
    constexpr int EPV = FMT == kBF16 ? 8 : FMT == kFP8 ? 16 : 32;  // elements per vector
    constexpr int U = FMT == kBF16 ? 4 : 2;  // vectors per row in flight per lane
    for (int c0 = lane * EPV; c0 < L; c0 += 32 * EPV * U) {
        uint4 va[U], vb[U];
        uint32_t ea[U], eb[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + u * 32 * EPV;
            ea[u] = eb[u] = 0u;
            if (c < L) {
                va[u] = ld_stream_u4(wa + row_bytes<FMT>(c));
                vb[u] = ld_stream_u4(wb + row_bytes<FMT>(c));
                if constexpr (FMT == kFP4) {
                    ea[u] = __ldg(qa + c / 32);
                    eb[u] = __ldg(qb + c / 32);
                }
            } else {
                va[u] = make_uint4(0, 0, 0, 0);
                vb[u] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + u * 32 * EPV;
            if (c >= L) break;
            if constexpr (FMT == kFP4) {
                // two halves of 16 elements, each a scaled partial sum per token
                const float sa = e8m0_to_float(ea[u]), sb = e8m0_to_float(eb[u]);
                const uint32_t wa4[4] = {va[u].x, va[u].y, va[u].z, va[u].w};
                const uint32_t wb4[4] = {vb[u].x, vb[u].y, vb[u].z, vb[u].w};
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float fa[16], fb[16];
                    e2m1x16_to_float(wa4[2 * half], wa4[2 * half + 1], fa);
                    e2m1x16_to_float(wb4[2 * half], wb4[2 * half + 1], fb);
                    dot16_rows<NT>(fa, fb, sa, sb, xs, L, c + 16 * half, acc_a, acc_b);
                }
            } else {
                float fa[EPV], fb[EPV];
                if constexpr (FMT == kFP8) {
                    e4m3x16_to_float(va[u], fa);
                    e4m3x16_to_float(vb[u], fb);
                } else {
                    bf16x8_to_float(va[u], fa);
                    bf16x8_to_float(vb[u], fb);
                }
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const uint4* xp = reinterpret_cast<const uint4*>(xs + (size_t)t * L + c);
                    float xf[EPV];
                    bf16x8_to_float(xp[0], xf);
                    if constexpr (FMT == kFP8) bf16x8_to_float(xp[1], xf + 8);
                    float ra = acc_a[t], rb = acc_b[t];
#pragma unroll
                    for (int i = 0; i < EPV; ++i) {
                        ra = fmaf(fa[i], xf[i], ra);
                        rb = fmaf(fb[i], xf[i], rb);
                    }
                    acc_a[t] = ra;
                    acc_b[t] = rb;
                }
            }
        }
    }
}

// Scales of one expert (sexp): FP8 fp32 [rows], one per row; FP4 E8M0 bytes
// [rows, L / 32], one per 32-element block of a row.
template <int FMT>
__device__ __forceinline__ float row_scale(const void* sexp, int r) {
    return FMT == kFP8 ? static_cast<const float*>(sexp)[r] : 1.f;
}
template <int FMT>
__device__ __forceinline__ const uint8_t* block_scales(const void* sexp, int r, int L) {
    return FMT == kFP4 ? static_cast<const uint8_t*>(sexp) + (size_t)r * (L / 32) : nullptr;
}

template <int NT, int FMT>
__device__ void gate_up_rows(const uint8_t* __restrict__ wexp, const void* sexp,
                             const __nv_bfloat16* xs, int d, int F, int f_base, int lane,
                             __nv_bfloat16* __restrict__ h, long row0) {
    for (int i = 0; i < ROWS_PER_WARP; ++i) {
        const int f = f_base + i;
        if (f >= F) break;
        float g[NT], u[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) g[t] = u[t] = 0.f;
        pair_dots<NT, FMT>(wexp + (size_t)f * row_bytes<FMT>(d),
                           wexp + (size_t)(F + f) * row_bytes<FMT>(d),
                           block_scales<FMT>(sexp, f, d), block_scales<FMT>(sexp, F + f, d), xs,
                           d, lane, g, u);
        const float sg = row_scale<FMT>(sexp, f), su = row_scale<FMT>(sexp, F + f);
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

template <int NT, int FMT>
__device__ void down_rows(const uint8_t* __restrict__ wexp, const void* sexp,
                          const __nv_bfloat16* hs, int d, int F, int i_base, int lane,
                          __nv_bfloat16* __restrict__ y, long row0) {
    for (int p = 0; p < ROWS_PER_WARP; p += 2) {
        const int i = i_base + p;
        if (i >= d) break;
        float a[NT], b[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) a[t] = b[t] = 0.f;
        pair_dots<NT, FMT>(wexp + (size_t)i * row_bytes<FMT>(F),
                           wexp + (size_t)(i + 1) * row_bytes<FMT>(F),
                           block_scales<FMT>(sexp, i, F), block_scales<FMT>(sexp, i + 1, F), hs,
                           F, lane, a, b);
        const float sa = row_scale<FMT>(sexp, i), sb = row_scale<FMT>(sexp, i + 1);
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

// The scales of expert e, whose weight has `rows` rows of L elements.
template <int FMT>
__device__ __forceinline__ const void* expert_scales(const void* s, int e, int rows, int L) {
    if (FMT == kFP8) return static_cast<const float*>(s) + (size_t)e * rows;
    if (FMT == kFP4) return static_cast<const uint8_t*>(s) + (size_t)e * rows * (L / 32);
    return nullptr;
}

template <int FMT>
__global__ void __launch_bounds__(SWARPS * 32)
gate_up_stream_kernel(const __nv_bfloat16* __restrict__ xperm, const int* __restrict__ offsets,
                      const uint8_t* __restrict__ wgu, const void* __restrict__ s_gu,
                      __nv_bfloat16* __restrict__ h, int d, int F) {
    pdl_launch_and_wait();
    extern __shared__ __align__(16) uint8_t smem[];
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem);
    const int e = blockIdx.y;
    const int r0 = offsets[e];
    const int n = offsets[e + 1] - r0;
    if (n <= 0) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int f_base = blockIdx.x * ROWS_PER_CTA + warp * ROWS_PER_WARP;
    const uint8_t* wexp = wgu + (size_t)e * 2 * F * row_bytes<FMT>(d);
    const void* sexp = expert_scales<FMT>(s_gu, e, 2 * F, d);
    for (int p = 0; p < n; p += NTMAX) {
        const int nt = min(NTMAX, n - p);
        __syncthreads();
        stage_rows(xs, xperm + (size_t)(r0 + p) * d, nt, d);
        __syncthreads();
        const long row0 = (long)r0 + p;
        switch (nt) {
            case 1: gate_up_rows<1, FMT>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
            case 2: gate_up_rows<2, FMT>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
            case 3: gate_up_rows<3, FMT>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
            case 4: gate_up_rows<4, FMT>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
            case 5: gate_up_rows<5, FMT>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
            case 6: gate_up_rows<6, FMT>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
            case 7: gate_up_rows<7, FMT>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
            default: gate_up_rows<8, FMT>(wexp, sexp, xs, d, F, f_base, lane, h, row0); break;
        }
    }
}

template <int FMT>
__global__ void __launch_bounds__(SWARPS * 32)
down_stream_kernel(const __nv_bfloat16* __restrict__ h, const int* __restrict__ offsets,
                   const uint8_t* __restrict__ wd, const void* __restrict__ s_d,
                   __nv_bfloat16* __restrict__ y, int d, int F) {
    pdl_launch_and_wait();
    extern __shared__ __align__(16) uint8_t smem[];
    __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(smem);
    const int e = blockIdx.y;
    const int r0 = offsets[e];
    const int n = offsets[e + 1] - r0;
    if (n <= 0) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i_base = blockIdx.x * ROWS_PER_CTA + warp * ROWS_PER_WARP;
    const uint8_t* wexp = wd + (size_t)e * d * row_bytes<FMT>(F);
    const void* sexp = expert_scales<FMT>(s_d, e, d, F);
    for (int p = 0; p < n; p += NTMAX) {
        const int nt = min(NTMAX, n - p);
        __syncthreads();
        stage_rows(hs, h + (size_t)(r0 + p) * F, nt, F);
        __syncthreads();
        const long row0 = (long)r0 + p;
        switch (nt) {
            case 1: down_rows<1, FMT>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
            case 2: down_rows<2, FMT>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
            case 3: down_rows<3, FMT>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
            case 4: down_rows<4, FMT>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
            case 5: down_rows<5, FMT>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
            case 6: down_rows<6, FMT>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
            case 7: down_rows<7, FMT>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
            default: down_rows<8, FMT>(wexp, sexp, hs, d, F, i_base, lane, y, row0); break;
        }
    }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

int weight_format(const moe_config& c) {
    if (c.flags & MOE_FLAG_FP4_WEIGHTS) return kFP4;
    if (c.flags & MOE_FLAG_FP8_WEIGHTS) return kFP8;
    return kBF16;
}

template <int FMT>
cudaError_t gate_up(const moe_config& c, const void* x_perm, const int32_t* offsets,
                    const void* w_gate_up, const void* s_gate_up, void* h, cudaStream_t s) {
    const size_t smem = (size_t)NTMAX * c.d * 2;
    const dim3 grid((c.d_ff + ROWS_PER_CTA - 1) / ROWS_PER_CTA, c.E);
    cudaError_t err = set_smem(gate_up_stream_kernel<FMT>, smem);
    if (err != cudaSuccess) return err;
    err = launch_pdl(
        gate_up_stream_kernel<FMT>, grid, dim3(SWARPS * 32), smem, s,
        static_cast<const __nv_bfloat16*>(x_perm), offsets, static_cast<const uint8_t*>(w_gate_up),
        s_gate_up, static_cast<__nv_bfloat16*>(h), c.d, c.d_ff);
    return err != cudaSuccess ? err : cudaGetLastError();
}

template <int FMT>
cudaError_t down(const moe_config& c, const void* h, const int32_t* offsets, const void* w_down,
                 const void* s_down, void* y, cudaStream_t s) {
    const size_t smem = (size_t)NTMAX * c.d_ff * 2;
    const dim3 grid((c.d + ROWS_PER_CTA - 1) / ROWS_PER_CTA, c.E);
    cudaError_t err = set_smem(down_stream_kernel<FMT>, smem);
    if (err != cudaSuccess) return err;
    err = launch_pdl(
        down_stream_kernel<FMT>, grid, dim3(SWARPS * 32), smem, s,
        static_cast<const __nv_bfloat16*>(h), offsets, static_cast<const uint8_t*>(w_down), s_down,
        static_cast<__nv_bfloat16*>(y), c.d, c.d_ff);
    return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate_up_stream(const moe_config& c, const void* x_perm, const int32_t* offsets,
                                  const void* w_gate_up, const void* s_gate_up, void* h,
                                  cudaStream_t s) {
    switch (weight_format(c)) {
        case kFP4: return gate_up<kFP4>(c, x_perm, offsets, w_gate_up, s_gate_up, h, s);
        case kFP8: return gate_up<kFP8>(c, x_perm, offsets, w_gate_up, s_gate_up, h, s);
        default: return gate_up<kBF16>(c, x_perm, offsets, w_gate_up, nullptr, h, s);
    }
}

cudaError_t launch_down_stream(const moe_config& c, const void* h, const int32_t* offsets,
                               const void* w_down, const void* s_down, void* y, cudaStream_t s) {
    switch (weight_format(c)) {
        case kFP4: return down<kFP4>(c, h, offsets, w_down, s_down, y, s);
        case kFP8: return down<kFP8>(c, h, offsets, w_down, s_down, y, s);
        default: return down<kBF16>(c, h, offsets, w_down, nullptr, y, s);
    }
}

}  // namespace moe
