// common.cuh -- small device helpers shared by the library's kernels (the
// bit-level ones also compile as host code, for host-side checks).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>
#include <string.h>

namespace moe {

// Bit casts between float and uint32_t, for host and device code.
__host__ __device__ __forceinline__ float f32_from_bits(uint32_t u) {
#ifdef __CUDA_ARCH__
    return __uint_as_float(u);
#else
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
#endif
}
__host__ __device__ __forceinline__ uint32_t f32_bits(float f) {
#ifdef __CUDA_ARCH__
    return __float_as_uint(f);
#else
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return u;
#endif
}

// bf16 pair (packed in a 32-bit word, low half first) -> two floats. Exact.
__host__ __device__ __forceinline__ float2 bf16x2_to_float2(uint32_t v) {
    return make_float2(f32_from_bits(v << 16), f32_from_bits(v & 0xFFFF0000u));
}

// Eight bf16 in a 16-byte vector -> eight floats.
__device__ __forceinline__ void bf16x8_to_float(const uint4& v, float f[8]) {
    float2 a = bf16x2_to_float2(v.x), b = bf16x2_to_float2(v.y);
    float2 c = bf16x2_to_float2(v.z), d = bf16x2_to_float2(v.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
    f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

// Two e4m3 codes (low byte first) -> two floats, exactly (via the hardware
// e4m3x2 -> f16x2 conversion; every e4m3 value is an f16 value).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t v) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)v, __NV_E4M3);
    return __half22float2(*reinterpret_cast<__half2*>(&h));
}

// Sixteen e4m3 codes in a 16-byte vector -> sixteen floats.
__device__ __forceinline__ void e4m3x16_to_float(const uint4& v, float f[16]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 lo = e4m3x2_to_float2((uint16_t)(w[i] & 0xFFFF));
        float2 hi = e4m3x2_to_float2((uint16_t)(w[i] >> 16));
        f[4 * i + 0] = lo.x; f[4 * i + 1] = lo.y; f[4 * i + 2] = hi.x; f[4 * i + 3] = hi.y;
    }
}

// Sixteen E2M1 codes in two 32-bit words (two per byte, the even element in
// the low nibble, words and bytes in increasing element order) -> sixteen
// floats, exactly: the hardware e2m1x2 -> f16x2 conversion takes the low
// nibble to the low half, and every E2M1 value is an f16 value.
__device__ __forceinline__ void e2m1x16_to_float(uint32_t w0, uint32_t w1, float f[16]) {
    const uint32_t w[2] = {w0, w1};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            __half2_raw h = __nv_cvt_fp4x2_to_halfraw2(
                (__nv_fp4x2_storage_t)((w[i] >> (8 * j)) & 0xFFu), __NV_E2M1);
            const float2 p = __half22float2(*reinterpret_cast<__half2*>(&h));
            f[8 * i + 2 * j] = p.x;
            f[8 * i + 2 * j + 1] = p.y;
        }
    }
}

// Two e4m3 codes placed as u = code1 << 24 | code0 << 8 (other bytes zero) ->
// a bf16x2 whose halves are the codes' values times 2^-120: the seven
// exponent+mantissa bits move to bf16 bits 4..10, the sign stays at bit 15
// (the FP8 GEMM's widening multiplies by 2^120 afterwards).
__host__ __device__ __forceinline__ uint32_t e4m3_pair_scaled_bits(uint32_t u) {
    return ((u & 0x7F007F00u) >> 4) | (u & 0x80008000u);
}

// One byte of two E2M1 codes (the even code in the low nibble) -> a bf16x2
// whose halves (the even code low) are the codes' values times 2^-126: the
// byte is copied into both 16-bit halves (times 0x1001: the low nibble at bits
// 0..3, the high one at 16..19), the three exponent+mantissa bits move to
// bf16 bits 6..8 and the sign to bit 15 (adding sign * 4032 turns the sign's
// copy at bit 9 into bit 15). An E2M1 value 2^(e-1) (1 + m/2) then reads as
// 2^(e-127) (1 + m/2), and the subnormal 0.5 as the bf16 subnormal 2^-127
// (the FP4 GEMM's widening multiplies by the block scale times 2^126).
__host__ __device__ __forceinline__ uint32_t e2m1_pair_scaled_bits(uint32_t byte) {
    const uint32_t t = (byte * 0x1001u) & 0x000F000Fu;
    return (t << 6) + (t & 0x00080008u) * 4032u;
}

// E8M0 scale byte b -> 2^(b - 127) (b = 0 gives the subnormal 2^-127; b = 255,
// not a scale, gives infinity).
__device__ __forceinline__ float e8m0_to_float(uint32_t b) {
    return b ? __uint_as_float(b << 23) : __uint_as_float(0x00400000u);
}

// Round a float to bf16 (nearest-even) and return the 16-bit pattern.
__host__ __device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    uint16_t u;
    memcpy(&u, &b, sizeof u);
    return u;
}

__host__ __device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    return (uint32_t)float_to_bf16_bits(lo) | ((uint32_t)float_to_bf16_bits(hi) << 16);
}

// Read-only, L1-bypassing 16-byte load for data streamed exactly once.
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float sigmoidf_acc(float z) { return 1.0f / (1.0f + expf(-z)); }

// Router score functions (both increasing in the logit): 0 the sigmoid (Hy3),
// 1 sqrt(softplus(z)) = sqrt(log(1 + e^z)) (the V4-Flash column of
// "Tencent Hy3-295B 架构深度拆解" §2.2), evaluated as
// sqrt(max(z, 0) + log1p(e^-|z|)), which neither overflows nor loses the
// small softplus of a very negative logit.
__device__ __forceinline__ float sqrt_softplusf(float z) {
    return sqrtf(fmaxf(z, 0.f) + log1pf(expf(-fabsf(z))));
}
__device__ __forceinline__ float score_value(float z, int score_fn) {
    return score_fn ? sqrt_softplusf(z) : sigmoidf_acc(z);
}

// Warp-collective top-k of one token's router scores. sc[q] holds the biased
// logit of expert lane + 32 q (-INFINITY where that expert does not exist, so
// E <= 256). k <= 32 rounds; each takes the warp maximum with one redux.sync
// on an order-preserving unsigned key of the value and, among the lanes that
// hold it, the lowest expert index with a second one (ties to the lower
// index). The score function (score_value) is increasing, so these are the k
// largest scores. Lane j < k writes the j-th selection: idx_row[j] and
// w_row[j] = scale * score_j / sum of the k scores (summed in j order).
__host__ __device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t b = f32_bits(f + 0.0f);  // -0 -> +0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__host__ __device__ __forceinline__ float key_value(uint32_t key) {
    return f32_from_bits((key & 0x80000000u) ? (key ^ 0x80000000u) : ~key);
}

//
// With prob (the lane's 8 scores; sc then holds the choice values
// score + e_score_correction_bias), the weights renormalise prob of the chosen
// experts instead of the scores of the ranked values.
__device__ __forceinline__ void warp_select_topk(float (&sc)[8], int k, float scale,
                                                 int* __restrict__ idx_row,
                                                 float* __restrict__ w_row,
                                                 const float* prob = nullptr,
                                                 int score_fn = 0) {
    const int lane = threadIdx.x & 31;
    uint32_t key[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) key[q] = order_key(sc[q]);  // removed entries get key 0
    int my_e = 0;
    float my_s = 0.f;
    for (int r = 0; r < k; ++r) {
        uint32_t bk = key[0];
        int bq = 0;
#pragma unroll
        for (int q = 1; q < 8; ++q)
            if (key[q] > bk) { bk = key[q]; bq = q; }
        const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t be = __reduce_min_sync(0xffffffffu,
                                              bk == m ? (uint32_t)(lane + 32 * bq) : 0xffffffffu);
        float pv = 0.f;
        if (prob) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if ((int)(be >> 5) == q) pv = prob[q];
            pv = __shfl_sync(0xffffffffu, pv, (int)(be & 31u));
        }
        if (lane == r) { my_e = (int)be; my_s = prob ? pv : score_value(key_value(m), score_fn); }
        if ((int)(be & 31u) == lane) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if ((int)(be >> 5) == q) key[q] = 0u;
        }
    }
    float sum = 0.f;
    for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, my_s, j);
    if (lane < k) {
        idx_row[lane] = my_e;
        w_row[lane] = scale * my_s / sum;
    }
}

// SwiGLU's SiLU(g) * u with the fast exponential and division intrinsics: their
// relative error (~1e-6) sits far below the bf16 rounding of the result
// (2^-9), and for g below about -87 the quotient is 0, SiLU's limit.
// Programmatic dependent launch: let the next kernel on the stream begin
// launching (its thread blocks take SMs as this grid's leave, and wait in
// their own pdl_launch_and_wait), then wait until the previous kernel on the
// stream has completed and its writes are visible. Every kernel of the layer
// calls this before it touches global memory; for a launch without the
// programmatic-serialization attribute both steps do nothing.
__device__ __forceinline__ void pdl_launch_and_wait() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ float silu_mul(float g, float u) {
    return __fdividef(g, 1.0f + __expf(-g)) * u;
}

}  // namespace moe
