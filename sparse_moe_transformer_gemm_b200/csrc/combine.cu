// combine.cu -- fp32 weighted combine and unpermute.
//
// enable_moe_fp32_combine (Hy3 commentary, wmrh.cn/news/24252, §2.3): the
// expert branch outputs are converted to fp32, summed with their routing
// weights in fp32 and cast back to bf16 once, so that small contributions
// next to a large one are not rounded away. The weighted sum over the k
// selected experts replaces the pages' per-expert loop with index_add_
// ("DeepSeek V4-Flash 架构 QA", Q8.4) by a gather: token t reads its k expert
// rows y[row_of[t*k + j]] (no atomics, fixed j order, deterministic). With a
// shared expert ("Tencent Hy3-Flash QA" Q4.7) each token has one more slot,
// the last, weighted 1.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// CTA (token t, column block b): 128 threads, one 8-column vector each. The k
// expert rows are loaded 8 at a time before their FMAs (independent loads in
// flight), the FMAs run in j order.
constexpr int CT = 128;

__global__ void __launch_bounds__(CT)
combine_kernel(const __nv_bfloat16* __restrict__ y, const int* __restrict__ row_of,
               const float* __restrict__ w, int k_routed, int k, int d,
               __nv_bfloat16* __restrict__ out) {
    pdl_launch_and_wait();
    // k slots per token; slots at and past k_routed (the shared expert) weigh 1
    __shared__ int rows[33];
    __shared__ float wts[33];
    const long t = blockIdx.x;
    if (threadIdx.x < k) {
        rows[threadIdx.x] = row_of[t * k + threadIdx.x];
        wts[threadIdx.x] = threadIdx.x < k_routed ? w[t * k_routed + threadIdx.x] : 1.0f;
    }
    __syncthreads();
    const int v = blockIdx.y * CT + threadIdx.x;
    if (v >= d / 8) return;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int j0 = 0; j0 < k; j0 += 8) {
        uint4 u[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            const int j = j0 + jj;
            const int r = (j < k) ? rows[j] : -1;
            u[jj] = (r >= 0) ? __ldcs(reinterpret_cast<const uint4*>(y + (long)r * d) + v)
                             : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            const int j = j0 + jj;
            if (j >= k || rows[j] < 0) continue;
            float f[8];
            bf16x8_to_float(u[jj], f);
            const float wj = wts[j];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = fmaf(wj, f[i], acc[i]);
        }
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(out + t * d + v * 8) = o;
}

}  // namespace

cudaError_t launch_combine(const moe_config& c, const void* y, const int32_t* row_of,
                           const float* topk_w, void* out, cudaStream_t s) {
    const dim3 grid(c.T, (c.d / 8 + CT - 1) / CT);
    const cudaError_t err = launch_pdl(combine_kernel, grid, dim3(CT), 0, s,
                                       static_cast<const __nv_bfloat16*>(y), row_of, topk_w, c.k,
                                       c.k + shared_slots(c), c.d,
                                       static_cast<__nv_bfloat16*>(out));
    return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
