// router_tc.cu -- router on the tensor cores: logits GEMM with tcgen05,
// sigmoid, top-k with lowest-index tie-break, renormalisation and scale.
//
// Same method as router.cu ("Tencent Hy3-295B 架构深度拆解" §4.1: fp32 logits,
// element-wise sigmoid, top-8, renormalise the selected scores, x2.826; an
// optional logit bias added before the sigmoid, Hy3 commentary §3.3).
//
// Tile: 128 tokens (MMA M, tokens in TMEM lanes) x all E experts (MMA N = E
// rounded up to 16, <= 256) over a K slice of the hidden size, bf16 x bf16 ->
// fp32. So that small batches still spread over the GPU, the K dimension is
// split over S CTAs per token tile (S chosen so that tiles * S ~ SM count).
// Every CTA writes its fp32 partial logits [128, E] to the workspace; the last
// CTA of a token tile to arrive (arrival counter, no waiting) adds the S
// partials in split order -- the result does not depend on arrival order --
// and selects per token in-thread: one epilogue thread per token scans the E
// sigmoid scores keeping a sorted top-k list (strictly greater enters, so an
// equal score never displaces a lower expert index).
//
// CTA: 192 threads -- warp 0 TMA producer, warp 1 TMEM owner + MMA issuer,
// warps 2-5 epilogue / selection. Waits are bounded (MOE_ERR_TIMEOUT).
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace moe {

int router_splits(int T, int d);  // defined below, also used for the workspace size

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int UK = 16;
constexpr int THREADS = 192;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;         // x tile
constexpr int B_BYTES_MAX = 256 * BK * 2;    // W_gate tile (<= 256 experts)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES_MAX;

struct Ctrl {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int last;
};

constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + (int)sizeof(Ctrl);
static_assert(BM * (256 + 1) * 4 <= STAGES * STAGE_BYTES, "selection rows fit in the stage ring");

// Top-k of one token from its E logits (a shared-memory row), then the
// renormalised, scaled weights. Strictly greater enters the sorted list, so
// an equal score never displaces a lower expert index.
template <int K>
__device__ __forceinline__ void select_topk(const float* row, const float* __restrict__ bias, int E,
                                            float scale, int* __restrict__ idx_out,
                                            float* __restrict__ w_out) {
    float v[K];
    int id[K];
#pragma unroll
    for (int j = 0; j < K; ++j) { v[j] = -1.f; id[j] = 0; }
    for (int e = 0; e < E; ++e) {
        const float sc = sigmoidf_acc(bias ? row[e] + __ldg(bias + e) : row[e]);
        if (sc > v[K - 1]) {
            v[K - 1] = sc;
            id[K - 1] = e;
#pragma unroll
            for (int j = K - 1; j > 0; --j) {
                if (v[j] > v[j - 1]) {
                    const float tv = v[j]; v[j] = v[j - 1]; v[j - 1] = tv;
                    const int ti = id[j]; id[j] = id[j - 1]; id[j - 1] = ti;
                }
            }
        }
    }
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < K; ++j) sum += v[j];
#pragma unroll
    for (int j = 0; j < K; ++j) {
        idx_out[j] = id[j];
        w_out[j] = scale * v[j] / sum;
    }
}

// grid: (token tiles, splits). tmX: x [T, d] box 64 x 128; tmW: W_gate [E, d] box 64 x n_pad.
// part: fp32 [S][T_pad][E]; counters: one per token tile (zero on entry, reset on exit).
__global__ void __launch_bounds__(THREADS, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 const float* __restrict__ bias, int T, int d, int E, int k, int n_pad,
                 float scale, float* __restrict__ part, int* __restrict__ counters,
                 int* __restrict__ idx_out, float* __restrict__ w_out, int* __restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Ctrl& c = *reinterpret_cast<Ctrl*>(smem + STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tile = blockIdx.x, split = blockIdx.y, S = gridDim.y;
    const int KB = d / BK;
    const int kb0 = split * KB / S, kb1 = (split + 1) * KB / S;  // S <= KB: never empty
    const int T_pad = gridDim.x * BM;

    if (warp == 0 && lane == 0) {
        c.abort = 0;
        tc::prefetch_tensormap(&tmX);
        tc::prefetch_tensormap(&tmW);
    } else if (warp == 1) {
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                tc::mbar_init(&c.full[s], 1);
                tc::mbar_init(&c.empty[s], 1);
            }
            tc::mbar_init(&c.acc_full, 1);
            tc::mbar_init(&c.drain, 1);
            tc::fence_mbar_init();
        }
        __syncwarp();
        tc::tmem_alloc(&c.tmem_base, 256);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem_base = c.tmem_base;
    const volatile int* abort_flag = &c.abort;
    const uint32_t b_bytes = (uint32_t)n_pad * BK * 2;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_parity[STAGES] = {};
            bool issued[STAGES] = {};
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!tc::mbar_wait(&c.empty[stage], phase ^ 1u, abort_flag)) {
                    *reinterpret_cast<volatile int*>(&c.abort) = 1;
                    atomicExch(status, MOE_ERR_TIMEOUT);
                    break;
                }
                uint8_t* s = smem + stage * STAGE_BYTES;
                tc::mbar_arrive_expect_tx(&c.full[stage], A_BYTES + b_bytes);
                tc::tma_load_2d(s, &tmX, &c.full[stage], kb * BK, tile * BM);
                tc::tma_load_2d(s + A_BYTES, &tmW, &c.full[stage], kb * BK, 0);
                issued[stage] = true;
                issued_parity[stage] = phase;
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            const int zero = 0;
            for (int s = 0; s < STAGES; ++s)
                if (issued[s] && !tc::mbar_wait(&c.full[s], issued_parity[s], &zero))
                    atomicExch(status, MOE_ERR_TIMEOUT);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            const uint32_t idesc = tc::idesc_bf16_f32(BM, n_pad);
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!tc::mbar_wait(&c.full[stage], phase, abort_flag)) {
                    *reinterpret_cast<volatile int*>(&c.abort) = 1;
                    atomicExch(status, MOE_ERR_TIMEOUT);
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                const uint32_t a_addr = tc::smem_u32(smem + stage * STAGE_BYTES);
                const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / UK; ++kk)
                    tc::mma_bf16(tmem_base, tc::desc_sw128(a_addr + kk * UK * 2),
                                 tc::desc_sw128(b_addr + kk * UK * 2), idesc,
                                 (kb > kb0 || kk > 0) ? 1u : 0u);
                tc::mma_commit(&c.empty[stage]);
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (ok) tc::mma_commit(&c.acc_full);
            tc::mma_commit(&c.drain);
            const int zero = 0;
            if (!tc::mbar_wait(&c.drain, 0, &zero)) atomicExch(status, MOE_ERR_TIMEOUT);
        }
    } else {
        // epilogue: TMEM -> this split's partial logits
        const int quad = warp & 3;
        const int row = quad * 32 + lane;               // token within the tile
        const long t = (long)tile * BM + row;
        float* my = part + ((long)split * T_pad + t) * E;
        bool ok = tc::mbar_wait(&c.acc_full, 0, abort_flag);
        if (!ok) {
            *reinterpret_cast<volatile int*>(&c.abort) = 1;
            atomicExch(status, MOE_ERR_TIMEOUT);
        } else {
            tc::fence_after_sync();
            const uint32_t tb = tmem_base + ((uint32_t)(quad * 32) << 16);
            for (int c0 = 0; c0 < n_pad; c0 += 32) {
                uint32_t r[32];
                tc::tmem_ld32(tb + c0, r);
                tc::tmem_ld_wait();
                if (c0 + 32 <= E) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4*>(my + c0 + j) =
                            make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                        __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (c0 + j < E) my[c0 + j] = __uint_as_float(r[j]);
                }
            }
        }
        tc::fence_before_sync();
        // arrival among the 128 epilogue threads (named barrier 1)
        __threadfence();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (warp == 2 && lane == 0) {
            const int ticket = atomicAdd(&counters[tile], 1);
            c.last = (ticket == S - 1);
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (c.last) {
            __threadfence();
            // Sum the S partials of this tile in split order into shared memory
            // (the stage ring is idle now), rows padded to E+1 floats so that
            // the per-token reads below hit distinct banks.
            float* red = reinterpret_cast<float*>(smem);
            const int es = E + 1;
            const int etid = threadIdx.x - 64;
            const long stride = (long)T_pad * E;
            const float* tile_part = part + (long)tile * BM * E;
            const int n4 = BM * E / 4;
#pragma unroll 4
            for (int v = etid; v < n4; v += 128) {
                float4 a = __ldcg(reinterpret_cast<const float4*>(tile_part) + v);
                for (int sp = 1; sp < S; ++sp) {
                    const float4 q =
                        __ldcg(reinterpret_cast<const float4*>(tile_part + sp * stride) + v);
                    a.x += q.x; a.y += q.y; a.z += q.z; a.w += q.w;
                }
                const int r = (v * 4) / E, e = (v * 4) - r * E;
                float* dst = red + r * es + e;
                dst[0] = a.x; dst[1] = a.y; dst[2] = a.z; dst[3] = a.w;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (t < T) {
                const float* rw = red + row * es;
                int* io = idx_out + t * k;
                float* wo = w_out + t * k;
                switch (k) {
                    case 1: select_topk<1>(rw, bias, E, scale, io, wo); break;
                    case 2: select_topk<2>(rw, bias, E, scale, io, wo); break;
                    case 3: select_topk<3>(rw, bias, E, scale, io, wo); break;
                    case 4: select_topk<4>(rw, bias, E, scale, io, wo); break;
                    case 5: select_topk<5>(rw, bias, E, scale, io, wo); break;
                    case 6: select_topk<6>(rw, bias, E, scale, io, wo); break;
                    case 7: select_topk<7>(rw, bias, E, scale, io, wo); break;
                    default: select_topk<8>(rw, bias, E, scale, io, wo); break;
                }
            }
            if (warp == 2 && lane == 0) counters[tile] = 0;
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem_base, 256);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Splits of the hidden dimension per token tile: enough CTAs for the 148 SMs
// of a B200 (a fixed count, so the workspace size does not depend on the device).
int router_splits(int T, int d) {
    const int tiles = (T + BM - 1) / BM;
    int s = 148 / tiles;
    if (s < 1) s = 1;
    if (s > 8) s = 8;
    const int kb = d / BK;
    if (s > kb) s = kb;
    return s;
}

bool router_tc_supported(const moe_config& c) { return c.k <= 8 && c.E % 4 == 0; }

cudaError_t launch_router_tc(const moe_config& c, const void* x, const void* w_gate,
                             const float* gate_bias, int32_t* idx, float* w, float* part,
                             int32_t* counters, int* status, cudaStream_t s) {
    const int tiles = (c.T + BM - 1) / BM;
    const int S = router_splits(c.T, c.d);
    const int n_pad = (c.E + 15) & ~15;
    CUtensorMap mx, mw;
    if (!make_map(&mx, x, c.T, c.d, BM) || !make_map(&mw, w_gate, c.E, c.d, n_pad))
        return cudaErrorInvalidValue;
    cudaError_t err =
        cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (err != cudaSuccess) return err;
    router_tc_kernel<<<dim3(tiles, S), THREADS, SMEM, s>>>(mx, mw, gate_bias, c.T, c.d, c.E, c.k,
                                                           n_pad, c.scale, part, counters, idx, w,
                                                           status);
    return cudaGetLastError();
}

}  // namespace moe
