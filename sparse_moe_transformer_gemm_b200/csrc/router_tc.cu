// router_tc.cu -- router on the tensor cores: logits GEMM with tcgen05,
// sigmoid, top-k with lowest-index tie-break, renormalisation and scale.
//
// Same method as router.cu ("Tencent Hy3-295B 架构深度拆解" §4.1: fp32 logits,
// element-wise sigmoid, top-8, renormalise the selected scores, x2.826; an
// optional logit bias added before the sigmoid, Hy3 commentary §3.3).
//
// Tile: 128 tokens (MMA M, tokens in TMEM lanes) x all E experts (MMA N = E
// rounded up to 16, <= 256) over a K slice of the hidden size, bf16 x bf16 ->
// fp32. So that small batches still spread over the GPU, the hidden dimension
// is split over S in {1, 2, 4, 8} CTAs per token tile, launched as one thread-
// block cluster. Each CTA moves its partial logits from TMEM to its own shared
// memory; after a cluster barrier, CTA j sums rows [j*128/S, (j+1)*128/S) over
// the S CTAs through distributed shared memory (16-byte loads, several in
// flight per thread), in split order (the result does not depend on timing),
// and selects for those rows, S lanes per row (each scans a contiguous range
// of experts; shuffle merges combine the lists), ties to the lower expert
// index. The sigmoid is increasing, so the k largest (biased) logits are the k
// largest scores; it is evaluated for the k selected only. With score_fn 1
// the score is sqrt(softplus(logit)) (the V4-Flash router, same page §2.2),
// also increasing.
//
// CTA: 192 threads -- warp 0 TMA producer, warp 1 TMEM owner + MMA issuer,
// warps 2-5 epilogue / reduction / selection. Waits are bounded
// (MOE_ERR_TIMEOUT in the status word).
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace moe {

int router_splits(int T, int d);  // defined below

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
    // the logit bias (0 where none, and past E: the selection reads 8 at a time)
    alignas(16) float bias[256 + 8];
    alignas(16) float sbias[256 + 8];  // the e_score_correction_bias, when given
};

constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + (int)sizeof(Ctrl);
// Row stride (floats) of the logit rows in shared memory: a multiple of 4 (16-byte
// rows) that is 4 mod 32, so a warp's 16-byte row stores take the minimum of
// four wavefronts.
__host__ __device__ constexpr int logit_stride(int E) { return ((E + 31) / 32) * 32 + 4; }
// (the selection reads up to 7 floats past a row's E logits; the ring has room)
static_assert(BM * logit_stride(256) * 4 + 32 <= STAGES * STAGE_BYTES, "logit rows fit in the ring");

// Top-k of one token over the experts [e_lo, e_hi) by one thread, from its
// logits (a shared-memory row, 16-byte aligned, read as float4: with a row
// stride of 4 mod 32 floats the 16-byte reads of a warp's rows take the
// minimum number of wavefronts): a sorted list (8 entries, the first K in use,
// the rest -inf) of the K largest (biased) logits where only a strictly
// greater value enters, so equal values keep the lower expert index (experts
// are visited in increasing order). e_lo is a multiple of 8; e_hi is E or a
// multiple of 8. The bias is staged in shared memory (per-element global
// loads of it made the scan ~3x slower).
template <int K, bool SB>
__device__ __forceinline__ void scan_topk(const float* row, const float* sbias, const float* cbias,
                                          int e_lo, int e_hi, int E, int score_fn, float (&v)[8],
                                          float (&p)[8], int (&id)[8]) {
    // SB: rank sigmoid(logit) + cbias (the e_score_correction_bias) and keep
    // the sigmoid scores p of the list for the weights
#pragma unroll
    for (int j = 0; j < 8; ++j) { v[j] = -INFINITY; p[j] = 0.f; id[j] = 0x7fffffff; }
    for (int e0 = e_lo; e0 < e_hi; e0 += 8) {
        // 8 logits and their biases in flight, then visited in increasing order
        const float4 a0 = *reinterpret_cast<const float4*>(row + e0);
        const float4 a1 = *reinterpret_cast<const float4*>(row + e0 + 4);
        const float4 b0 = *reinterpret_cast<const float4*>(sbias + e0);
        const float4 b1 = *reinterpret_cast<const float4*>(sbias + e0 + 4);
        const float z8[8] = {a0.x + b0.x, a0.y + b0.y, a0.z + b0.z, a0.w + b0.w,
                             a1.x + b1.x, a1.y + b1.y, a1.z + b1.z, a1.w + b1.w};
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = e0 + u;
            float z = z8[u], pz = 0.f;
            if (SB && e < E) {
                pz = score_value(z, score_fn);
                z = pz + cbias[e];
            }
            if (e < E && z > v[K - 1]) {
                v[K - 1] = z;
                p[K - 1] = pz;
                id[K - 1] = e;
#pragma unroll
                for (int j = K - 1; j > 0; --j) {
                    if (v[j] > v[j - 1]) {
                        const float tv = v[j]; v[j] = v[j - 1]; v[j - 1] = tv;
                        const float tp = p[j]; p[j] = p[j - 1]; p[j - 1] = tp;
                        const int ti = id[j]; id[j] = id[j - 1]; id[j - 1] = ti;
                    }
                }
            }
        }
    }
}

// Entry a ranks before entry b: a larger value, or an equal value and a lower
// expert index.
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

// Merge this lane's sorted 8-entry list with the one of lane ^ m (same order,
// disjoint experts) into the 8 best of both, sorted, in both lanes: the
// element-wise better of the list and the partner's reversed list is a
// bitonic sequence holding the 8 best, and three half-cleaner stages sort it.
__device__ __forceinline__ void merge_topk(float (&v)[8], float (&p)[8], int (&id)[8], int m) {
    float ov[8], op[8];
    int oi[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        ov[j] = __shfl_xor_sync(0xffffffffu, v[j], m);
        op[j] = __shfl_xor_sync(0xffffffffu, p[j], m);
        oi[j] = __shfl_xor_sync(0xffffffffu, id[j], m);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
        if (ranks_before(ov[7 - j], oi[7 - j], v[j], id[j])) {
            v[j] = ov[7 - j];
            p[j] = op[7 - j];
            id[j] = oi[7 - j];
        }
#pragma unroll
    for (int s = 4; s > 0; s >>= 1)
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if ((j & s) == 0 && ranks_before(v[j + s], id[j + s], v[j], id[j])) {
                const float tv = v[j]; v[j] = v[j + s]; v[j + s] = tv;
                const float tp = p[j]; p[j] = p[j + s]; p[j + s] = tp;
                const int ti = id[j]; id[j] = id[j + s]; id[j + s] = ti;
            }
}

// The selection of one token by P adjacent lanes (P a power of two <= 8; P
// = 1: one thread): lane `part` scans its range of experts (contiguous,
// increasing with part), and log2 P shuffle merges give every lane the
// token's sorted list -- the same list, in the same order, as one thread's
// scan of all experts. Part 0 then evaluates the score of the K selected,
// renormalises (summed in list order) and scales. Every lane of the warp
// takes part (the merges shuffle across the whole warp); `write` gates the
// output. (A warp per token, k rounds of a warp-wide argmax, measured ~3 us
// per token here.)
template <int K, bool SB, int P>
__device__ __forceinline__ void select_topk(const float* row, const float* sbias,
                                            const float* cbias, int E, float scale, int score_fn,
                                            int part, bool write, int* __restrict__ idx_out,
                                            float* __restrict__ w_out) {
    const int chunk = ((E + P - 1) / P + 7) & ~7;
    const int e_lo = part * chunk;
    const int e_hi = min(E, e_lo + chunk);
    float v[8], p[8];
    int id[8];
    scan_topk<K, SB>(row, sbias, cbias, e_lo, e_hi, E, score_fn, v, p, id);
#pragma unroll
    for (int m = 1; m < P; m <<= 1) merge_topk(v, p, id, m);
    if (!write || part != 0) return;
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < K; ++j) {
        v[j] = SB ? p[j] : score_value(v[j], score_fn);
        sum += v[j];
    }
#pragma unroll
    for (int j = 0; j < K; ++j) {
        idx_out[j] = id[j];
        w_out[j] = scale * v[j] / sum;
    }
}

template <bool SB, int P>
__device__ __forceinline__ void select_k(int k, const float* row, const float* sbias,
                                         const float* cbias, int E, float scale, int score_fn,
                                         int part, bool write, int* __restrict__ idx_out,
                                         float* __restrict__ w_out) {
    switch (k) {
        case 1: select_topk<1, SB, P>(row, sbias, cbias, E, scale, score_fn, part, write, idx_out, w_out); break;
        case 2: select_topk<2, SB, P>(row, sbias, cbias, E, scale, score_fn, part, write, idx_out, w_out); break;
        case 3: select_topk<3, SB, P>(row, sbias, cbias, E, scale, score_fn, part, write, idx_out, w_out); break;
        case 4: select_topk<4, SB, P>(row, sbias, cbias, E, scale, score_fn, part, write, idx_out, w_out); break;
        case 5: select_topk<5, SB, P>(row, sbias, cbias, E, scale, score_fn, part, write, idx_out, w_out); break;
        case 6: select_topk<6, SB, P>(row, sbias, cbias, E, scale, score_fn, part, write, idx_out, w_out); break;
        case 7: select_topk<7, SB, P>(row, sbias, cbias, E, scale, score_fn, part, write, idx_out, w_out); break;
        default: select_topk<8, SB, P>(row, sbias, cbias, E, scale, score_fn, part, write, idx_out, w_out); break;
    }
}

// grid: (token tiles, S) with clusters of (1, S). tmX: x [T, d] box 64 x 128;
// tmW: W_gate [E, d] box 64 x n_pad.
template <int S>
__global__ void __launch_bounds__(THREADS, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 const float* __restrict__ bias, const float* __restrict__ sbias, int T,
                 int d, int E, int k, int n_pad,
                 float scale, int score_fn, int* __restrict__ idx_out,
                 float* __restrict__ w_out, int* __restrict__ status) {
    pdl_launch_and_wait();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Ctrl& c = *reinterpret_cast<Ctrl*>(smem + STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tile = blockIdx.x;
    const int split = (S > 1) ? (int)tc::cluster_ctarank() : 0;
    const int KB = d / BK;
    const int kb0 = split * KB / S, kb1 = (split + 1) * KB / S;  // S <= KB: never empty
    const int es = logit_stride(E);
    float* red = reinterpret_cast<float*>(smem);  // [128][es], reuses the stage ring

    if (warp >= 2) {
        for (int e = threadIdx.x - 64; e < 256 + 8; e += 128) {
            c.bias[e] = (bias && e < E) ? bias[e] : 0.f;
            c.sbias[e] = (sbias && e < E) ? sbias[e] : 0.f;
        }
    }
    if (warp == 0 && lane == 0) {
        c.abort = 0;
        tc::prefetch_tensormap(&tmX);
        tc::prefetch_tensormap(&tmW);
    } else if (warp == 1) {
        if (lane == 0) {
            for (int st = 0; st < STAGES; ++st) {
                tc::mbar_init(&c.full[st], 1);
                tc::mbar_init(&c.empty[st], 1);
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
                uint8_t* st = smem + stage * STAGE_BYTES;
                tc::mbar_arrive_expect_tx(&c.full[stage], A_BYTES + b_bytes);
                tc::tma_load_2d(st, &tmX, &c.full[stage], kb * BK, tile * BM);
                tc::tma_load_2d(st + A_BYTES, &tmW, &c.full[stage], kb * BK, 0);
                issued[stage] = true;
                issued_parity[stage] = phase;
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            const int zero = 0;
            for (int st = 0; st < STAGES; ++st)
                if (issued[st] && !tc::mbar_wait(&c.full[st], issued_parity[st], &zero))
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
        // epilogue: this CTA's partial logits, TMEM -> shared memory row `row`
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        if (!tc::mbar_wait(&c.acc_full, 0, abort_flag)) {
            *reinterpret_cast<volatile int*>(&c.abort) = 1;
            atomicExch(status, MOE_ERR_TIMEOUT);
        } else {
            tc::fence_after_sync();
            const uint32_t tb = tmem_base + ((uint32_t)(quad * 32) << 16);
            float* my = red + row * es;
            for (int c0 = 0; c0 < n_pad; c0 += 32) {  // n_pad <= es - 4: inside the row
                uint32_t r[32];
                tc::tmem_ld32(tb + c0, r);
                tc::tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4*>(my + c0 + j) =
                        make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                    __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
            }
        }
        tc::fence_before_sync();
    }

    constexpr int ROWS = BM / S;  // rows this CTA reduces and selects
    if constexpr (S > 1) {
        tc::cluster_sync();  // every CTA's partial rows are in its shared memory
        if (warp >= 2) {
            // 16-byte vectors of this CTA's rows; U vectors (U*S loads) in flight
            constexpr int U = S >= 8 ? 2 : 16 / S;
            const int etid = threadIdx.x - 64;
            const uint32_t red_addr = tc::smem_u32(red);
            uint32_t base[S];
#pragma unroll
            for (int sp = 0; sp < S; ++sp) base[sp] = tc::map_to_cta(red_addr, sp);
            const int v_row = (E + 3) / 4;
            const int n = ROWS * v_row;
            for (int i0 = etid; i0 < n; i0 += 128 * U) {
                float4 v[U][S];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int i = i0 + 128 * u;
                    if (i < n) {
                        const int r = split * ROWS + i / v_row, e4 = i - (i / v_row) * v_row;
                        const uint32_t off = (uint32_t)(r * es + 4 * e4) * 4u;
#pragma unroll
                        for (int sp = 0; sp < S; ++sp) v[u][sp] = tc::ld_cluster_f32x4(base[sp] + off);
                    }
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int i = i0 + 128 * u;
                    if (i < n) {
                        const int r = split * ROWS + i / v_row, e4 = i - (i / v_row) * v_row;
                        float4 z = v[u][0];
#pragma unroll
                        for (int sp = 1; sp < S; ++sp) {
                            z.x += v[u][sp].x; z.y += v[u][sp].y;
                            z.z += v[u][sp].z; z.w += v[u][sp].w;
                        }
                        // rows of this CTA's slice: read by no other CTA
                        *reinterpret_cast<float4*>(red + r * es + 4 * e4) = z;
                    }
                }
            }
        }
        tc::cluster_sync();  // all remote reads done before any CTA moves on or exits
    } else {
        __syncthreads();
    }
    if (warp >= 2) {
        // S lanes per token row of this CTA's slice (ROWS * S = 128 threads)
        const int tid = threadIdx.x - 64;
        const int rr = tid / S, part = tid % S;
        const long t = (long)tile * BM + split * ROWS + rr;
        const float* rw = red + (split * ROWS + rr) * es;
        const bool write = t < T;
        int* io = idx_out + (write ? t : 0) * k;
        float* wo = w_out + (write ? t : 0) * k;
        if (sbias)
            select_k<true, S>(k, rw, c.bias, c.sbias, E, scale, score_fn, part, write, io, wo);
        else
            select_k<false, S>(k, rw, c.bias, c.sbias, E, scale, score_fn, part, write, io, wo);
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

// Splits of the hidden dimension per token tile: a power of two <= 8 (the
// cluster size) such that tiles * S stays near the 148 SMs of a B200.
int router_splits(int T, int d) {
    const int tiles = (T + BM - 1) / BM;
    int s = 1;
    while (s < 8 && tiles * s * 2 <= 148 && s * 2 <= d / BK) s *= 2;
    return s;
}

bool router_tc_supported(const moe_config& c) { return c.k <= 8; }

namespace {

template <int S>
cudaError_t launch_s(dim3 grid, const CUtensorMap& mx, const CUtensorMap& mw, const moe_config& c,
                     int n_pad, const float* gate_bias, const float* score_bias, int score_fn,
                     int32_t* idx, float* w, int* status, cudaStream_t s) {
    cudaError_t err = cudaFuncSetAttribute(router_tc_kernel<S>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_pdl
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = S;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, router_tc_kernel<S>, mx, mw, gate_bias, score_bias, c.T, c.d,
                              c.E, c.k, n_pad, c.scale, score_fn, idx, w, status);
}

}  // namespace

cudaError_t launch_router_tc(const moe_config& c, const void* x, const void* w_gate,
                             const float* gate_bias, const float* score_bias, int score_fn,
                             int32_t* idx, float* w, int* status, cudaStream_t s) {
    const int tiles = (c.T + BM - 1) / BM;
    const int S = router_splits(c.T, c.d);
    const int n_pad = (c.E + 15) & ~15;
    CUtensorMap mx, mw;
    if (!make_map(&mx, x, c.T, c.d, BM) || !make_map(&mw, w_gate, c.E, c.d, n_pad))
        return cudaErrorInvalidValue;
    const dim3 grid(tiles, S);
    cudaError_t err;
    switch (S) {
        case 1:
            err = launch_s<1>(grid, mx, mw, c, n_pad, gate_bias, score_bias, score_fn, idx, w,
                               status, s);
            break;
        case 2:
            err = launch_s<2>(grid, mx, mw, c, n_pad, gate_bias, score_bias, score_fn, idx, w,
                               status, s);
            break;
        case 4:
            err = launch_s<4>(grid, mx, mw, c, n_pad, gate_bias, score_bias, score_fn, idx, w,
                               status, s);
            break;
        default:
            err = launch_s<8>(grid, mx, mw, c, n_pad, gate_bias, score_bias, score_fn, idx, w,
                               status, s);
            break;
    }
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

}  // namespace moe
