// experts_gemm.cu -- tensor-core grouped GEMMs of the SwiGLU experts (sm_100a).
//
// The pages replace the per-expert loop by a batched / grouped matrix multiply
// for throughput ("Tencent Hy3-Flash QA" Q6.4); the expert is a SwiGLU MLP
// without bias ("DeepSeek V4-Flash 架构 QA" Q4.5) whose gate and up projections
// are fused into one [2*d_ff, d] weight ("Tencent Hy3-295B 架构深度拆解" §2.3).
//
//   gate_up: h[r, f] = bf16( SiLU(<x_r, W[e, f]>) * <x_r, W[e, F + f]> )
//   down:    y[r, i] = bf16( <h_r, Wd[e, i]> )
//
// Mapping (swap-AB): the MMA's M side is 128 weight rows (output features) and
// its N side the expert's token rows, so an expert with ~170 rows fills one
// N <= 256 tile instead of padding 128-row token tiles. Each tile is
// 128 features x N tokens with N a multiple of 32 (token rows arrive in 32-row
// TMA boxes); an expert with more than 256 rows is split into equal tiles.
// The gate_up tile runs two MMAs per K step -- gate rows [f0, f0+128) and the
// matching up rows [F+f0, F+f0+128) -- into two TMEM accumulators, so the
// epilogue thread that owns feature f holds both g and u for every token and
// applies SiLU(g)*u in fp32 before the single bf16 rounding of h.
//
// Kernel: persistent, one CTA per SM, 224 threads.
//   warp 0     weight producer: per K block of 64, the weight tile(s) (128 rows
//              x 128 B, 128-byte swizzle) into a ring of shared-memory stages
//              (full/empty mbarriers), evict-first in L2;
//   warp 6     token producer: the tile's 32-row token boxes into a second,
//              shallower ring, evict-last in L2 (they are re-read by the CTAs
//              that share the expert);
//   warp 1     TMEM owner (alloc/dealloc of 512 columns) and MMA issuer:
//              tcgen05.mma kind::f16 (bf16 x bf16 -> fp32), M=128, K=16;
//              tcgen05.commit frees a stage / publishes an accumulator;
//   warps 2-5  epilogue: tcgen05.ld of their 32-lane quarter, SwiGLU (gate_up)
//              and bf16 stores of the tile's valid rows.
// Tiles are enumerated expert by expert (token tile major, weight tile minor),
// so the CTAs working at one time share the same experts' token rows in L2.
// Every mbarrier wait is bounded; a wait that gives up records MOE_ERR_TIMEOUT
// in the status word, drains its in-flight copies and MMAs and returns.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace moe {
namespace {

constexpr int BM = 128;     // weight rows per tile (MMA M)
constexpr int BK = 64;      // K per stage: one 128-byte swizzle row of bf16
constexpr int UK = 16;      // K per MMA instruction
constexpr int NMAX = 256;   // token rows per tile (MMA N upper bound)
constexpr int NBOX = 32;    // token rows per TMA box
constexpr int A_BYTES = BM * BK * 2;
constexpr int BOX_BYTES = NBOX * BK * 2;
constexpr int B_BYTES = NMAX * BK * 2;
constexpr int THREADS = 224;
constexpr int MAX_E = 256;

// Two rings: the weight tiles (streamed from HBM once) get the deeper one, the
// token boxes (re-read from L2 by the CTAs sharing an expert) a shallower one,
// each filled by its own producer warp.
template <bool GATE_UP>
struct Shape {
    static constexpr int A_TILES = GATE_UP ? 2 : 1;
    static constexpr int A_STAGE = A_TILES * A_BYTES;  // 32 KB / 16 KB
    static constexpr int A_STAGES = GATE_UP ? 3 : 6;
    static constexpr int B_STAGES = 3;
    static constexpr int RING_BYTES = A_STAGES * A_STAGE + B_STAGES * B_BYTES;
    static constexpr int ACC_STAGES = GATE_UP ? 1 : 2;
    static constexpr int ACC_COLS = GATE_UP ? 512 : 256;  // TMEM columns per accumulator stage
};

struct Ctrl {
    uint64_t a_full[6];
    uint64_t a_empty[6];
    uint64_t b_full[3];
    uint64_t b_empty[3];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int total;
    int off[MAX_E + 1];
    int tile_start[MAX_E + 1];
};

template <bool GATE_UP>
constexpr int smem_bytes() {
    return Shape<GATE_UP>::RING_BYTES + 1024 + (int)sizeof(Ctrl);
}

struct TileInfo {
    int e, m, row0, len, n;
};

__device__ __forceinline__ TileInfo decode_tile(const Ctrl& c, int E, int m_tiles, int t) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (c.tile_start[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int local = t - c.tile_start[e];
    const int n_e = c.off[e + 1] - c.off[e];
    const int nt = (n_e + NMAX - 1) / NMAX;
    const int j = local / m_tiles;
    const int base = n_e / nt, rem = n_e - base * nt;
    TileInfo ti;
    ti.e = e;
    ti.m = local - j * m_tiles;
    ti.row0 = c.off[e] + j * base + min(j, rem);
    ti.len = base + (j < rem ? 1 : 0);
    ti.n = (ti.len + NBOX - 1) & ~(NBOX - 1);
    return ti;
}

__device__ __forceinline__ void raise_timeout(Ctrl& c, int* status) {
    *reinterpret_cast<volatile int*>(&c.abort) = 1;
    atomicExch(status, MOE_ERR_TIMEOUT);
}

// Wait (bounded, abort ignored) until the last load issued into each stage of a
// ring has landed, so that no copy is in flight when the CTA exits.
template <int N>
__device__ __forceinline__ void drain_ring(uint64_t* full, const bool (&issued)[N],
                                           const uint32_t (&parity)[N], int* status) {
    const int zero = 0;
    for (int s = 0; s < N; ++s)
        if (issued[s] && !tc::mbar_wait(&full[s], parity[s], &zero))
            atomicExch(status, MOE_ERR_TIMEOUT);
}

// tmA: weights as a 2-D [rows = E*A_rows_per_expert, K] bf16 map, box 64 x 128.
// tmB: token rows as a 2-D [R, K] bf16 map, box 64 x 32.
// A_rows_per_expert = 2F (gate_up) or d (down); m_tiles = F/128 or d/128;
// out_ld = F (h) or d (y).
template <bool GATE_UP>
__global__ void __launch_bounds__(THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const int* __restrict__ offsets, int E, int K, int a_rows_per_expert,
                    int m_tiles, __nv_bfloat16* __restrict__ out, int out_ld,
                    int* __restrict__ status) {
    pdl_launch_and_wait();
    using S = Shape<GATE_UP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* a_ring = smem;
    uint8_t* b_ring = smem + S::A_STAGES * S::A_STAGE;
    Ctrl& c = *reinterpret_cast<Ctrl*>(smem + S::RING_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = K / BK;

    // ---- prologue: tile table (warp 0), barriers and TMEM (warp 1)
    if (warp == 0) {
        int carry = 0;
        for (int b = 0; b <= E; b += 32) {
            const int e = b + lane;
            int o = 0, cnt = 0;
            if (e <= E) {
                o = offsets[e];
                c.off[e] = o;
            }
            __syncwarp();
            if (e < E) {
                const int n_e = offsets[e + 1] - o;
                cnt = ((n_e + NMAX - 1) / NMAX) * m_tiles;
            }
            int incl = cnt;
#pragma unroll
            for (int s = 1; s < 32; s <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, s);
                if (lane >= s) incl += v;
            }
            if (e < E) c.tile_start[e] = carry + incl - cnt;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            c.tile_start[E] = carry;
            c.total = carry;
            c.abort = 0;
            tc::prefetch_tensormap(&tmA);
            tc::prefetch_tensormap(&tmB);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            for (int s = 0; s < S::A_STAGES; ++s) {
                tc::mbar_init(&c.a_full[s], 1);
                tc::mbar_init(&c.a_empty[s], 1);
            }
            for (int s = 0; s < S::B_STAGES; ++s) {
                tc::mbar_init(&c.b_full[s], 1);
                tc::mbar_init(&c.b_empty[s], 1);
            }
            for (int a = 0; a < S::ACC_STAGES; ++a) {
                tc::mbar_init(&c.acc_full[a], 1);
                tc::mbar_init(&c.acc_empty[a], 128);
            }
            tc::mbar_init(&c.drain, 1);
            tc::fence_mbar_init();
        }
        __syncwarp();
        tc::tmem_alloc(&c.tmem_base, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem_base = c.tmem_base;
    const int total = c.total;
    const volatile int* abort_flag = &c.abort;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- weight-tile producer (HBM stream, evict-first in L2)
            const uint64_t pol = tc::policy_evict_first();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t parity[S::A_STAGES] = {};
            bool issued[S::A_STAGES] = {};
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const TileInfo ti = decode_tile(c, E, m_tiles, t);
                const int a_row = ti.e * a_rows_per_expert + ti.m * BM;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!tc::mbar_wait(&c.a_empty[stage], phase ^ 1u, abort_flag)) {
                        raise_timeout(c, status);
                        ok = false;
                        break;
                    }
                    uint8_t* s = a_ring + stage * S::A_STAGE;
                    tc::mbar_arrive_expect_tx(&c.a_full[stage], S::A_STAGE);
                    tc::tma_load_2d_hint(s, &tmA, &c.a_full[stage], kb * BK, a_row, pol);
                    if (GATE_UP)
                        tc::tma_load_2d_hint(s + A_BYTES, &tmA, &c.a_full[stage], kb * BK,
                                             a_row + a_rows_per_expert / 2, pol);
                    issued[stage] = true;
                    parity[stage] = phase;
                    if (++stage == S::A_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            drain_ring(c.a_full, issued, parity, status);
        }
    } else if (warp == 6) {
        if (lane == 0) {
            // ---------------- token-box producer (L2-resident rows, evict-last)
            const uint64_t pol = tc::policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t parity[S::B_STAGES] = {};
            bool issued[S::B_STAGES] = {};
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const TileInfo ti = decode_tile(c, E, m_tiles, t);
                const int nb = ti.n / NBOX;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!tc::mbar_wait(&c.b_empty[stage], phase ^ 1u, abort_flag)) {
                        raise_timeout(c, status);
                        ok = false;
                        break;
                    }
                    uint8_t* s = b_ring + stage * B_BYTES;
                    tc::mbar_arrive_expect_tx(&c.b_full[stage], nb * BOX_BYTES);
                    for (int b = 0; b < nb; ++b)
                        tc::tma_load_2d_hint(s + b * BOX_BYTES, &tmB, &c.b_full[stage], kb * BK,
                                             ti.row0 + b * NBOX, pol);
                    issued[stage] = true;
                    parity[stage] = phase;
                    if (++stage == S::B_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            drain_ring(c.b_full, issued, parity, status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            int as = 0, bs = 0;
            uint32_t aph = 0, bph = 0;
            bool ok = true;
            int it = 0;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
                const TileInfo ti = decode_tile(c, E, m_tiles, t);
                const int acc = it % S::ACC_STAGES;
                const uint32_t acc_phase = (uint32_t)(it / S::ACC_STAGES) & 1u;
                if (!tc::mbar_wait(&c.acc_empty[acc], acc_phase ^ 1u, abort_flag)) {
                    raise_timeout(c, status);
                    break;
                }
                tc::fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * S::ACC_COLS;
                const uint32_t idesc = tc::idesc_bf16_f32(BM, ti.n);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!tc::mbar_wait(&c.a_full[as], aph, abort_flag) ||
                        !tc::mbar_wait(&c.b_full[bs], bph, abort_flag)) {
                        raise_timeout(c, status);
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint32_t a_addr = tc::smem_u32(a_ring + as * S::A_STAGE);
                    const uint32_t b_addr = tc::smem_u32(b_ring + bs * B_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / UK; ++k) {
                        const uint64_t bdesc = tc::desc_sw128(b_addr + k * UK * 2);
                        const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
                        tc::mma_bf16(d_tmem, tc::desc_sw128(a_addr + k * UK * 2), bdesc, idesc,
                                     accum);
                        if (GATE_UP)
                            tc::mma_bf16(d_tmem + 256, tc::desc_sw128(a_addr + A_BYTES + k * UK * 2),
                                         bdesc, idesc, accum);
                    }
                    tc::mma_commit(&c.a_empty[as]);
                    tc::mma_commit(&c.b_empty[bs]);
                    if (++as == S::A_STAGES) {
                        as = 0;
                        aph ^= 1u;
                    }
                    if (++bs == S::B_STAGES) {
                        bs = 0;
                        bph ^= 1u;
                    }
                }
                if (ok) tc::mma_commit(&c.acc_full[acc]);
            }
            // drain: all MMAs issued by this thread have completed
            tc::mma_commit(&c.drain);
            const int zero = 0;
            if (!tc::mbar_wait(&c.drain, 0, &zero)) atomicExch(status, MOE_ERR_TIMEOUT);
        }
    } else {
        // ---------------- epilogue: warps 2..5 own TMEM lane quarters (warp % 4)
        const int quad = warp & 3;
        const int row_in_tile = quad * 32 + lane;
        uint16_t* o16 = reinterpret_cast<uint16_t*>(out);
        int it = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
            const TileInfo ti = decode_tile(c, E, m_tiles, t);
            const int acc = it % S::ACC_STAGES;
            const uint32_t acc_phase = (uint32_t)(it / S::ACC_STAGES) & 1u;
            if (!tc::mbar_wait(&c.acc_full[acc], acc_phase, abort_flag)) {
                raise_timeout(c, status);
                break;
            }
            tc::fence_after_sync();
            const uint32_t tbase = tmem_base + acc * S::ACC_COLS + ((uint32_t)(quad * 32) << 16);
            const int col = ti.m * BM + row_in_tile;
            for (int c0 = 0; c0 < ti.n; c0 += 32) {
                uint32_t g[32];
                tc::tmem_ld32(tbase + c0, g);
                if constexpr (GATE_UP) {
                    uint32_t u[32];
                    tc::tmem_ld32(tbase + 256 + c0, u);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int n = c0 + j;
                        if (n < ti.len) {
                            const float gv = __uint_as_float(g[j]), uv = __uint_as_float(u[j]);
                            const float hv = silu_mul(gv, uv);
                            o16[(size_t)(ti.row0 + n) * out_ld + col] = float_to_bf16_bits(hv);
                        }
                    }
                } else {
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int n = c0 + j;
                        if (n < ti.len)
                            o16[(size_t)(ti.row0 + n) * out_ld + col] =
                                float_to_bf16_bits(__uint_as_float(g[j]));
                    }
                }
            }
            tc::fence_before_sync();
            tc::mbar_arrive(&c.acc_empty[acc]);
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem_base, 512);
    }
}

// ---------------------------------------------------------------- host side

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

// Row-major [rows, cols] bf16 tensor, box of box_rows x 64 columns, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int sm_count() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

template <bool GATE_UP>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& b, const int32_t* offsets, int E,
                   int K, int a_rows_per_expert, int m_tiles, void* out, int out_ld, int* status,
                   cudaStream_t s) {
    const int smem = smem_bytes<GATE_UP>();
    cudaError_t err = cudaFuncSetAttribute(grouped_gemm_kernel<GATE_UP>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    err = launch_pdl(grouped_gemm_kernel<GATE_UP>, dim3(sm_count()), dim3(THREADS), smem, s, a, b,
                     offsets, E, K, a_rows_per_expert, m_tiles, static_cast<__nv_bfloat16*>(out),
                     out_ld, status);
    return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate_up_gemm(const moe_config& c, const void* x_perm, const int32_t* offsets,
                                const void* w_gate_up, void* h, int* status, cudaStream_t s) {
    CUtensorMap a, b;
    const uint64_t R = (uint64_t)c.T * c.k;
    if (!make_map(&a, w_gate_up, (uint64_t)c.E * 2 * c.d_ff, c.d, BM) ||
        !make_map(&b, x_perm, R, c.d, NBOX))
        return cudaErrorInvalidValue;
    return launch<true>(a, b, offsets, c.E, c.d, 2 * c.d_ff, c.d_ff / BM, h, c.d_ff, status, s);
}

cudaError_t launch_down_gemm(const moe_config& c, const void* h, const int32_t* offsets,
                             const void* w_down, void* y, int* status, cudaStream_t s) {
    CUtensorMap a, b;
    const uint64_t R = (uint64_t)c.T * c.k;
    if (!make_map(&a, w_down, (uint64_t)c.E * c.d, c.d_ff, BM) ||
        !make_map(&b, h, R, c.d_ff, NBOX))
        return cudaErrorInvalidValue;
    return launch<false>(a, b, offsets, c.E, c.d_ff, c.d, c.d / BM, y, c.d, status, s);
}

}  // namespace moe
