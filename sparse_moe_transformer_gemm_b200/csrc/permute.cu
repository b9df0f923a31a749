// permute.cu -- group token-slots by expert (a stable counting sort) and gather
// the activation rows into expert-contiguous order for the expert GEMMs.
//
// The pages run the experts as a loop over the selected experts with an
// index_add_ accumulation ("DeepSeek V4-Flash 架构 QA", Q8.4) and name batched
// / grouped matrix multiplication as the production form ("Tencent Hy3-Flash
// QA", Q6.4). Grouping the rows of each expert contiguously is what makes the
// grouped form possible.
//
// Definition (integer, bit-exact): slot s = t*k + j with expert e = idx[s] goes
// to row offsets[e] + #{s' < s : idx[s'] == e}; offsets is the exclusive prefix
// sum of the per-expert counts.
//
// Three launches (moe_permute):
//   rank    one CTA per chunk of kPermuteChunk slots, a warp per quarter of it:
//           rank of each slot among the earlier slots of its chunk with the
//           same expert (__match_any_sync per 32-slot group, running
//           per-expert counters in shared memory, the earlier warps' counts
//           added in a second pass), and the chunk's per-expert histogram;
//   scan    one CTA: per expert, exclusive prefix over chunks (the chunk base),
//           the totals (counts) and the exclusive prefix over experts (offsets);
//   scatter one warp per slot: row = offsets[e] + chunk base + rank; copies the
//           token's d-element row into x_perm with 16-byte vectors.
// Slots whose expert id is outside [0, E) are dropped: row_of = -1.
//
// moe_permute_index runs the same rank and scan and replaces the scatter by an
// index-only one (thread per slot) that also writes token_of_row, the token of
// each grouped row; the gate_up GEMM then gathers the token rows from x
// itself and no permuted copy of the activations is written. Small batches
// (at most 4096 slots) run all of it in one CTA.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int CH = kPermuteChunk;

// The expert of token-slot s. Without a shared expert the slots are the
// routing array itself (kk == k); with one, every token has kk = k + 1 slots
// and its last slot is the shared expert e_shared.
struct Slots {
    const int* idx;  // [T, k]
    int k, kk, e_shared;
};

__device__ __forceinline__ int slot_expert(const Slots& m, long s) {
    if (m.kk == m.k) return m.idx[s];
    const long t = s / m.kk;
    const int j = (int)(s - t * m.kk);
    return j < m.k ? m.idx[t * m.k + j] : m.e_shared;
}

inline Slots slots_of(const moe_config& c, const int32_t* idx) {
    return Slots{idx, c.k, c.k + shared_slots(c), c.E};
}

// One warp copies a row of n16 16-byte vectors, eight loads in flight per lane.
__device__ __forceinline__ void copy_row(uint4* __restrict__ dst, const uint4* __restrict__ src,
                                         int n16, int lane) {
    for (int v0 = lane; v0 < n16; v0 += 32 * 8) {
        uint4 u[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (v0 + 32 * i < n16) u[i] = src[v0 + 32 * i];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (v0 + 32 * i < n16) dst[v0 + 32 * i] = u[i];
    }
}

// Ranking: CTA per chunk of CH slots, RW warps on consecutive sub-chunks of
// CH / RW slots. Each warp ranks its slots among its own earlier ones; the
// per-expert counts of the warps are then prefix-summed so that a second pass
// adds each warp's base.
constexpr int RW = 4;
constexpr int SUB = CH / RW;

__global__ void __launch_bounds__(RW * 32)
permute_rank_kernel(Slots sl, long R, int E, int* __restrict__ hist, int* __restrict__ rank) {
    pdl_launch_and_wait();
    __shared__ int cnt[RW][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < RW * 256; i += blockDim.x) cnt[i >> 8][i & 255] = 0;
    __syncthreads();
    const long base = (long)blockIdx.x * CH + (long)warp * SUB;
    for (int g = 0; g < SUB; g += 32) {
        const long s = base + g + lane;
        int e = (s < R) ? slot_expert(sl, s) : -1;
        if (e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int before = (e >= 0) ? cnt[warp][e] : 0;
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) cnt[warp][e] = before + __popc(peers);
        __syncwarp();
        if (s < R) rank[s] = before + __popc(peers & ((1u << lane) - 1u));
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < RW; ++w) {
            const int v = cnt[w][e];
            cnt[w][e] = run;
            run += v;
        }
        hist[(long)blockIdx.x * E + e] = run;
    }
    __syncthreads();
    if (warp == 0) return;  // warp 0's base is 0 for every expert
    for (int g = 0; g < SUB; g += 32) {
        const long s = base + g + lane;
        if (s < R) {
            const int e = slot_expert(sl, s);
            if (e >= 0 && e < E) rank[s] += cnt[warp][e];
        }
    }
}

__global__ void __launch_bounds__(256)
permute_scan_kernel(int* __restrict__ hist, int C, int E, int* __restrict__ counts,
                    int* __restrict__ offsets) {
    pdl_launch_and_wait();
    __shared__ int tile[32][256];
    __shared__ int tot[256];
    const int e = threadIdx.x;
    int running = 0;
    for (int c0 = 0; c0 < C; c0 += 32) {
        const int nc = min(32, C - c0);
        __syncthreads();
        for (int v = threadIdx.x; v < nc * E; v += blockDim.x)
            tile[v / E][v % E] = hist[(long)c0 * E + v];
        __syncthreads();
        if (e < E)
            for (int c = 0; c < nc; ++c) {
                const int v = tile[c][e];
                tile[c][e] = running;
                running += v;
            }
        __syncthreads();
        for (int v = threadIdx.x; v < nc * E; v += blockDim.x)
            hist[(long)c0 * E + v] = tile[v / E][v % E];
    }
    tot[e] = (e < E) ? running : 0;
    __syncthreads();
    if (threadIdx.x < 32) {
        // exclusive prefix over the experts: lane handles experts [8*lane, 8*lane+8)
        const int lane = threadIdx.x;
        int v[8], sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[i] = tot[lane * 8 + i];
            sum += v[i];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        int run = incl - sum;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            tot[lane * 8 + i] = run;
            run += v[i];
        }
        if (lane == 31) offsets[E] = incl;
    }
    __syncthreads();
    if (e < E) {
        counts[e] = running;
        offsets[e] = tot[e];
    }
}

__global__ void __launch_bounds__(256)
permute_scatter_kernel(Slots sl, const int* __restrict__ hist, const int* __restrict__ rank,
                       const int* __restrict__ offsets, const __nv_bfloat16* __restrict__ x,
                       long R, int E, int d, int* __restrict__ row_of,
                       __nv_bfloat16* __restrict__ xperm) {
    pdl_launch_and_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long s = (long)blockIdx.x * 8 + warp;
    if (s >= R) return;
    const int e = slot_expert(sl, s);
    if (e < 0 || e >= E) {
        if (lane == 0) row_of[s] = -1;
        return;
    }
    const long c = s / CH;
    const int row = offsets[e] + hist[c * E + e] + rank[s];
    if (lane == 0) row_of[s] = row;
    const long t = s / sl.kk;
    const uint4* src = reinterpret_cast<const uint4*>(x + t * d);
    uint4* dst = reinterpret_cast<uint4*>(xperm + (long)row * d);
    copy_row(dst, src, d / 8, lane);
}

// Index-only scatter, one thread per slot: row_of and its inverse
// token_of_row[row] = t, for expert GEMMs that gather the token rows
// themselves.
__global__ void __launch_bounds__(256)
permute_index_kernel(Slots sl, const int* __restrict__ hist, const int* __restrict__ rank,
                     const int* __restrict__ offsets, long R, int E, int* __restrict__ row_of,
                     int* __restrict__ token_of_row) {
    pdl_launch_and_wait();
    const long s = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= R) return;
    const int e = slot_expert(sl, s);
    if (e < 0 || e >= E) {
        row_of[s] = -1;
        return;
    }
    const int row = offsets[e] + hist[(s / CH) * E + e] + rank[s];
    row_of[s] = row;
    token_of_row[row] = (int)(s / sl.kk);
}

// The whole index-only grouping in one CTA for small batches (R <= SW * 128
// slots, decode): warp w owns the slots [w*per, (w+1)*per). Pass 1 counts each
// warp's slots per expert; a scan over warps (per expert) and over experts
// gives each warp's first row per expert; pass 2 ranks the slots again in the
// same order and writes row_of and token_of_row. Same result as the
// rank/scan/scatter launches.
constexpr int SW = 32;  // warps of the small-batch kernel
constexpr long kSmallSlots = SW * 128;

__global__ void __launch_bounds__(SW * 32)
permute_small_kernel(Slots sl, long R, int E, int* __restrict__ counts,
                     int* __restrict__ offsets, int* __restrict__ row_of,
                     int* __restrict__ token_of_row) {
    pdl_launch_and_wait();
    __shared__ int cnt[SW][256];
    __shared__ int base[256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per = (int)(((R + SW - 1) / SW + 31) & ~31L);
    for (int i = threadIdx.x; i < SW * 256; i += blockDim.x) cnt[i >> 8][i & 255] = 0;
    __syncthreads();
    const long s0 = (long)warp * per;
    for (int g = 0; g < per; g += 32) {
        const long s = s0 + g + lane;
        int e = (s < R) ? slot_expert(sl, s) : -1;
        if (e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && lane == __ffs(peers) - 1) cnt[warp][e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // per expert: exclusive prefix over warps; totals into base[]
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int w = 0; w < SW; ++w) {
            const int v = cnt[w][e];
            cnt[w][e] = run;
            run += v;
        }
        base[e] = run;
        counts[e] = run;
    }
    __syncthreads();
    if (warp == 0) {
        // exclusive prefix over experts: lane handles experts [8*lane, 8*lane+8)
        int v[8], sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane * 8 + i;
            v[i] = (e < E) ? base[e] : 0;
            sum += v[i];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        int run = incl - sum;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane * 8 + i;
            if (e < E) {
                base[e] = run;
                offsets[e] = run;
            }
            run += v[i];
        }
        if (lane == 31) offsets[E] = incl;
    }
    __syncthreads();
    for (int g = 0; g < per; g += 32) {
        const long s = s0 + g + lane;
        int e = (s < R) ? slot_expert(sl, s) : -1;
        if (e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int before = (e >= 0) ? cnt[warp][e] : 0;
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) cnt[warp][e] = before + __popc(peers);
        __syncwarp();
        if (s < R) {
            if (e < 0) {
                row_of[s] = -1;
            } else {
                const int row = base[e] + before + __popc(peers & ((1u << lane) - 1u));
                row_of[s] = row;
                token_of_row[row] = (int)(s / sl.kk);
            }
        }
    }
}

// x_perm[row] = x[token_of_row[row]] for rows [0, offsets[E]): one warp per row.
__global__ void __launch_bounds__(256)
gather_rows_kernel(const __nv_bfloat16* __restrict__ x, const int* __restrict__ token_of_row,
                   const int* __restrict__ offsets, long R, int E, int d,
                   __nv_bfloat16* __restrict__ xperm) {
    pdl_launch_and_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long row = (long)blockIdx.x * 8 + warp;
    if (row >= R || row >= offsets[E]) return;
    const uint4* src = reinterpret_cast<const uint4*>(x + (long)token_of_row[row] * d);
    uint4* dst = reinterpret_cast<uint4*>(xperm + row * d);
    copy_row(dst, src, d / 8, lane);
}

}  // namespace

cudaError_t launch_permute_index(const moe_config& c, const int32_t* idx, int32_t* counts,
                                 int32_t* offsets, int32_t* row_of, int32_t* token_of_row,
                                 int32_t* hist, int32_t* rank, cudaStream_t s) {
    const moe_config g = grouped_config(c);
    const Slots sl = slots_of(c, idx);
    const long R = (long)g.T * g.k;
    if (R <= kSmallSlots) {
        const cudaError_t err = launch_pdl(permute_small_kernel, dim3(1), dim3(SW * 32), 0, s, sl,
                                           R, g.E, counts, offsets, row_of, token_of_row);
        return err != cudaSuccess ? err : cudaGetLastError();
    }
    const int C = n_permute_chunks(g);
    cudaError_t err = launch_pdl(permute_rank_kernel, dim3(C), dim3(RW * 32), 0, s, sl, R, g.E,
                                 hist, rank);
    if (err == cudaSuccess)
        err = launch_pdl(permute_scan_kernel, dim3(1), dim3(256), 0, s, hist, C, g.E, counts,
                         offsets);
    if (err == cudaSuccess)
        err = launch_pdl(permute_index_kernel, dim3((unsigned)((R + 255) / 256)), dim3(256), 0, s,
                         sl, hist, rank, offsets, R, g.E, row_of, token_of_row);
    return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t launch_gather_rows(const moe_config& c, const void* x, const int32_t* token_of_row,
                               const int32_t* offsets, void* x_perm, cudaStream_t s) {
    const moe_config g = grouped_config(c);
    const long R = (long)g.T * g.k;
    const cudaError_t err = launch_pdl(gather_rows_kernel, dim3((unsigned)((R + 7) / 8)), dim3(256),
                                       0, s, static_cast<const __nv_bfloat16*>(x), token_of_row,
                                       offsets, R, g.E, c.d, static_cast<__nv_bfloat16*>(x_perm));
    return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t launch_permute(const moe_config& c, const int32_t* idx, const void* x, int32_t* counts,
                           int32_t* offsets, int32_t* row_of, void* x_perm, int32_t* hist,
                           int32_t* rank, cudaStream_t s) {
    const moe_config g = grouped_config(c);
    const Slots sl = slots_of(c, idx);
    const long R = (long)g.T * g.k;
    const int C = n_permute_chunks(g);
    cudaError_t err = launch_pdl(permute_rank_kernel, dim3(C), dim3(RW * 32), 0, s, sl, R, g.E,
                                 hist, rank);
    if (err == cudaSuccess)
        err = launch_pdl(permute_scan_kernel, dim3(1), dim3(256), 0, s, hist, C, g.E, counts,
                         offsets);
    if (err == cudaSuccess)
        err = launch_pdl(permute_scatter_kernel, dim3((unsigned)((R + 7) / 8)), dim3(256), 0, s,
                         sl, hist, rank, offsets, static_cast<const __nv_bfloat16*>(x), R, g.E,
                         c.d, row_of, static_cast<__nv_bfloat16*>(x_perm));
    return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
