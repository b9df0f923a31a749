// ep.cu -- expert parallelism: the local expert of every row a rank receives.
//
// Expert parallelism ("DeepSeek V4-Flash 架构 QA", Q4.7 expert-parallel
// strategy and Q4.10 the MoE's communication): P ranks each hold E/P of the
// experts; every rank routes its own tokens, groups their token-slots by
// expert (moe_permute: experts of one rank are contiguous, so the grouped rows
// are already one block per destination rank) and sends each block to the
// rank that owns those experts. A receiving rank gets one block per source,
// each grouped by its E_local experts, with counts[src][e] rows of local
// expert e. To run its grouped GEMMs it regroups the received rows by expert
// (moe_permute with k = 1 and these ids as the routing), which needs the
// local expert of each received row: row r lies in segment (src, e) of the
// source-major, expert-minor concatenation. This kernel writes that id.
//
// Structure: every CTA computes the exclusive prefix sum of the n_seg =
// n_src * E_local counts in shared memory (a block-wide scan, counts in fixed
// order), then each thread takes rows of the CTA's chunk and finds its segment
// by binary search over the prefix sums. Rows at or past the counts' total
// get -1.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int EP_THREADS = 256;
constexpr int EP_ROWS_PER_CTA = 4096;

__global__ void __launch_bounds__(EP_THREADS)
ep_row_experts_kernel(const int32_t* __restrict__ counts, int n_seg, int e_local,
                      int32_t* __restrict__ expert_of_row, int n_rows) {
    pdl_launch_and_wait();
    extern __shared__ int start[];  // [n_seg + 1] exclusive prefix sums
    __shared__ int warp_tot[EP_THREADS / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // each thread sums a run of consecutive counts, the runs in thread order
    const int per = (n_seg + EP_THREADS - 1) / EP_THREADS;
    const int s0 = tid * per;
    int run = 0;
    for (int s = s0; s < min(s0 + per, n_seg); ++s) run += counts[s];
    // inclusive scan of the runs: within the warp, then over the warp totals
    int inc = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += v;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int wt = lane < EP_THREADS / 32 ? warp_tot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, wt, o);
            if (lane >= o) wt += v;
        }
        if (lane < EP_THREADS / 32) warp_tot[lane] = wt;  // inclusive over warps
    }
    __syncthreads();
    int base = inc - run + (warp > 0 ? warp_tot[warp - 1] : 0);  // exclusive
    for (int s = s0; s < min(s0 + per, n_seg); ++s) {
        start[s] = base;
        base += counts[s];
    }
    if (tid == EP_THREADS - 1) start[n_seg] = warp_tot[EP_THREADS / 32 - 1];
    __syncthreads();
    const int total = start[n_seg];
    const int r_end = min(n_rows, (blockIdx.x + 1) * EP_ROWS_PER_CTA);
    for (int r = blockIdx.x * EP_ROWS_PER_CTA + tid; r < r_end; r += EP_THREADS) {
        if (r >= total) {
            expert_of_row[r] = -1;
            continue;
        }
        // the last segment whose start is <= r (empty segments share a start)
        int lo = 0, hi = n_seg - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (start[mid] <= r) lo = mid; else hi = mid - 1;
        }
        expert_of_row[r] = lo % e_local;
    }
}

}  // namespace

cudaError_t launch_ep_row_experts(const int32_t* counts, int n_src, int e_local,
                                  int32_t* expert_of_row, int n_rows, cudaStream_t s) {
    const int n_seg = n_src * e_local;
    const int grid = (n_rows + EP_ROWS_PER_CTA - 1) / EP_ROWS_PER_CTA;
    const cudaError_t err = launch_pdl(ep_row_experts_kernel, grid, dim3(EP_THREADS),
                                       sizeof(int) * (n_seg + 1), s, counts, n_seg, e_local,
                                       expert_of_row, n_rows);
    return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe

extern "C" int moe_ep_row_experts(const int32_t* counts, int32_t n_src, int32_t e_local,
                                  int32_t* expert_of_row, int32_t n_rows, void* stream) {
    if (!counts || !expert_of_row) return MOE_ERR_INVALID_ARG;
    if (n_src < 1 || e_local < 1 || e_local > 256 || n_rows < 1 ||
        (long long)n_src * e_local > MOE_EP_MAX_SEGMENTS)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    return moe::launch_ep_row_experts(counts, n_src, e_local, expert_of_row, n_rows,
                                      static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}
