// experts_gemm2.cu -- the SwiGLU experts' grouped GEMMs on pairs of SMs
// (tcgen05 cta_group::2), for shapes whose weight rows split into 256-row tiles.
//
// Same mathematics as experts_gemm.cu ("DeepSeek V4-Flash 架构 QA" Q4.5 SwiGLU;
// "Tencent Hy3-295B 架构深度拆解" §2.3 fused gate_up_proj [2F, d] and down_proj
// [d, F]; "Tencent Hy3-Flash QA" Q6.4 grouped matmul):
//   gate_up: h[r, f] = bf16( SiLU(<x_r, W[e, f]>) * <x_r, W[e, F + f]> )
//   down:    y[r, i] = bf16( <h_r, Wd[e, i]> )
//
// A cluster of two CTAs (two SMs) computes one 256-weight-row x N-token tile
// with M=256 MMAs: each CTA stages its own 128 weight rows and half of the N
// token rows, and the even CTA's single MMA thread drives the tensor cores of
// both. Compared with one CTA per 128 rows this halves the token rows each SM
// pulls from L2 per K step and frees shared memory for a deeper weight ring
// (more weight bytes in flight per SM, the bound of this HBM-bound stream).
//
// Per CTA (320 threads): warp 0 TMA producer (its weight rows + its token
// half; completion counted on the even CTA's "full" barrier, which expects the
// bytes of both CTAs), warp 1 TMEM owner (+ MMA issuer in the even CTA), warps
// 2-9 epilogue of the CTA's own 128 rows in two groups of four warps (one per
// TMEM lane quarter) that take alternate 32-token chunks. Stage release and
// accumulator hand-off are tcgen05.commit arrivals multicast to both CTAs; the
// epilogues hand the accumulator back with one arrival per CTA on the even
// CTA's barrier. No TMA load uses multicast. All waits are bounded.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace moe {
namespace {

constexpr int BM = 128;       // weight rows per CTA (MMA M = 256 per pair)
constexpr int BK = 64;
constexpr int UK = 16;
constexpr int NMAX = 256;     // token rows per pair tile
constexpr int NBOX = 16;      // token rows per TMA box
constexpr int A_BYTES = BM * BK * 2;
constexpr int EPI_GROUPS = 2;                      // epilogue warp groups (4 warps each)
constexpr int THREADS = 64 + 128 * EPI_GROUPS;     // producer, MMA, epilogue warps
constexpr int MAX_E = 256;
constexpr int EPI_N = 32;                          // tokens per epilogue chunk
constexpr int EPI_BYTES = 2 * EPI_N * BM * 2;      // two [EPI_N][BM] bf16 staging tiles

// Token-row tensor maps with boxes of 16, 32, 64 and 128 rows: a CTA's half of
// a tile (a multiple of 16 rows, at most 128) loads as at most four boxes
// (its binary decomposition) instead of up to eight 16-row boxes. The gather
// variant uses m[0] only, with a one-row box.
struct TokenMaps {
    CUtensorMap m[4];
};

__device__ __forceinline__ void load_token_rows(uint8_t* dst, const TokenMaps& tm,
                                                uint32_t bar_leader, int kx, int row, int rows,
                                                uint64_t pol) {
    // one copy site in a rolled loop: an unrolled form with four predicated copies
    // measured slower on B200 even where only the 16-row box was used
    for (int off = 0; off < rows;) {
        const int rem = rows - off;
        const int lg = rem >= 8 * NBOX ? 3 : rem >= 4 * NBOX ? 2 : rem >= 2 * NBOX ? 1 : 0;
        tc::tma_load_2d_pair(dst + off * (BK * 2), &tm.m[lg], bar_leader, kx, row + off, pol);
        off += NBOX << lg;
    }
}

// A pair tile takes two A tiles of 256 weight rows (128 per CTA) against the
// same token rows -- gate_up: the gate rows m*256.. and the up rows
// F + m*256..; down: the rows m*512.. and m*512 + 256.. -- into two TMEM
// accumulators, so each token stage feeds two MMAs per K step. (down with one
// A tile, a double-buffered accumulator and 6 stages ran 10% slower at the
// Hy3 prefill shape and 1.5% slower at decode.) Where d is an odd multiple of
// 256, down's last tile has its first A tile only.
//
// NM, the most token rows of a pair tile: 256, or 64 where no expert can have
// more rows (T <= 64: a token takes an expert once). With NM = 64 a stage
// holds 4 KB of token rows instead of 16, so the ring is 5 stages deep (the
// weight stream is HBM-bound and a shallower ring measured slower), and the
// two accumulators of 64 columns are double-buffered (the epilogue of a tile
// overlaps the next tile's MMAs).
template <bool GATE_UP, int NM = NMAX>
struct Shape {
    static constexpr int A_TILES = 2;
    static constexpr int BH = (NM / 2) * BK * 2;          // this CTA's half of the token rows
    static constexpr int STAGE_BYTES = A_TILES * A_BYTES + BH;  // 48 KB / 36 KB
    static constexpr int STAGES = NM == NMAX ? 4 : 5;
    static constexpr int U_OFF = NM;                      // the second accumulator's columns
    static constexpr int ACC_COLS = 2 * NM;               // two accumulators
    static constexpr int ACC_STAGES = 512 / ACC_COLS >= 2 ? 2 : 1;
    static constexpr int M_ROWS = GATE_UP ? 2 * BM : 4 * BM;  // weight rows per m (per expert)
};
constexpr int NM_SMALL = 64;

struct Ctrl {
    uint64_t full[6];       // even CTA: TMA bytes of both CTAs landed
    uint64_t empty[6];      // both CTAs: the pair MMAs finished reading the stage
    uint64_t acc_full[2];   // both CTAs: accumulator ready
    uint64_t acc_empty[2];  // even CTA: both epilogues done with the accumulator
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int total;
    int off[MAX_E + 1];
    int tile_start[MAX_E + 1];
};

template <bool GATE_UP, int NM>
constexpr int smem_bytes() {
    return Shape<GATE_UP, NM>::STAGES * Shape<GATE_UP, NM>::STAGE_BYTES + EPI_BYTES + 1024 +
           (int)sizeof(Ctrl);
}
static_assert(smem_bytes<true, NMAX>() <= 232448 && smem_bytes<false, NMAX>() <= 232448 &&
                  smem_bytes<true, NM_SMALL>() <= 232448 && smem_bytes<false, NM_SMALL>() <= 232448,
              "fits in 227 KB");
static_assert(Shape<true, NM_SMALL>::STAGES <= 6 && Shape<true, NMAX>::STAGES <= 6,
              "Ctrl's stage barriers");

struct TileInfo {
    int e, m, row0, len, n;  // n: MMA N of the pair, a multiple of 2*NBOX
};

template <int NM = NMAX, typename CtrlT>
__device__ __forceinline__ TileInfo decode_tile(const CtrlT& c, int E, int m_tiles, int t) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (c.tile_start[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int local = t - c.tile_start[e];
    const int n_e = c.off[e + 1] - c.off[e];
    // nt = ceil(n_e / NM) token tiles; all but the last hold 32q rows, so only
    // the last one pads its MMA N to a multiple of 32 (near-equal tiles would pad
    // every one: 341 rows as 171 + 170 run N = 192 + 192, as 192 + 149 run
    // 192 + 160). q = ceil(ceil(n_e / 32) / nt), or NM / 32 if that left the
    // last tile empty; every tile then holds 1..NM rows.
    const int nt = (n_e + NM - 1) / NM;
    const int units = (n_e + 2 * NBOX - 1) / (2 * NBOX);
    int q = (units + nt - 1) / nt;
    if (2 * NBOX * q * (nt - 1) >= n_e) q = NM / (2 * NBOX);
    // token tiles fastest: the tiles that read the same weight rows (same m,
    // next j) get neighbouring indices, so concurrent SM pairs stream those
    // weights from HBM once and from L2 for the others
    const int j = local % nt;
    TileInfo ti;
    ti.e = e;
    ti.m = local / nt;
    ti.row0 = c.off[e] + j * 2 * NBOX * q;
    ti.len = j < nt - 1 ? 2 * NBOX * q : n_e - 2 * NBOX * q * (nt - 1);
    ti.n = (ti.len + 2 * NBOX - 1) & ~(2 * NBOX - 1);
    return ti;
}

template <typename CtrlT>
__device__ __forceinline__ void raise_timeout(CtrlT& c, int* status) {
    *reinterpret_cast<volatile int*>(&c.abort) = 1;
    atomicExch(status, MOE_ERR_TIMEOUT);
}

// tmA: weights [E * a_rows_per_expert, K] bf16, box 64 x 128; with packed_a the
// same bytes in 128 x 64 blocks, viewed as [E * a_rows_per_expert * K / 64, 64].
// tmB: token rows [R, K] bf16, boxes of 64 columns x 16/32/64/128 rows.
// m_tiles: 256-row weight tiles per expert (F/256 for gate_up, d/256 for down).
// GATHER: tmB maps the unpermuted token rows x [T, K] with a one-row box and
// the token rows of each tile are gathered by index (token_of_row) with
// tile::gather4 instead of being read from a permuted copy.
template <bool GATE_UP, bool GATHER, int NM>
__global__ void __launch_bounds__(THREADS, 1)
grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ TokenMaps tmB, const int* __restrict__ offsets,
                         const int* __restrict__ token_of_row, int E, int K,
                         int a_rows_per_expert, int m_tiles, int packed_a,
                         __nv_bfloat16* __restrict__ out, int out_ld, int* __restrict__ status,
                         const uint8_t* __restrict__ pf, long long pf_bytes) {
    pdl_launch();
    // The weights are read-only in the layer, so their first pf_bytes (the
    // first experts' tiles) may be pulled into L2 before the wait for the
    // previous kernel: thread blocks that are resident while the router and
    // the grouping still run start the weight stream under them. One slice per
    // CTA, in 64 KB requests.
    if (pf_bytes > 0 && threadIdx.x == 0) {
        const long long per = ((pf_bytes + gridDim.x - 1) / gridDim.x + 15) & ~15ll;
        const long long b0 = (long long)blockIdx.x * per;
        const long long b1 = b0 + per < pf_bytes ? b0 + per : pf_bytes;
        for (long long o = b0; o < b1; o += 65536)
            tc::prefetch_l2_bulk(pf + o, (uint32_t)(b1 - o < 65536 ? b1 - o : 65536));
    }
    pdl_wait();
    using S = Shape<GATE_UP, NM>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint16_t* epi = reinterpret_cast<uint16_t*>(smem + S::STAGES * S::STAGE_BYTES);
    Ctrl& c = *reinterpret_cast<Ctrl*>(smem + S::STAGES * S::STAGE_BYTES + EPI_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)(tc::cluster_ctarank() & 1u);
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    const int KB = K / BK;

    // ---- prologue: tile table (warp 0), barriers and TMEM (warp 1), in both CTAs
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
                cnt = ((n_e + NM - 1) / NM) * m_tiles;
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
            for (int m = 0; m < (GATHER ? 1 : 4); ++m) tc::prefetch_tensormap(&tmB.m[m]);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            for (int s = 0; s < S::STAGES; ++s) {
                tc::mbar_init(&c.full[s], 1);
                tc::mbar_init(&c.empty[s], 1);
            }
            for (int a = 0; a < S::ACC_STAGES; ++a) {
                tc::mbar_init(&c.acc_full[a], 1);
                tc::mbar_init(&c.acc_empty[a], 2);
            }
            tc::mbar_init(&c.drain, 1);
            tc::fence_mbar_init();
        }
        __syncwarp();
        tc::tmem_alloc_pair(&c.tmem_base, 512);
        tc::tmem_relinquish_pair();
    }
    tc::fence_before_sync();
    tc::cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
    tc::fence_after_sync();
    const uint32_t tmem_base = c.tmem_base;
    const int total = c.total;
    const volatile int* abort_flag = &c.abort;
    // the second A tile's row offset, and whether a tile has it (see Shape)
    const int b_off = GATE_UP ? a_rows_per_expert / 2 : 2 * BM;
    auto has_second = [&](const TileInfo& ti) {
        return GATE_UP || ti.m * S::M_ROWS + 2 * BM < a_rows_per_expert;
    };

    if (warp == 0) {
        // ---------------- producer: this CTA's weight rows and token half. Lane 0
        // waits for each stage and issues the weight loads and (copy path) the
        // token boxes; with GATHER every lane l with 4l < half also gathers rows
        // 4l..4l+3 of x with one tile::gather4.
        const uint64_t pol_w = tc::policy_evict_first();
        const uint64_t pol_x = tc::policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        uint32_t parity[S::STAGES] = {};
        bool issued[S::STAGES] = {};
        bool ok = true;
        if (!GATHER && lane != 0) ok = false;  // the copy path issues from lane 0 alone
        for (int t = pair; t < total && ok; t += n_pairs) {
            const TileInfo ti = decode_tile<NM>(c, E, m_tiles, t);
            const int half = ti.n / 2;
            const int a_row = ti.e * a_rows_per_expert + ti.m * S::M_ROWS + rank * BM;
            const int b_row = ti.row0 + rank * half;
            const bool two = has_second(ti);
            const uint32_t pair_bytes = 2u * ((two ? 2 : 1) * A_BYTES + half * BK * 2);
            int tok[4] = {0, 0, 0, 0};
            if (GATHER) {
                // rows past the tile's end repeat its first row (in range, ignored)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = b_row + 4 * lane + i;
                    tok[i] = token_of_row[r < ti.row0 + ti.len ? r : ti.row0];
                }
            }
            for (int kb = 0; kb < KB; ++kb) {
                if (lane == 0 && !tc::mbar_wait(&c.empty[stage], phase ^ 1u, abort_flag)) {
                    raise_timeout(c, status);
                    ok = false;
                }
                if (GATHER) ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                const uint32_t full_leader = tc::map_to_cta(tc::smem_u32(&c.full[stage]), 0);
                uint8_t* s = smem + stage * S::STAGE_BYTES;
                uint8_t* sb = s + S::A_TILES * A_BYTES;
                if (lane == 0) {
                    if (leader) tc::mbar_arrive_expect_tx(&c.full[stage], pair_bytes);
                    if (packed_a) {
                        // 128 x 64 blocks stored contiguously: block (row / 128, kb)
                        tc::tma_load_2d_pair(s, &tmA, full_leader, 0, ((a_row / BM) * KB + kb) * BM,
                                             pol_w);
                        if (two)
                            tc::tma_load_2d_pair(s + A_BYTES, &tmA, full_leader, 0,
                                                 (((a_row + b_off) / BM) * KB + kb) * BM, pol_w);
                    } else {
                        tc::tma_load_2d_pair(s, &tmA, full_leader, kb * BK, a_row, pol_w);
                        if (two)
                            tc::tma_load_2d_pair(s + A_BYTES, &tmA, full_leader, kb * BK,
                                                 a_row + b_off, pol_w);
                    }
                    if (!GATHER)
                        load_token_rows(sb, tmB, full_leader, kb * BK, b_row, half, pol_x);
                    issued[stage] = true;
                    parity[stage] = phase;
                }
                if (GATHER) {
                    __syncwarp();
                    if (4 * lane < half)
                        tc::tma_gather4_pair(sb + lane * (4 * BK * 2), &tmB.m[0], full_leader,
                                             kb * BK, tok[0], tok[1], tok[2], tok[3], pol_x);
                }
                if (++stage == S::STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (lane == 0) {
            // drain: this CTA's copies have landed (the even CTA's full barrier saw
            // every byte of both CTAs when its last phase completed)
            const int zero = 0;
            for (int s = 0; s < S::STAGES; ++s)
                if (issued[s] && !tc::mbar_wait(leader ? &c.full[s] : &c.empty[s], parity[s], &zero))
                    atomicExch(status, MOE_ERR_TIMEOUT);
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---------------- MMA issuer (even CTA), M = 256 across the pair
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int it = 0;
            for (int t = pair; t < total && ok; t += n_pairs, ++it) {
                const TileInfo ti = decode_tile<NM>(c, E, m_tiles, t);
                const int acc = it % S::ACC_STAGES;
                const uint32_t acc_phase = (uint32_t)(it / S::ACC_STAGES) & 1u;
                if (!tc::mbar_wait(&c.acc_empty[acc], acc_phase ^ 1u, abort_flag)) {
                    raise_timeout(c, status);
                    break;
                }
                tc::fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * S::ACC_COLS;
                const uint32_t idesc = tc::idesc_bf16_f32(2 * BM, ti.n);
                const bool two = has_second(ti);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!tc::mbar_wait(&c.full[stage], phase, abort_flag)) {
                        raise_timeout(c, status);
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint32_t a_addr = tc::smem_u32(smem + stage * S::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + S::A_TILES * A_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / UK; ++k) {
                        const uint64_t bdesc = tc::desc_sw128(b_addr + k * UK * 2);
                        const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
                        tc::mma_bf16_pair(d_tmem, tc::desc_sw128(a_addr + k * UK * 2), bdesc,
                                          idesc, accum);
                        if (two)
                            tc::mma_bf16_pair(d_tmem + S::U_OFF,
                                              tc::desc_sw128(a_addr + A_BYTES + k * UK * 2), bdesc,
                                              idesc, accum);
                    }
                    tc::mma_commit_pair(&c.empty[stage], 0x3);
                    if (++stage == S::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) tc::mma_commit_pair(&c.acc_full[acc], 0x3);
            }
            tc::mma_commit_pair(&c.drain, 0x1);
            const int zero = 0;
            if (!tc::mbar_wait(&c.drain, 0, &zero)) atomicExch(status, MOE_ERR_TIMEOUT);
        }
    } else if (warp >= 2 && warp < 2 + 4 * EPI_GROUPS) {
        // ---------------- epilogue: this CTA's 128 weight rows (TMEM lanes). Group
        // g takes the 32-token chunks g, g + EPI_GROUPS, ...: each of its warps
        // writes its 32 rows x 32 tokens as bf16 into the group's shared [32
        // tokens][128 rows] tile, and after a named barrier the group stores the
        // tile as 256-byte row segments of the output with 16-byte vectors.
        // Named barriers: 1 + g within a group, 1 + EPI_GROUPS across all groups.
        const int quad = warp & 3;
        const int grp = (warp - 2) >> 2;
        const int et = threadIdx.x - 64 - 128 * grp;  // 0..127 within the group
        const int bar_grp = 1 + grp, bar_all = 1 + EPI_GROUPS;
        uint16_t* tile = epi + grp * (EPI_N * BM);
        uint16_t* o16 = reinterpret_cast<uint16_t*>(out);
        const bool arriver = (warp == 2 && lane == 0);
        int it = 0;
        for (int t = pair; t < total; t += n_pairs, ++it) {
            const TileInfo ti = decode_tile<NM>(c, E, m_tiles, t);
            const int acc = it % S::ACC_STAGES;
            const uint32_t acc_phase = (uint32_t)(it / S::ACC_STAGES) & 1u;
            const bool waited = tc::mbar_wait(&c.acc_full[acc], acc_phase, abort_flag);
            if (tc::bar_any(bar_all, 128 * EPI_GROUPS, !waited)) {  // all warps leave together
                raise_timeout(c, status);
                break;
            }
            tc::fence_after_sync();
            const uint32_t tbase = tmem_base + acc * S::ACC_COLS + ((uint32_t)(quad * 32) << 16);
            const int col0 = ti.m * S::M_ROWS + rank * BM;
            const int parts = GATE_UP ? 1 : (has_second(ti) ? 2 : 1);
            // gate_up: h = SiLU(g) u from the two accumulators; down: the two
            // accumulators are two 256-column ranges of y (part 1: 256 columns on)
            for (int cc = grp; cc < parts * ((ti.n + EPI_N - 1) / EPI_N); cc += EPI_GROUPS) {
                const int nch = (ti.n + EPI_N - 1) / EPI_N;
                const int part = cc / nch, c0 = (cc - part * nch) * EPI_N;
                uint32_t g[32];
                tc::tmem_ld32(tbase + part * S::U_OFF + c0, g);
                if constexpr (GATE_UP) {
                    uint32_t u[32];
                    tc::tmem_ld32(tbase + S::U_OFF + c0, u);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float gv = __uint_as_float(g[j]), uv = __uint_as_float(u[j]);
                        tile[j * BM + quad * 32 + lane] = float_to_bf16_bits(silu_mul(gv, uv));
                    }
                } else {
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        tile[j * BM + quad * 32 + lane] = float_to_bf16_bits(__uint_as_float(g[j]));
                }
                tc::bar_sync(bar_grp, 128);  // the group's tile is written
#pragma unroll
                for (int q = 0; q < EPI_N * BM / 8 / 128; ++q) {
                    const int id = et + 128 * q;
                    const int n = id / (BM / 8), ch = id % (BM / 8);
                    if (c0 + n < ti.len)
                        *reinterpret_cast<uint4*>(o16 + (size_t)(ti.row0 + c0 + n) * out_ld + col0 +
                                                  part * b_off + ch * 8) =
                            *reinterpret_cast<const uint4*>(tile + n * BM + ch * 8);
                }
                tc::bar_sync(bar_grp, 128);  // the group's tile is read
            }
            // every warp's TMEM reads are complete before the accumulator is handed back
            tc::fence_before_sync();
            tc::bar_sync(bar_all, 128 * EPI_GROUPS);
            if (arriver)
                tc::mbar_arrive_cluster(tc::map_to_cta(tc::smem_u32(&c.acc_empty[acc]), 0));
        }
    }

    // Neither CTA leaves while the other may still signal its barriers or read
    // its shared memory.
    tc::fence_before_sync();
    tc::cluster_sync();
    if (warp == 1) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc_pair(tmem_base, 512);
    }
}

// ======================================================================
// Quantised expert weights: FP8 (e4m3 codes, fp32 per-output-row scale) and
// FP4 (E2M1 codes, an E8M0 scale per 32 codes of a row). The MMA stays
// kind::f16 (bf16 x bf16, fp32 accumulate) on weights widened exactly to bf16
// on chip. Per K block, warp 0 TMA-loads this CTA's raw weight tile(s) (128
// rows x 64 codes: 64 bytes of e4m3, 64-byte swizzle; 32 bytes of E2M1,
// 32-byte swizzle) into a "raw" ring on the CTA's own barrier; warp 15 loads
// its half of the token rows (bf16, 128-byte swizzle) into a token ring
// completing on the even CTA's barrier. Converter warps, in two groups of
// four that take K blocks round-robin (so the latencies of consecutive blocks
// overlap), widen the weights into an "op" stage of tensor memory, release
// the raw stage and arrive on the even CTA's operand barrier; the pair MMA
// reads A from TMEM (tcgen05.mma [d], [a_tmem], b_desc) and B from the token
// stage and releases both. The raw stages live only from load to conversion,
// so their ring keeps the weight stream deep.
//
// FP8: the per-output-row fp32 scale multiplies the finished dot product in
// the epilogue (before SiLU for gate_up, before the bf16 store for down):
// sum_c x_c q_c s_row = s_row sum_c x_c q_c. Every e4m3 value is a bf16 value,
// so the widening loses nothing. FP4: the block scale is folded into the
// widening (every E2M1 value times a power of two is a bf16 value, below the
// bf16 overflow), so the epilogue applies no scale.
//
// A goes straight into TMEM (tcgen05.st, one thread per A row): writing it
// as a shared-memory tile instead ran the tensor pipe at ~51% against ~57%,
// the tile's writes and the MMA's reads competing with the raw reads. TMEM
// then holds the accumulators and the op stages, which caps a token tile at
// NM = 192 rows. A pair tile takes two A tiles of 256 weight rows (128 per
// CTA) against the same token rows -- gate_up: the gate rows m*256.. and the
// up rows F + m*256..; down: the rows m*512.. and m*512 + 256.. -- so one
// token stage feeds two MMAs per K step: two accumulators (2 x 192 columns)
// + 2 op stages of 64 (both tiles' K block). (down with one A tile and a
// double-buffered accumulator, each token stage feeding one MMA, ran 2-4%
// slower for FP8 and 13% for FP4; smaller op stages, twice as many, 8-10%
// slower: more barrier and signal work for less conversion each.) Where d is
// an odd multiple of 256, down's last pair tile has its first A tile only.
//
// Once the experts average 128+ grouped rows, down runs the transposed split
// (TT): one A tile of 256 rows against two token sub-tiles of up to SUB = 192
// rows each (a pair tile of up to 384 token rows; each CTA's token stage holds
// its half of both sub-tiles in two regions), two accumulators of 192 columns
// and 4 op stages of 32. Each K block of weights is then widened once for up
// to 384 tokens instead of 192: at the Hy3 FP8 shape (T=8192, ~341 rows per
// expert) down ran 12% faster (the layer 1.5% under the power cap).

constexpr int THREADS_Q = 512;        // warps 6-14 converters, warp 15 token producer
constexpr int MAX_RAW_STAGES = 16, MAX_B_STAGES = 4, MAX_OP_STAGES = 4;  // QCtrl's arrays
template <bool GATE_UP, bool FP4, bool TT = false>
struct QShape {
    static constexpr int A_TILES = TT ? 1 : 2;                     // A tiles per pair tile
    static constexpr int RAW_ROW = FP4 ? 32 : 64;                  // bytes of 64 codes
    static constexpr int RAW_TILE = BM * RAW_ROW;                  // 128 rows
    static constexpr int RAW_STAGE = A_TILES * RAW_TILE;
    static constexpr int SUB = 192;                                // token rows per accumulator
    static constexpr int NM = TT ? 2 * SUB : SUB;                  // token rows per pair tile
    static constexpr int REGION = (SUB / 2) * BK * 2;              // a CTA's half of SUB rows
    static constexpr int BH = (TT ? 2 : 1) * REGION;               // a CTA's token stage (bytes)
    static constexpr int RAW_STAGES = FP4 ? 16 : (TT ? 12 : 8);
    static constexpr int B_STAGES = 4;
    static constexpr int OP_STAGES = TT ? 4 : 2;
    // converter warps: GROUPS groups of four (one per TMEM lane quarter) take
    // K blocks round-robin
    static constexpr int GROUPS = 2;
    static constexpr int GROUP_WARPS = 4;
    static constexpr int CONV_THREADS = GROUP_WARPS * 32;
    // FP4 scale chunks (8 bytes of a row: 4 K blocks), per converter group
    static constexpr int SC_STAGES = 4;
    static constexpr int SC_BYTES = FP4 ? GROUPS * SC_STAGES * A_TILES * BM * 8 : 0;
    static constexpr int RING_BYTES = RAW_STAGES * RAW_STAGE + B_STAGES * BH + SC_BYTES;
    static constexpr int ACC_STAGES = 1;
    // TMEM columns: the two accumulators, then the op stages
    static constexpr int U_OFF = SUB;                              // the second accumulator
    static constexpr int ACC_COLS = 2 * SUB;
    static constexpr int A_COL = ACC_STAGES * ACC_COLS;
    static constexpr int A_TILE_COLS = BK / 2;                     // one tile's K block: two bf16 a column
    static constexpr int A_STAGE_COLS = A_TILES * A_TILE_COLS;     // 64
    // weight rows (gate_up: gate rows; the up rows follow F on) per m (per expert)
    static constexpr int M_ROWS = GATE_UP ? 2 * BM : (TT ? 2 * BM : 4 * BM);
    static constexpr int EPI_BYTES = EPI_N * BM * 2;  // [32 tokens][128 rows] bf16 staging
};

constexpr int CONV_WARPS = 9;                          // warps 6..14 (warp 14 idles)
constexpr int TOKEN_WARP = 6 + CONV_WARPS;
template <bool G, bool FP4, bool TT = false>
constexpr bool shape_ok() {
    using S = QShape<G, FP4, TT>;
    return S::RAW_STAGES % S::GROUPS == 0 && S::OP_STAGES % S::GROUPS == 0 &&
           S::GROUPS * S::GROUP_WARPS <= CONV_WARPS && S::GROUP_WARPS == 4 &&
           S::RAW_STAGES <= MAX_RAW_STAGES && S::B_STAGES <= MAX_B_STAGES &&
           S::OP_STAGES <= MAX_OP_STAGES && S::A_COL + S::OP_STAGES * S::A_STAGE_COLS <= 512 &&
           S::BH % 1024 == 0 && S::REGION % 1024 == 0 && S::RAW_TILE % 1024 == 0;
}
// Each group owns whole raw stages and op stages (both ring lengths are
// multiples of GROUPS), and a group's previous wait on a stage proves that its
// last reader finished (parity waits cannot see a stale phase); every stage
// index stays inside QCtrl's barrier arrays.
static_assert(shape_ok<true, false>() && shape_ok<false, false>() && shape_ok<true, true>() &&
                  shape_ok<false, true>() && shape_ok<false, false, true>(),
              "quantised pair GEMM shape");
static_assert(THREADS_Q == 32 * (TOKEN_WARP + 1), "warp roles cover the block");

struct QCtrl {
    uint64_t raw_full[MAX_RAW_STAGES];   // each CTA: its raw weight tile(s) landed
    uint64_t raw_empty[MAX_RAW_STAGES];  // each CTA: the converters are done with the raw stage
    uint64_t b_full[MAX_B_STAGES];       // even CTA: token bytes of both CTAs landed
    uint64_t b_empty[MAX_B_STAGES];      // both CTAs: the pair MMAs finished with the token stage
    uint64_t op_full[MAX_OP_STAGES];     // even CTA: both CTAs' groups filled the op stage
    uint64_t op_empty[MAX_OP_STAGES];    // both CTAs: the pair MMAs finished with the op stage
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    alignas(16) uint32_t sig[MAX_OP_STAGES][4];  // even CTA: landing slots of the odd CTA's signals
    alignas(16) uint32_t sig_src[4];             // odd CTA: the signals' (unread) source bytes
    uint32_t tmem_base;
    int abort;
    int total;
    int off[MAX_E + 1];
    int tile_start[MAX_E + 1];
};

template <bool GATE_UP, bool FP4, bool TT = false>
constexpr int q_smem_bytes() {
    return QShape<GATE_UP, FP4, TT>::RING_BYTES + QShape<GATE_UP, FP4, TT>::EPI_BYTES + 1024 +
           (int)sizeof(QCtrl);
}
static_assert(q_smem_bytes<true, false>() <= 232448 && q_smem_bytes<false, false>() <= 232448 &&
                  q_smem_bytes<true, true>() <= 232448 && q_smem_bytes<false, true>() <= 232448 &&
                  q_smem_bytes<false, false, true>() <= 232448,
              "fits in 227 KB");

// A bf16x2 multiply kept in program order with respect to the waits around it
// (volatile), so that a conversion stays ahead of the wait that follows it.
__device__ __forceinline__ uint32_t mul_bf16x2_here(uint32_t a, uint32_t b) {
    uint32_t d;
    asm volatile("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Four e4m3 codes (one 32-bit word, code i in byte i) -> four bf16 in two
// bf16x2 words (codes 0, 1 in lo; 2, 3 in hi; the even code in the low half),
// exactly, on the integer and FMA pipes instead of the conversion pipe (whose
// ~16 results per clock per SM bounded the converters): a byte permute puts
// each code in the high byte of a 16-bit half, its seven exponent+mantissa
// bits move down to bf16 bits 4..10 and its sign stays at bit 15. That bf16
// reads as the code's value times 2^-120 (exponent field e = the code's, its
// three mantissa bits on top of bf16's seven; a subnormal code, e = 0, is a
// bf16 subnormal of the same scaled value), and one bf16x2 multiply by 2^120
// (bf16 0x7B80: a power of two, exact, subnormal inputs included) restores
// it. Signed zeros carry over. NaN codes (S.1111.111) give a finite value:
// NaN weights are unspecified.
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
    constexpr uint32_t kTwoPow120 = 0x7B807B80u;  // bf16x2 (2^120, 2^120)
    lo = mul_bf16x2_here(e4m3_pair_scaled_bits(__byte_perm(w, 0u, 0x1404)), kTwoPow120);
    hi = mul_bf16x2_here(e4m3_pair_scaled_bits(__byte_perm(w, 0u, 0x3424)), kTwoPow120);
}

// 32 E2M1 codes (16 bytes: code 2i in the low nibble of byte i) of one scale
// block, whose E8M0 byte is b -> 16 bf16x2 words (byte i -> word i, the even
// code in the low half), exactly: each byte becomes a bf16 pair worth value *
// 2^-126 (e2m1_pair_scaled_bits); one bf16x2 multiply by 2^(b-1) -- a normal
// bf16 for b <= 128 -- gives value * 2^(b-127); for b > 128 it is two
// multiplies, by 2^126 and by 2^(b-127). Products of magnitude >= 2^128
// (b >= 253) overflow, as the value itself does in bf16.
__device__ __forceinline__ void e2m1x32_to_bf16(const uint32_t* w, uint32_t b, uint32_t* o) {
    const bool one = b <= 128u;
    const uint32_t f1 = one ? ((b + 126u) << 7) : 0x7E80u;  // 2^(b-1) or 2^126
    const uint32_t f1x2 = f1 | (f1 << 16);
    const uint32_t f2x2 = (b << 7) | (b << 23);              // 2^(b-127), used if b > 128
#pragma unroll
    for (int j4 = 0; j4 < 4; ++j4)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t v = e2m1_pair_scaled_bits(__byte_perm(w[j4], 0u, 0x4440u | j));
            v = mul_bf16x2_here(v, f1x2);
            if (!one) v = mul_bf16x2_here(v, f2x2);
            o[4 * j4 + j] = v;
        }
}

// One thread's widened A row for every A tile of an op stage (tiles in
// adjacent column ranges) into its TMEM lane: one tcgen05.st.
template <int A_TILES>
__device__ __forceinline__ void tc_store_row(uint32_t taddr, const uint32_t (&o)[A_TILES * 32]) {
    if constexpr (A_TILES == 2)
        tc::tmem_st64(taddr, o);
    else
        tc::tmem_st32(taddr, o);
}

// tmA: FP8 e4m3 weights [E * a_rows_per_expert, K] bytes, box 64 x 128,
// 64-byte swizzle; FP4 E2M1 codes [E * a_rows_per_expert, K / 2] bytes, box 32
// x 128, 32-byte swizzle. tmB: token rows [R, K] bf16, boxes of 16..128 rows x
// 64. scales_v: FP8 fp32 row scales [E * a_rows_per_expert]; FP4 E8M0 block
// scales [E * a_rows_per_expert, K / 32] bytes.
template <bool GATE_UP, bool FP4, bool TT>
__global__ void __launch_bounds__(THREADS_Q, 1)
grouped_gemm_pair_fp8_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ TokenMaps tmB,
                             const int* __restrict__ offsets, const void* __restrict__ scales_v,
                             int E, int K, int a_rows_per_expert, int m_tiles,
                             __nv_bfloat16* __restrict__ out, int out_ld,
                             int* __restrict__ status) {
    pdl_launch_and_wait();
    using S = QShape<GATE_UP, FP4, TT>;
    static_assert(!(TT && (FP4 || GATE_UP)), "two token sub-tiles: FP8 down only");
    const float* __restrict__ scales = static_cast<const float*>(scales_v);
    const uint8_t* __restrict__ scales8 = static_cast<const uint8_t*>(scales_v);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* b_ring = smem;  // 1024-aligned stages
    uint8_t* raw_ring = b_ring + S::B_STAGES * S::BH;
    uint8_t* sc_ring = raw_ring + S::RAW_STAGES * S::RAW_STAGE;  // FP4 only
    uint16_t* epi = reinterpret_cast<uint16_t*>(smem + S::RING_BYTES);
    QCtrl& c = *reinterpret_cast<QCtrl*>(smem + S::RING_BYTES + S::EPI_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)(tc::cluster_ctarank() & 1u);
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    const int KB = K / BK;

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
                cnt = ((n_e + S::NM - 1) / S::NM) * m_tiles;
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
            for (int m = 0; m < 4; ++m) tc::prefetch_tensormap(&tmB.m[m]);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            for (int s = 0; s < S::RAW_STAGES; ++s) {
                tc::mbar_init(&c.raw_full[s], 1);
                tc::mbar_init(&c.raw_empty[s], 1);
            }
            for (int s = 0; s < S::B_STAGES; ++s) {
                tc::mbar_init(&c.b_full[s], 1);
                tc::mbar_init(&c.b_empty[s], 1);
            }
            for (int s = 0; s < S::OP_STAGES; ++s) {
                tc::mbar_init(&c.op_full[s], 1);
                tc::mbar_init(&c.op_empty[s], 1);
            }
            for (int a = 0; a < S::ACC_STAGES; ++a) {
                tc::mbar_init(&c.acc_full[a], 1);
                tc::mbar_init(&c.acc_empty[a], 2);
            }
            tc::mbar_init(&c.drain, 1);
            tc::fence_mbar_init();
        }
        __syncwarp();
        tc::tmem_alloc_pair(&c.tmem_base, 512);
        tc::tmem_relinquish_pair();
    }
    tc::fence_before_sync();
    tc::cluster_sync();
    tc::fence_after_sync();
    const uint32_t tmem_base = c.tmem_base;
    const int total = c.total;
    const volatile int* abort_flag = &c.abort;
    // A pair tile's weight rows: this CTA's rows of the first A tile, the offset
    // of the second's (gate_up: the up rows; down: 256 rows on), and whether
    // the second exists (not in down's last tile where d is an odd multiple of
    // 256).
    // With TT (down) a pair tile has one A tile of 256 rows against up to 2 SUB
    // token rows, SUB per accumulator.
    const int b_off = GATE_UP ? a_rows_per_expert / 2 : 2 * BM;
    auto first_row = [&](const TileInfo& ti) {
        return ti.e * a_rows_per_expert + ti.m * S::M_ROWS + rank * BM;
    };
    auto has_second = [&](const TileInfo& ti) {
        return !TT && (GATE_UP || ti.m * S::M_ROWS + 2 * BM < a_rows_per_expert);
    };
    // the tile's token rows per accumulator: n0 (at most SUB), then n1
    auto sub_n0 = [&](const TileInfo& ti) { return TT ? min(ti.n, S::SUB) : ti.n; };

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- raw weight producer (this CTA's rows, own barrier)
            const uint64_t pol_w = tc::policy_evict_first();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t parity[S::RAW_STAGES] = {};
            bool issued[S::RAW_STAGES] = {};
            bool ok = true;
            for (int t = pair; t < total && ok; t += n_pairs) {
                const TileInfo ti = decode_tile<S::NM>(c, E, m_tiles, t);
                const int a_row = first_row(ti);
                const bool two = has_second(ti);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!tc::mbar_wait(&c.raw_empty[stage], phase ^ 1u, abort_flag)) {
                        raise_timeout(c, status);
                        ok = false;
                        break;
                    }
                    uint8_t* st = raw_ring + stage * S::RAW_STAGE;
                    tc::mbar_arrive_expect_tx(&c.raw_full[stage], two ? S::RAW_STAGE : S::RAW_TILE);
                    const int kx = kb * S::RAW_ROW;  // byte column of the K block's 64 codes
                    tc::tma_load_2d_hint(st, &tmA, &c.raw_full[stage], kx, a_row, pol_w);
                    if (two)  // (without it the stage's second tile holds stale codes, unused)
                        tc::tma_load_2d_hint(st + S::RAW_TILE, &tmA, &c.raw_full[stage], kx,
                                             a_row + b_off, pol_w);
                    issued[stage] = true;
                    parity[stage] = phase;
                    if (++stage == S::RAW_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            const int zero = 0;
            for (int s = 0; s < S::RAW_STAGES; ++s)
                if (issued[s] && !tc::mbar_wait(&c.raw_full[s], parity[s], &zero))
                    atomicExch(status, MOE_ERR_TIMEOUT);
        }
    } else if (warp == TOKEN_WARP) {
        if (lane == 0) {
            // ---------------- token-half producer; completes on the even CTA's b_full
            const uint64_t pol_x = tc::policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t parity[S::B_STAGES] = {};
            bool issued[S::B_STAGES] = {};
            bool ok = true;
            for (int t = pair; t < total && ok; t += n_pairs) {
                const TileInfo ti = decode_tile<S::NM>(c, E, m_tiles, t);
                // each CTA holds half of each accumulator's rows: n0 / 2 in the
                // stage's first region, n1 / 2 in the second (TT)
                const int n0 = sub_n0(ti), n1 = ti.n - n0;
                const uint32_t pair_bytes = (uint32_t)ti.n * (BK * 2);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!tc::mbar_wait(&c.b_empty[stage], phase ^ 1u, abort_flag)) {
                        raise_timeout(c, status);
                        ok = false;
                        break;
                    }
                    const uint32_t full_leader = tc::map_to_cta(tc::smem_u32(&c.b_full[stage]), 0);
                    if (leader) tc::mbar_arrive_expect_tx(&c.b_full[stage], pair_bytes);
                    uint8_t* st = b_ring + stage * S::BH;
                    load_token_rows(st, tmB, full_leader, kb * BK, ti.row0 + rank * (n0 / 2), n0 / 2,
                                    pol_x);
                    if (TT && n1 > 0)
                        load_token_rows(st + S::REGION, tmB, full_leader, kb * BK,
                                        ti.row0 + n0 + rank * (n1 / 2), n1 / 2, pol_x);
                    issued[stage] = true;
                    parity[stage] = phase;
                    if (++stage == S::B_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            const int zero = 0;
            for (int s = 0; s < S::B_STAGES; ++s)
                if (issued[s] && !tc::mbar_wait(leader ? &c.b_full[s] : &c.b_empty[s], parity[s], &zero))
                    atomicExch(status, MOE_ERR_TIMEOUT);
        }
    } else if (warp >= 6 && warp < 6 + CONV_WARPS) {
        // ---------------- converters: raw codes -> bf16 A rows in a TMEM op stage.
        // Each thread widens one A row of this CTA -- row r = 32 (warp % 4) +
        // lane, the TMEM lane its warp may write -- for every A tile of the K
        // block: the 64 codes of its raw row (the swizzle puts the eight rows of
        // a quarter-warp's 16-byte loads on distinct banks: chunk c of row r
        // sits at chunk c ^ ((r / 2) % 4) for e4m3, c ^ ((r / 4) % 2) for E2M1)
        // into 32 TMEM columns (two bf16 a column, the even K index in the low
        // half). A group converts the K blocks j = group, group + GROUPS, ...
        // (warp 14 idles). The widening runs before the wait for the op stage.
        //
        // The group's threads complete their stores (tcgen05.wait::st, then the
        // tcgen05 fence) and meet at a named barrier; then one thread releases
        // the raw stage and signals the even CTA's op_full: in the even CTA a
        // local arrive that expects 16 bytes, in the odd CTA a 16-byte
        // shared-to-shared bulk copy into the even CTA that completes on that
        // barrier. A remote mbarrier arrive with cluster-scope release, the
        // other way to signal across the pair, stalled its warp ~1.5k cycles
        // per K block on B200 -- longer than the widening itself. The group
        // agrees on its bounded waits (bar.red.or) and leaves together; the
        // MMA's bounded wait on op_full then gives up.
        const int group = (warp - 6) / S::GROUP_WARPS;
        const int ct = threadIdx.x - 192 - group * S::CONV_THREADS;  // 0..CONV_THREADS-1
        const int r = 32 * (warp & 3) + lane;
        const uint32_t rsw = FP4 ? (uint32_t)((r >> 2) & 1) : (uint32_t)((r >> 1) & 3);
        const uint32_t raw0 = tc::smem_u32(raw_ring) + r * S::RAW_ROW;
        const uint32_t a_lane = tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) + S::A_COL;
        // this CTA's K blocks in order: j = tile_iteration * KB + kb
        int n_my_tiles = 0;
        for (int t = pair; t < total; t += n_pairs) ++n_my_tiles;
        const long n_blocks = (long)n_my_tiles * KB;
        // FP4: the scale bytes of this thread's rows come as 8-byte chunks, one
        // per 4 K blocks (the 32-code blocks 8 q .. 8 q + 7 of the row): chunk
        // G = j / 4 of the CTA's block sequence, which the group uses for two of
        // its blocks. Each thread copies its own chunks into a ring of SC_STAGES
        // shared-memory slots with cp.async, SC_STAGES - 1 chunks ahead (loads
        // into registers one or two blocks ahead left the converters waiting
        // on them), and reads chunk G when the group reaches it.
        const long n_chunks = n_blocks / 4;  // K blocks per tile: a multiple of 4
        const long sblocks = K / 32;
        const uint32_t sc_slot0 =
            tc::smem_u32(sc_ring) + (uint32_t)(group * S::SC_STAGES * S::A_TILES * BM * 8 + r * 8);
        long fetch_it = -1, fetch_row = 0;  // the tile of the last fetch, its row
        bool fetch_two = true;               // and whether it has a second A tile
        auto fetch_chunk = [&](long G) {  // one copy group per chunk, empty past the end
            if (G < n_chunks) {
                const long it = G / (KB / 4);
                const int q = (int)(G - it * (KB / 4));
                if (it != fetch_it) {  // a new tile: one lookup per tile, not per chunk
                    const TileInfo ti = decode_tile<S::NM>(c, E, m_tiles, pair + (int)it * n_pairs);
                    fetch_row = (long)first_row(ti) + r;
                    fetch_two = has_second(ti);
                    fetch_it = it;
                }
                const long row = fetch_row;
                const uint32_t dst = sc_slot0 + (uint32_t)((G % S::SC_STAGES) * S::A_TILES * BM * 8);
#pragma unroll
                for (int a = 0; a < S::A_TILES; ++a)
                    if (a == 0 || fetch_two)  // no scales past the expert's rows
                        tc::cp_async8(dst + a * BM * 8, scales8 + (row + a * b_off) * sblocks + 8 * q);
            }
            tc::cp_async_commit();
        };
        uint2 sc_cur[S::A_TILES] = {};
        long cur_chunk = -1;
        const long j0 = group < S::GROUPS ? group : n_blocks;
        if (FP4 && j0 < n_blocks)
            for (int g = 0; g < S::SC_STAGES - 1; ++g) fetch_chunk((j0 >> 2) + g);
        for (long jb = j0; jb < n_blocks; jb += S::GROUPS) {
            const int rs = (int)(jb % S::RAW_STAGES), os = (int)(jb % S::OP_STAGES);
            const uint32_t rph = (uint32_t)(jb / S::RAW_STAGES) & 1u;
            const uint32_t oph = (uint32_t)(jb / S::OP_STAGES) & 1u;
            uint32_t sc[S::A_TILES] = {};  // FP4: this block's two scale bytes per A tile
            if constexpr (FP4) {
                if ((jb >> 2) != cur_chunk) {
                    cur_chunk = jb >> 2;
                    // the slot of chunk G + SC_STAGES - 1 held chunk G - 1, read already
                    fetch_chunk(cur_chunk + S::SC_STAGES - 1);
                    tc::cp_async_wait_pending<S::SC_STAGES - 1>();  // chunk G has landed
                    const uint32_t src =
                        sc_slot0 + (uint32_t)((cur_chunk % S::SC_STAGES) * S::A_TILES * BM * 8);
#pragma unroll
                    for (int a = 0; a < S::A_TILES; ++a)
                        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                                     : "=r"(sc_cur[a].x), "=r"(sc_cur[a].y)
                                     : "r"(src + a * BM * 8));
                }
                const int kq = (int)(jb & 3);  // the block's place in its chunk
#pragma unroll
                for (int a = 0; a < S::A_TILES; ++a)
                    sc[a] = ((kq < 2 ? sc_cur[a].x : sc_cur[a].y) >> (16 * (kq & 1))) & 0xFFFFu;
            }
            const bool rok = tc::mbar_wait(&c.raw_full[rs], rph, abort_flag);
            if (tc::bar_any(2 + group, S::CONV_THREADS, !rok)) {  // the group leaves together
                raise_timeout(c, status);
                break;
            }
            const uint32_t raw = raw0 + rs * S::RAW_STAGE;
            constexpr int CHUNKS = S::RAW_ROW / 16;
            uint32_t w[S::A_TILES][4 * CHUNKS];
#pragma unroll
            for (int a = 0; a < S::A_TILES; ++a)
#pragma unroll
                for (int ch = 0; ch < CHUNKS; ++ch)
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(w[a][4 * ch]), "=r"(w[a][4 * ch + 1]),
                                   "=r"(w[a][4 * ch + 2]), "=r"(w[a][4 * ch + 3])
                                 : "r"(raw + a * S::RAW_TILE + ((ch ^ rsw) << 4)));
            uint32_t o[S::A_TILES * 32];  // tile a in o[32 a ..], its TMEM columns in order
#pragma unroll
            for (int a = 0; a < S::A_TILES; ++a) {
                if constexpr (FP4) {
#pragma unroll
                    for (int ch = 0; ch < 2; ++ch)
                        e2m1x32_to_bf16(&w[a][4 * ch], (sc[a] >> (8 * ch)) & 0xFFu,
                                        &o[32 * a + 16 * ch]);
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        e4m3x4_to_bf16x4(w[a][j], o[32 * a + 2 * j], o[32 * a + 2 * j + 1]);
                }
            }
            const bool ook = tc::mbar_wait(&c.op_empty[os], oph ^ 1u, abort_flag);
            if (tc::bar_any(2 + group, S::CONV_THREADS, !ook)) {
                raise_timeout(c, status);
                break;
            }
            tc::fence_after_sync();  // the MMAs that read this op stage are complete
            tc_store_row<S::A_TILES>(a_lane + os * S::A_STAGE_COLS, o);
            tc::tmem_st_wait();
            tc::fence_before_sync();
            tc::bar_sync(2 + group, S::CONV_THREADS);
            if (ct == 0) {
                tc::mbar_arrive(&c.raw_empty[rs]);
                if (leader)
                    tc::mbar_arrive_expect_tx(&c.op_full[os], 16);
                else
                    tc::bulk_copy_smem_to_cluster(tc::map_to_cta(tc::smem_u32(&c.sig[os][0]), 0),
                                                  tc::smem_u32(&c.sig_src[0]), 16,
                                                  tc::map_to_cta(tc::smem_u32(&c.op_full[os]), 0));
            }
        }
        if constexpr (FP4) tc::cp_async_wait_pending<0>();  // no copy outlives the loop
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---------------- MMA issuer (even CTA): A from the TMEM op stage, B from the token stage
            int bs = 0, os = 0;
            uint32_t oph = 0, bph = 0;
            bool ok = true;
            int it = 0;
            for (int t = pair; t < total && ok; t += n_pairs, ++it) {
                const TileInfo ti = decode_tile<S::NM>(c, E, m_tiles, t);
                const int acc = it % S::ACC_STAGES;
                const uint32_t acc_phase = (uint32_t)(it / S::ACC_STAGES) & 1u;
                if (!tc::mbar_wait(&c.acc_empty[acc], acc_phase ^ 1u, abort_flag)) {
                    raise_timeout(c, status);
                    break;
                }
                tc::fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * S::ACC_COLS;
                const int n0 = sub_n0(ti), n1 = ti.n - n0;
                const uint32_t idesc = tc::idesc_bf16_f32(2 * BM, n0);
                const uint32_t idesc1 = tc::idesc_bf16_f32(2 * BM, n1 > 0 ? n1 : n0);
                const bool two = has_second(ti);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!tc::mbar_wait(&c.op_full[os], oph, abort_flag) ||
                        !tc::mbar_wait(&c.b_full[bs], bph, abort_flag)) {
                        raise_timeout(c, status);
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint32_t a_tm = tmem_base + S::A_COL + os * S::A_STAGE_COLS;
                    const uint32_t b_addr = tc::smem_u32(b_ring + bs * S::BH);
#pragma unroll
                    for (int k = 0; k < BK / UK; ++k) {  // K = 16 of A is 8 TMEM columns
                        const uint64_t bdesc = tc::desc_sw128(b_addr + k * UK * 2);
                        const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
                        tc::mma_bf16_pair_ta(d_tmem, a_tm + k * (UK / 2), bdesc, idesc, accum);
                        if (TT && n1 > 0)  // the same A against the second region's rows
                            tc::mma_bf16_pair_ta(d_tmem + S::U_OFF, a_tm + k * (UK / 2),
                                                 tc::desc_sw128(b_addr + S::REGION + k * UK * 2),
                                                 idesc1, accum);
                        if (two)  // the second A tile's columns follow the first's
                            tc::mma_bf16_pair_ta(d_tmem + S::U_OFF,
                                                 a_tm + S::A_TILE_COLS + k * (UK / 2), bdesc,
                                                 idesc, accum);
                    }
                    tc::mma_commit_pair(&c.op_empty[os], 0x3);
                    tc::mma_commit_pair(&c.b_empty[bs], 0x3);
                    if (++os == S::OP_STAGES) {
                        os = 0;
                        oph ^= 1u;
                    }
                    if (++bs == S::B_STAGES) {
                        bs = 0;
                        bph ^= 1u;
                    }
                }
                if (ok) tc::mma_commit_pair(&c.acc_full[acc], 0x3);
            }
            tc::mma_commit_pair(&c.drain, 0x1);
            const int zero = 0;
            if (!tc::mbar_wait(&c.drain, 0, &zero)) atomicExch(status, MOE_ERR_TIMEOUT);
        }
    } else if (warp >= 2 && warp <= 5) {
        // ---------------- epilogue (scales applied to the finished dot products)
        const int quad = warp & 3;
        // Per 32-token chunk the four warps write bf16 into the shared [32 tokens]
        // [128 rows] tile and, after a named barrier, store it as 256-byte row
        // segments with 16-byte vectors (as the bf16 kernel's epilogue does).
        const int row_in_tile = quad * 32 + lane;
        const int et = threadIdx.x - 64;  // 0..127
        uint16_t* o16 = reinterpret_cast<uint16_t*>(out);
        const bool arriver = (warp == 2 && lane == 0);
        int it = 0;
        for (int t = pair; t < total; t += n_pairs, ++it) {
            const TileInfo ti = decode_tile<S::NM>(c, E, m_tiles, t);
            const int acc = it % S::ACC_STAGES;
            const uint32_t acc_phase = (uint32_t)(it / S::ACC_STAGES) & 1u;
            const bool waited = tc::mbar_wait(&c.acc_full[acc], acc_phase, abort_flag);
            if (tc::bar_any(1, 128, !waited)) {  // the four warps leave together
                raise_timeout(c, status);
                break;
            }
            tc::fence_after_sync();
            const uint32_t tbase = tmem_base + acc * S::ACC_COLS + ((uint32_t)(quad * 32) << 16);
            const int col0 = ti.m * S::M_ROWS + rank * BM;
            const bool two = has_second(ti);
            const long srow = (long)ti.e * a_rows_per_expert + col0 + row_in_tile;
            // FP8: the row scales multiply the finished dot products; FP4 folded
            // its block scales into the widening
            const float sa = FP4 || TT ? 1.f : __ldg(scales + srow);
            const float sb = (FP4 || TT || !two) ? 1.f : __ldg(scales + srow + b_off);
            if constexpr (TT) {
                // part p: the tile's token rows p SUB.. (accumulator p), 128
                // columns of y each
                const int n0 = sub_n0(ti);
                const int f0 = ti.m * S::M_ROWS + rank * BM;
                const float sr = __ldg(scales + (long)ti.e * a_rows_per_expert + f0 + row_in_tile);
                for (int part = 0; part < (ti.n > n0 ? 2 : 1); ++part) {
                    const int np = part ? ti.n - n0 : n0, rb = part * S::SUB;
                    for (int c0 = 0; c0 < np; c0 += EPI_N) {
                        uint32_t g[32];
                        tc::tmem_ld32(tbase + part * S::U_OFF + c0, g);
                        tc::tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            epi[j * BM + row_in_tile] = float_to_bf16_bits(__uint_as_float(g[j]) * sr);
                        tc::bar_sync(1, 128);  // the tile is written
#pragma unroll
                        for (int q = 0; q < EPI_N * BM / 8 / 128; ++q) {
                            const int id = et + 128 * q;
                            const int n = id / (BM / 8), ch = id % (BM / 8);
                            if (rb + c0 + n < ti.len)
                                *reinterpret_cast<uint4*>(o16 + (size_t)(ti.row0 + rb + c0 + n) * out_ld +
                                                          f0 + ch * 8) =
                                    *reinterpret_cast<const uint4*>(epi + n * BM + ch * 8);
                        }
                        tc::bar_sync(1, 128);  // the tile is read
                    }
                }
            } else
            // gate_up: h = SiLU(g) u from the two accumulators; down: the two
            // accumulators are two 256-column ranges of y (part 1: 256 columns on)
            for (int c0 = 0; c0 < ti.n; c0 += EPI_N) {
                for (int part = 0; part < (GATE_UP ? 1 : (two ? 2 : 1)); ++part) {
                    uint32_t g[32];
                    tc::tmem_ld32(tbase + part * S::U_OFF + c0, g);
                    if constexpr (GATE_UP) {
                        uint32_t u[32];
                        tc::tmem_ld32(tbase + S::U_OFF + c0, u);
                        tc::tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float gv = __uint_as_float(g[j]) * sa;
                            const float uv = __uint_as_float(u[j]) * sb;
                            epi[j * BM + row_in_tile] = float_to_bf16_bits(silu_mul(gv, uv));
                        }
                    } else {
                        tc::tmem_ld_wait();
                        const float sp = part ? sb : sa;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            epi[j * BM + row_in_tile] = float_to_bf16_bits(__uint_as_float(g[j]) * sp);
                    }
                    tc::bar_sync(1, 128);  // the tile is written
                    const int cp = col0 + part * b_off;
#pragma unroll
                    for (int q = 0; q < EPI_N * BM / 8 / 128; ++q) {
                        const int id = et + 128 * q;
                        const int n = id / (BM / 8), ch = id % (BM / 8);
                        if (c0 + n < ti.len)
                            *reinterpret_cast<uint4*>(o16 + (size_t)(ti.row0 + c0 + n) * out_ld + cp +
                                                      ch * 8) =
                                *reinterpret_cast<const uint4*>(epi + n * BM + ch * 8);
                    }
                    tc::bar_sync(1, 128);  // the tile is read
                }
            }
            // every warp's TMEM reads are complete before the accumulator is handed back
            tc::fence_before_sync();
            tc::bar_sync(1, 128);
            if (arriver)
                tc::mbar_arrive_cluster(tc::map_to_cta(tc::smem_u32(&c.acc_empty[acc]), 0));
        }
    }

    tc::fence_before_sync();
    tc::cluster_sync();
    if (warp == 1) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc_pair(tmem_base, 512);
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

// Row-major [rows, cols] bytes (e4m3 codes, or E2M1 code pairs), box of
// box_rows x box_cols bytes with the given swizzle (box_cols at most its span).
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                 uint32_t box_rows, uint32_t box_cols, CUtensorMapSwizzle swizzle) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Expert weights [rows_total, cols] bf16, box 64 x 128; packed: the same bytes as
// [rows_total * cols / 64, 64] (128 x 64 blocks).
bool make_weight_map(CUtensorMap* m, const void* w, uint64_t rows_total, uint64_t cols,
                     bool packed) {
    return packed ? make_map(m, w, rows_total * (cols / BK), BK, BM)
                  : make_map(m, w, rows_total, cols, BM);
}

bool make_token_maps(TokenMaps* tm, const void* base, uint64_t rows, uint64_t cols) {
    for (int lg = 0; lg < 4; ++lg)
        if (!make_map(&tm->m[lg], base, rows, cols, NBOX << lg)) return false;
    return true;
}

int sm_pairs() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return (n > 1 ? n : 148) / 2;
}

// Bytes of the first experts' weights each bf16 pair GEMM pulls into L2 before
// it waits for the previous kernel (0: none).
constexpr long long kGateUpPrefetch = 96ll << 20;
constexpr long long kDownPrefetch = 32ll << 20;

template <bool GATE_UP, bool GATHER, int NM>
cudaError_t launch_nm(const CUtensorMap& a, const TokenMaps& b, const int32_t* offsets, int E,
                      int K, int a_rows_per_expert, int m_tiles, bool packed_a, void* out,
                      int out_ld, int* status, cudaStream_t s, const int32_t* token_of_row,
                      const void* pf, long long pf_bytes) {
    const int smem = smem_bytes<GATE_UP, NM>();
    cudaError_t err = cudaFuncSetAttribute(grouped_gemm_pair_kernel<GATE_UP, GATHER, NM>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * sm_pairs(), 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_pdl
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    err = cudaLaunchKernelEx(&cfg, grouped_gemm_pair_kernel<GATE_UP, GATHER, NM>, a, b, offsets,
                             token_of_row, E, K, a_rows_per_expert, m_tiles, (int)packed_a,
                             static_cast<__nv_bfloat16*>(out), out_ld, status,
                             static_cast<const uint8_t*>(pf), pf_bytes);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

// T <= 64: no expert has more than T rows (a token takes an expert once), so
// the tiles hold at most NM_SMALL token rows (more rows would only take more
// tiles, any NM is correct for any grouping).
template <bool GATE_UP, bool GATHER = false>
cudaError_t launch(int T, const CUtensorMap& a, const TokenMaps& b, const int32_t* offsets, int E,
                   int K, int a_rows_per_expert, int m_tiles, bool packed_a, void* out,
                   int out_ld, int* status, cudaStream_t s,
                   const int32_t* token_of_row = nullptr, const void* w = nullptr,
                   long long w_bytes = 0) {
    // the first experts' weights go to L2 ahead of the first tiles (see the kernel)
    const long long cap = GATE_UP ? kGateUpPrefetch : kDownPrefetch;
    const long long pf_bytes = w ? (w_bytes < cap ? w_bytes : cap) : 0;
    if (T <= NM_SMALL)
        return launch_nm<GATE_UP, GATHER, NM_SMALL>(a, b, offsets, E, K, a_rows_per_expert,
                                                     m_tiles, packed_a, out, out_ld, status, s,
                                                     token_of_row, w, pf_bytes);
    return launch_nm<GATE_UP, GATHER, NMAX>(a, b, offsets, E, K, a_rows_per_expert, m_tiles,
                                            packed_a, out, out_ld, status, s, token_of_row, w,
                                            pf_bytes);
}

template <bool GATE_UP, bool FP4 = false, bool TT = false>
cudaError_t launch_fp8(const CUtensorMap& a, const TokenMaps& b, const int32_t* offsets,
                       const void* scales, int E, int K, int a_rows_per_expert, int m_tiles,
                       void* out, int out_ld, int* status, cudaStream_t s) {
    const int smem = q_smem_bytes<GATE_UP, FP4, TT>();
    cudaError_t err = cudaFuncSetAttribute(grouped_gemm_pair_fp8_kernel<GATE_UP, FP4, TT>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * sm_pairs(), 1, 1);
    cfg.blockDim = dim3(THREADS_Q, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_pdl
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    err = cudaLaunchKernelEx(&cfg, grouped_gemm_pair_fp8_kernel<GATE_UP, FP4, TT>, a, b, offsets, scales, E,
                             K, a_rows_per_expert, m_tiles, static_cast<__nv_bfloat16*>(out),
                             out_ld, status);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

}  // namespace

bool pair_gemm_supported(const moe_config& c) { return c.d % 256 == 0 && c.d_ff % 256 == 0; }

namespace {
// The FP8 down GEMM's pair tiles: one A tile of 256 rows against two token
// sub-tiles of up to 192 rows (each K block of weights widened once for up to
// 384 tokens) once the experts average at least 128 grouped rows; two A tiles
// against one token tile of up to 192 rows below that. (The same split for
// gate_up, its gate and up rows paired in each TMEM lane quarter, measured
// 2-3% slower: its epilogue then pairs g and u across lanes.)
bool fp8_two_subtiles(const moe_config& g) { return (long)g.T * g.k >= 128L * g.E; }
}  // namespace

cudaError_t launch_gate_up_gemm_pair_fp8(const moe_config& c, const void* x_perm,
                                         const int32_t* offsets, const void* w_gate_up,
                                         const float* s_gate_up, void* h, int* status,
                                         cudaStream_t s) {
    CUtensorMap a;
    TokenMaps b;
    const uint64_t R = (uint64_t)c.T * c.k;
    if (!make_map_u8(&a, w_gate_up, (uint64_t)c.E * 2 * c.d_ff, c.d, BM, 64, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_token_maps(&b, x_perm, R, c.d))
        return cudaErrorInvalidValue;
    return launch_fp8<true>(a, b, offsets, s_gate_up, c.E, c.d, 2 * c.d_ff, c.d_ff / (2 * BM), h,
                            c.d_ff, status, s);
}

cudaError_t launch_down_gemm_pair_fp8(const moe_config& c, const void* h, const int32_t* offsets,
                                      const void* w_down, const float* s_down, void* y,
                                      int* status, cudaStream_t s) {
    CUtensorMap a;
    TokenMaps b;
    const uint64_t R = (uint64_t)c.T * c.k;
    if (!make_map_u8(&a, w_down, (uint64_t)c.E * c.d, c.d_ff, BM, 64, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_token_maps(&b, h, R, c.d_ff))
        return cudaErrorInvalidValue;
    if (fp8_two_subtiles(c))
        return launch_fp8<false, false, true>(a, b, offsets, s_down, c.E, c.d_ff, c.d,
                                              (c.d + 2 * BM - 1) / (2 * BM), y, c.d, status, s);
    return launch_fp8<false>(a, b, offsets, s_down, c.E, c.d_ff, c.d, (c.d + 4 * BM - 1) / (4 * BM),
                             y, c.d, status, s);
}

cudaError_t launch_gate_up_gemm_pair_fp4(const moe_config& c, const void* x_perm,
                                         const int32_t* offsets, const void* w_gate_up,
                                         const void* s_gate_up, void* h, int* status,
                                         cudaStream_t s) {
    CUtensorMap a;
    TokenMaps b;
    const uint64_t R = (uint64_t)c.T * c.k;
    if (!make_map_u8(&a, w_gate_up, (uint64_t)c.E * 2 * c.d_ff, c.d / 2, BM, 32, CU_TENSOR_MAP_SWIZZLE_32B) ||
        !make_token_maps(&b, x_perm, R, c.d))
        return cudaErrorInvalidValue;
    return launch_fp8<true, true>(a, b, offsets, s_gate_up, c.E, c.d, 2 * c.d_ff,
                                  c.d_ff / (2 * BM), h, c.d_ff, status, s);
}

cudaError_t launch_down_gemm_pair_fp4(const moe_config& c, const void* h, const int32_t* offsets,
                                      const void* w_down, const void* s_down, void* y,
                                      int* status, cudaStream_t s) {
    CUtensorMap a;
    TokenMaps b;
    const uint64_t R = (uint64_t)c.T * c.k;
    if (!make_map_u8(&a, w_down, (uint64_t)c.E * c.d, c.d_ff / 2, BM, 32, CU_TENSOR_MAP_SWIZZLE_32B) ||
        !make_token_maps(&b, h, R, c.d_ff))
        return cudaErrorInvalidValue;
    return launch_fp8<false, true>(a, b, offsets, s_down, c.E, c.d_ff, c.d,
                                   (c.d + 4 * BM - 1) / (4 * BM), y, c.d, status, s);
}

cudaError_t launch_gate_up_gemm_pair(const moe_config& c, const void* x_perm,
                                     const int32_t* offsets, const void* w_gate_up, bool packed,
                                     void* h, int* status, cudaStream_t s) {
    CUtensorMap a;
    TokenMaps b;
    const uint64_t R = (uint64_t)c.T * c.k;
    if (!make_weight_map(&a, w_gate_up, (uint64_t)c.E * 2 * c.d_ff, c.d, packed) ||
        !make_token_maps(&b, x_perm, R, c.d))
        return cudaErrorInvalidValue;
    return launch<true>(c.T, a, b, offsets, c.E, c.d, 2 * c.d_ff, c.d_ff / (2 * BM), packed, h, c.d_ff,
                        status, s, nullptr, w_gate_up, (long long)c.E * 2 * c.d_ff * c.d * 2);
}

cudaError_t launch_gate_up_gemm_pair_gather(const moe_config& c, const void* x,
                                            const int32_t* token_of_row, const int32_t* offsets,
                                            const void* w_gate_up, bool packed, void* h,
                                            int* status, cudaStream_t s) {
    CUtensorMap a;
    TokenMaps b = {};
    if (!make_weight_map(&a, w_gate_up, (uint64_t)c.E * 2 * c.d_ff, c.d, packed) ||
        !make_map(&b.m[0], x, (uint64_t)c.T, c.d, 1))
        return cudaErrorInvalidValue;
    return launch<true, true>(c.T, a, b, offsets, c.E, c.d, 2 * c.d_ff, c.d_ff / (2 * BM), packed, h,
                              c.d_ff, status, s, token_of_row, w_gate_up,
                              (long long)c.E * 2 * c.d_ff * c.d * 2);
}

cudaError_t launch_down_gemm_pair(const moe_config& c, const void* h, const int32_t* offsets,
                                  const void* w_down, bool packed, void* y, int* status,
                                  cudaStream_t s) {
    CUtensorMap a;
    TokenMaps b;
    const uint64_t R = (uint64_t)c.T * c.k;
    if (!make_weight_map(&a, w_down, (uint64_t)c.E * c.d, c.d_ff, packed) ||
        !make_token_maps(&b, h, R, c.d_ff))
        return cudaErrorInvalidValue;
    return launch<false>(c.T, a, b, offsets, c.E, c.d_ff, c.d, (c.d + 4 * BM - 1) / (4 * BM), packed, y,
                         c.d, status, s, nullptr, w_down, (long long)c.E * c.d * c.d_ff * 2);
}

namespace {

// Packed block layout: 16-byte chunk i of the output is chunk i % 8 of row
// (i / 8) % 128 of block i / 1024; block b holds rows [128 (b / KB), +128) and
// columns [64 (b % KB), +64) of the [E * rows, cols] source (KB = cols / 64).
__global__ void __launch_bounds__(256)
pack_weights_kernel(const uint4* __restrict__ w, uint4* __restrict__ wp, long n16, int cols) {
    const int kbs = cols / BK;
    for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n16;
         i += (long)gridDim.x * blockDim.x) {
        const long b = i >> 10;
        const int r = (int)((i >> 3) & 127), ch = (int)(i & 7);
        const long row = (b / kbs) * BM + r;
        const long col = (b % kbs) * BK + ch * 8;
        wp[i] = w[(row * cols + col) / 8];
    }
}

}  // namespace

cudaError_t launch_pack_weights(int E, int rows, int cols, const void* w, void* w_packed,
                                cudaStream_t s) {
    const long n16 = (long)E * rows * cols / 8;
    const long blocks = (n16 + 255) / 256;
    pack_weights_kernel<<<(unsigned)(blocks < 148L * 64 ? blocks : 148L * 64), 256, 0, s>>>(
        static_cast<const uint4*>(w), static_cast<uint4*>(w_packed), n16, cols);
    return cudaGetLastError();
}

}  // namespace moe
