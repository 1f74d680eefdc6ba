// Grouped expert GEMMs for small token counts (decode), tcgen05 + TMEM + TMA.
//
// At decode an expert sees a handful of tokens, so the roles of the operands are
// swapped: the expert's weight rows are the 128-row MMA operand A and the tokens
// are the narrow operand B (a 32-token tile, MMA N = 32).  Every weight byte of
// a hit expert is streamed from HBM once per 32 tokens, the tensor pipe does no
// work on padding rows of weights, and the permuted token layout is padded to 32
// rows per expert instead of 128.  The accumulator D^T (TMEM lane = output
// feature, column = token) is transposed through shared memory so that every
// global store is a 16-byte piece of a token's row.
//
// Same warp roles and pipeline as the prefill kernels (warp 0 TMA, warp 1 MMA,
// warps 2-5 epilogue; a ring of 10 (gate_up) or 8 (down) stages of 16 KiB weights
// + 4 KiB tokens; two 32-column accumulators).  Same arithmetic ("GLM-4.5 MoE Forward", How it works):
//
// gate_up: one tile = 64 intermediate features of one expert x 32 tokens; A stacks
//   the 64 gate rows and the matching 64 up rows, so TMEM lanes 0..63 hold the
//   gate and 64..127 the up projection of the same features; the epilogue writes
//   h = SiLU(gate) * up in bf16.
// down: one tile = 128 output features x 32 tokens.  Routed tiles scale each
//   token by its routing weight and store its bf16 slot partial; the shared
//   expert's tiles come last and, after a bounded wait for every routed tile,
//   add the k slot partials in slot order plus the fp32 shared accumulator and
//   write y once.
#pragma once

#include "common.cuh"
#include "gemm_sm100.cuh"

namespace moe {

constexpr int DEC_BM = 128;     // weight rows per tile (MMA M)
constexpr int DEC_TT = 32;      // tokens per tile (MMA N)
constexpr int DEC_BK = 64;
constexpr int DEC_THREADS = 192;
constexpr int DEC_A_BYTES = DEC_BM * DEC_BK * 2;  // 16 KiB
constexpr int DEC_B_BYTES = DEC_TT * DEC_BK * 2;  // 4 KiB
constexpr int DEC_STAGE_BYTES = DEC_A_BYTES + DEC_B_BYTES;
constexpr int DEC_TMEM_COLS = 64;                 // 2 accumulators x 32 columns
constexpr int DEC_EPI_LD = 132;                   // floats per token row of the transpose buffer
constexpr int DEC_EPI_BYTES = DEC_TT * DEC_EPI_LD * 4;
// Ring depth per kernel.  A streaming kernel's bandwidth per SM is its bytes in
// flight over the memory latency: gate_up takes 10 stages (200 KiB of weights in
// flight; 2 % faster than 8 on the decode workloads).  The down kernel stays at 8:
// its combine reads the slot partials through L1, which the larger shared-memory
// carve-out shrinks (1-2 % slower at 10 stages).
template <int KIND> __host__ __device__ constexpr int dec_stages() { return KIND == GEMM_GATE_UP ? 10 : 8; }
template <int KIND> __host__ __device__ constexpr int dec_smem_bytes() {
    return 1024 + dec_stages<KIND>() * DEC_STAGE_BYTES + 256 + (2 * GEMM_MAXE + 1) * 4 +
           DEC_EPI_BYTES + 64;
}
static_assert(dec_smem_bytes<GEMM_GATE_UP>() <= 232448, "shared memory");
static_assert(dec_smem_bytes<GEMM_DOWN>() <= 232448, "shared memory");
// mbarriers (full/empty per stage, 2 tfull, 2 tempty, drain) and three words fit the
// 256 bytes after the ring
static_assert((2 * 10 + 5) * 8 + 12 <= 256, "barrier block");

struct DecArgs {
    const int32_t *tile_off; // [E+1] prefix of 32-token tiles per expert
    const int32_t *counts;   // [E]
    int32_t *meta;           // [0] routed tiles done (down), [2] routed token tiles
    int E, N, k;
    int nb_r, nb_s;          // feature blocks per routed / shared token tile
    int tt_s;                // shared token tiles
    int kb_r, kb_s;          // k-blocks of routed / shared tiles
    int a_rows_per_e;        // rows of one expert in the routed A map (2d or D)
    int up_off;              // gate_up: row offset of the up half (d)
    __nv_bfloat16 *out_r;    // gate_up: h_perm; down: slot
    int ld_r, ncols_r;
    __nv_bfloat16 *out_s;    // gate_up: h_sh; down: y
    int ld_s, ncols_s;
    const float *w_perm;
    const int32_t *pos_of;
    const __nv_bfloat16 *slot;
    uint64_t wait_limit_ns;
    int never_signal;
    float gate_max, up_max; // gate_up: SwiGLU limits (+infinity = plain SwiGLU)
};

struct DecTile {
    bool shared;
    int e;       // routed expert
    int row0;    // first token row (permuted row for routed, token for shared)
    int m_valid; // real tokens in the tile
    int fb;      // feature block
    int kb;      // k-blocks
};

__device__ __forceinline__ DecTile dec_decode_tile(int t, int routed_tiles, const DecArgs &a,
                                                   const int *s_off, const int *s_cnt) {
    DecTile c;
    if (t < routed_tiles) {
        const int mt = t / a.nb_r;
        c.fb = t - mt * a.nb_r;
        int lo = 0, hi = a.E - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_off[mid] <= mt) lo = mid; else hi = mid - 1;
        }
        c.shared = false;
        c.e = lo;
        c.row0 = mt * DEC_TT;
        c.m_valid = min(DEC_TT, s_cnt[lo] - (mt - s_off[lo]) * DEC_TT);
        c.kb = a.kb_r;
    } else {
        const int t2 = t - routed_tiles;
        const int mt = t2 / a.nb_s;
        c.fb = t2 - mt * a.nb_s;
        c.shared = true;
        c.e = -1;
        c.row0 = mt * DEC_TT;
        c.m_valid = min(DEC_TT, a.N - c.row0);
        c.kb = a.kb_s;
    }
    return c;
}

// KIND: GEMM_GATE_UP or GEMM_DOWN.
// Maps: mA_r routed weights (gate_up [E*2d, D] box 64 rows; down [E*D, d] box 128),
//       mB_r permuted tokens (x_perm / h_perm, box 32 rows),
//       mA_s0 / mA_s1 shared weights (sh_gate, sh_up box 64; sh_down box 128),
//       mB_s shared tokens (x / h_sh, box 32 rows).
template <int KIND>
__global__ void __launch_bounds__(DEC_THREADS, 1)
    grouped_gemm_decode_kernel(const __grid_constant__ CUtensorMap mA_r,
                               const __grid_constant__ CUtensorMap mB_r,
                               const __grid_constant__ CUtensorMap mA_s0,
                               const __grid_constant__ CUtensorMap mA_s1,
                               const __grid_constant__ CUtensorMap mB_s, const DecArgs a) {
    constexpr int DEC_STAGES = dec_stages<KIND>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + DEC_STAGES * DEC_STAGE_BYTES);
    uint64_t *empty = full + DEC_STAGES;
    uint64_t *tfull = empty + DEC_STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *combine_failed = abort_flag + 1;
    int *s_off = reinterpret_cast<int *>(smem + DEC_STAGES * DEC_STAGE_BYTES + 256);
    int *s_cnt = s_off + GEMM_MAXE + 1;
    float *epi = reinterpret_cast<float *>(s_cnt + GEMM_MAXE); // [DEC_TT][DEC_EPI_LD]

    const int warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < DEC_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        *combine_failed = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&mA_r);
        tma_prefetch_desc(&mB_r);
        tma_prefetch_desc(&mA_s0);
        if (KIND == GEMM_GATE_UP) tma_prefetch_desc(&mA_s1);
        tma_prefetch_desc(&mB_s);
    }
    // Nothing above reads or writes global memory or TMEM, so it may overlap the
    // previous kernel of the stream (programmatic launch); everything below follows it.
    grid_dep_wait();
    grid_dep_launch_dependents();
    if (warp == 1) {
        tmem_alloc(tmem_slot, DEC_TMEM_COLS);
        tmem_relinquish();
    }
    for (int i = threadIdx.x; i <= a.E; i += blockDim.x) {
        s_off[i] = a.tile_off[i];
        if (i < a.E) s_cnt[i] = a.counts[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int routed_tiles = a.meta[2] * a.nb_r;
    const int total_tiles = routed_tiles + a.tt_s * a.nb_s;
    const uint64_t limit = a.wait_limit_ns;

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                const DecTile c = dec_decode_tile(t, routed_tiles, a, s_off, s_cnt);
                const CUtensorMap *mB = c.shared ? &mB_s : &mB_r;
                // Feature blocks of one token tile run on neighbouring CTAs and share
                // the token tile; start each at a different k-block.
                const int rot = c.fb % c.kb;
                for (int i = 0; i < c.kb; ++i, ++it) {
                    const int kb = i + rot < c.kb ? i + rot : i + rot - c.kb;
                    const uint32_t s = it % DEC_STAGES, ph = (it / DEC_STAGES) & 1;
                    if (!mbar_wait(&empty[s], ph ^ 1, limit, abort_flag, 200)) { ok = false; break; }
                    uint8_t *sa = ring + s * DEC_STAGE_BYTES;
                    uint8_t *sb = sa + DEC_A_BYTES;
                    mbar_arrive_expect_tx(&full[s], DEC_STAGE_BYTES);
                    const int kx = kb * DEC_BK;
                    if (KIND == GEMM_GATE_UP) {
                        if (c.shared) {
                            tma_load_2d(&mA_s0, &full[s], sa, kx, c.fb * 64);
                            tma_load_2d(&mA_s1, &full[s], sa + DEC_A_BYTES / 2, kx, c.fb * 64);
                        } else {
                            const int r0 = c.e * a.a_rows_per_e + c.fb * 64;
                            tma_load_2d(&mA_r, &full[s], sa, kx, r0);
                            tma_load_2d(&mA_r, &full[s], sa + DEC_A_BYTES / 2, kx, r0 + a.up_off);
                        }
                    } else {
                        if (c.shared)
                            tma_load_2d(&mA_s0, &full[s], sa, kx, c.fb * DEC_BM);
                        else
                            tma_load_2d(&mA_r, &full[s], sa, kx, c.e * a.a_rows_per_e + c.fb * DEC_BM);
                    }
                    tma_load_2d(mB, &full[s], sb, kx, c.row0);
                }
            }
            if (!ok) {
                const uint32_t first = it > DEC_STAGES ? it - DEC_STAGES : 0;
                for (uint32_t j = first; j < it; ++j) {
                    volatile int no_abort = 0;
                    mbar_wait(&full[j % DEC_STAGES], (j / DEC_STAGES) & 1, 10000000ull, &no_abort, 201);
                }
            }
        }
        __syncwarp(); // lanes 1-31 wait here for lane 0: the warp reconverges
    } else if (warp == 1) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(DEC_BM, DEC_TT);
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++tc) {
                const DecTile c = dec_decode_tile(t, routed_tiles, a, s_off, s_cnt);
                const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
                if (!mbar_wait(&tempty[acc], aph ^ 1, limit, abort_flag, 210)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * DEC_TT;
                for (int i = 0; i < c.kb; ++i, ++it) {
                    const uint32_t s = it % DEC_STAGES, ph = (it / DEC_STAGES) & 1;
                    if (!mbar_wait(&full[s], ph, limit, abort_flag, 211)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(ring + s * DEC_STAGE_BYTES);
                    const uint32_t sb = sa + DEC_A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < DEC_BK / 16; ++kk)
                        umma_bf16_ss(d_tmem, umma_desc_sw128(sa + kk * 32),
                                     umma_desc_sw128(sb + kk * 32), idesc,
                                     (i > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[s]);
                }
                if (!ok) break;
                umma_commit(&tfull[acc]);
            }
            umma_commit(drain);
            volatile int no_abort = 0;
            mbar_wait(drain, 0, 100000000ull, &no_abort, 212);
        }
        __syncwarp();
    } else {
        // ------------------------------ epilogue ---------------------------------
        const int q = warp & 3;
        const int f = q * 32 + lane;      // TMEM lane = output feature row of the tile
        const int ep_tid = threadIdx.x - 64;
        uint32_t tc = 0;
        for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++tc) {
            const DecTile c = dec_decode_tile(t, routed_tiles, a, s_off, s_cnt);
            const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
            bool do_combine = true;
            if (KIND == GEMM_DOWN && c.shared) {
                if (ep_tid == 0 && !*combine_failed && !*abort_flag) {
                    const int target = routed_tiles + (a.never_signal ? 1 : 0);
                    const uint64_t t0 = globaltimer_ns();
                    while (ld_acquire_gpu(&a.meta[0]) < target) {
                        if (globaltimer_ns() - t0 > limit) {
                            record_error(DEV_TIMEOUT, 220);
                            *combine_failed = 1;
                            break;
                        }
                        __nanosleep(200);
                    }
                }
                named_bar_sync(1, 128);
                do_combine = !*combine_failed;
            }
            bool have = false;
            if (lane == 0) have = mbar_wait(&tfull[acc], aph, limit, abort_flag, 221);
            have = __shfl_sync(0xffffffffu, have ? 1 : 0, 0) != 0;
            __syncwarp();
            if (have) {
                tc_fence_after();
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + acc * DEC_TT + ((uint32_t)(q * 32) << 16), v);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
#pragma unroll
                for (int tk = 0; tk < DEC_TT; ++tk) epi[tk * DEC_EPI_LD + f] = __uint_as_float(v[tk]);
            }
            named_bar_sync(1, 128);
            if (have) {
                if (KIND == GEMM_GATE_UP) {
                    // 32 tokens x 8 pieces of 8 features (64 features per tile)
                    __nv_bfloat16 *out = c.shared ? a.out_s : a.out_r;
                    const int ld = c.shared ? a.ld_s : a.ld_r;
                    const int ncols = c.shared ? a.ncols_s : a.ncols_r;
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int i = ep_tid + 128 * jj;
                        const int tk = i >> 3, pc = i & 7;
                        const int col = c.fb * 64 + pc * 8;
                        if (tk < c.m_valid && col < ncols) {
                            const float *g = epi + tk * DEC_EPI_LD + pc * 8;
                            const float *u = g + 64;
                            uint32_t pk[4];
#pragma unroll
                            for (int h = 0; h < 4; ++h)
                                pk[h] = pack_bf16x2(swiglu_f(g[2 * h], u[2 * h], a.gate_max, a.up_max),
                                                    swiglu_f(g[2 * h + 1], u[2 * h + 1], a.gate_max,
                                                             a.up_max));
                            *reinterpret_cast<uint4 *>(out + (size_t)(c.row0 + tk) * ld + col) =
                                make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                } else if (!c.shared) {
                    // 32 tokens x 16 pieces of 8 output features, scaled by the routing weight
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int i = ep_tid + 128 * jj;
                        const int tk = i >> 4, pc = i & 15;
                        const int col = c.fb * DEC_BM + pc * 8;
                        if (tk < c.m_valid && col < a.ncols_r) {
                            const float wr = a.w_perm[c.row0 + tk];
                            const float *o = epi + tk * DEC_EPI_LD + pc * 8;
                            uint32_t pk[4];
#pragma unroll
                            for (int h = 0; h < 4; ++h)
                                pk[h] = pack_bf16x2(wr * o[2 * h], wr * o[2 * h + 1]);
                            *reinterpret_cast<uint4 *>(a.out_r + (size_t)(c.row0 + tk) * a.ld_r + col) =
                                make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                } else if (do_combine) {
                    // y[n] = sum of the k slot partials in slot order + shared accumulator
#pragma unroll 1
                    for (int jj = 0; jj < 4; ++jj) {
                        const int i = ep_tid + 128 * jj;
                        const int tk = i >> 4, pc = i & 15;
                        const int col = c.fb * DEC_BM + pc * 8;
                        if (tk < c.m_valid && col < a.ncols_s) {
                            const int n = c.row0 + tk;
                            float sum[8];
#pragma unroll
                            for (int h = 0; h < 8; ++h) sum[h] = 0.f;
                            // eight slots fetched before any is added; adds in slot order
                            for (int jb = 0; jb < a.k; jb += 8) {
                                uint4 w[8];
#pragma unroll
                                for (int jj = 0; jj < 8; ++jj) {
                                    const int j = jb + jj;
                                    const int p = j < a.k ? a.pos_of[(size_t)n * a.k + j] : -1;
                                    w[jj] = p >= 0 ? __ldcg(reinterpret_cast<const uint4 *>(
                                                         a.slot + (size_t)p * a.ld_r + col))
                                                   : make_uint4(0u, 0u, 0u, 0u);
                                }
#pragma unroll
                                for (int jj = 0; jj < 8; ++jj) acc_bf16x8(sum, w[jj]);
                            }
                            const float *o = epi + tk * DEC_EPI_LD + pc * 8;
                            uint32_t pk[4];
#pragma unroll
                            for (int h = 0; h < 4; ++h)
                                pk[h] = pack_bf16x2(sum[2 * h] + o[2 * h], sum[2 * h + 1] + o[2 * h + 1]);
                            *reinterpret_cast<uint4 *>(a.out_s + (size_t)n * a.ld_s + col) =
                                make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                }
            }
            if (KIND == GEMM_DOWN && !c.shared) __threadfence();
            named_bar_sync(1, 128); // the transpose buffer is free again
            if (KIND == GEMM_DOWN && !c.shared && ep_tid == 0 && have) atomicAdd(&a.meta[0], 1);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, DEC_TMEM_COLS);
    }
}

}  // namespace moe
