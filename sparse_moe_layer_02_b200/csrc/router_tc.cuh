// Router logits on the tensor cores for bf16 tokens and a bf16 router matrix
// ("GLM-4.5 Group Router", How it works: r = x W_g^T in float32; bf16 x bf16
// products are exact in fp32 and tcgen05 accumulates in fp32).
//
// One cluster of CLK CTAs per 128 tokens: CTA r multiplies the tokens' rows by
// W_g over the r-th slice of the hidden dimension (M = 128 tokens, N = E
// experts, K = 16 per instruction; TMA-fed 4-stage ring; one 128 x E fp32
// accumulator in TMEM).  The partial logits go to shared memory; after a cluster
// barrier, warps take whole tokens, sum the CLK partial rows in rank order
// (distributed shared memory; a fixed order, so the result is deterministic) and
// run the same warp-shuffle selection as the CUDA-core router.  CLK = 1 for
// large batches; small batches split K over up to 8 CTAs so more SMs stream W_g.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "router.cuh"

namespace moe {

constexpr int RTC_BM = 128;
constexpr int RTC_BK = 64;
constexpr int RTC_STAGES = 4;
constexpr int RTC_THREADS = 256;   // warp 0 TMA, warp 1 MMA, warps 4-7 TMEM drain, all select
constexpr int RTC_A_BYTES = RTC_BM * RTC_BK * 2;     // 16 KiB
constexpr int RTC_B_BYTES_MAX = 256 * RTC_BK * 2;    // 32 KiB (E <= 256)
constexpr int RTC_STAGE_BYTES = RTC_A_BYTES + RTC_B_BYTES_MAX;
constexpr int RTC_PART_LD = 257;                     // floats per token row of the partials
constexpr int RTC_SMEM_BYTES = 1024 + RTC_STAGES * RTC_STAGE_BYTES + 256 +
                               (RTC_THREADS / 32) * ROUTER_MAXV * 32 * 4;
static_assert(RTC_BM * RTC_PART_LD * 4 <= RTC_STAGES * RTC_STAGE_BYTES,
              "partial logits reuse the operand ring");

template <int EV>
__global__ void __launch_bounds__(RTC_THREADS, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mW,
                     const RouterParams p, uint64_t limit) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + RTC_STAGES * RTC_STAGE_BYTES);
    uint64_t *empty = full + RTC_STAGES;
    uint64_t *tfull = empty + RTC_STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tfull + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *spbuf = reinterpret_cast<float *>(smem + RTC_STAGES * RTC_STAGE_BYTES + 256);
    float *part = reinterpret_cast<float *>(ring); // [128][RTC_PART_LD] after the main loop

    cg::cluster_group cluster = cg::this_cluster();
    const int CLK = gridDim.x;
    const int rank = blockIdx.x;
    const int t0 = blockIdx.y * RTC_BM;
    const int warp = warp_id(), lane = lane_id();
    const int E = p.E;
    const int KB = (p.D + RTC_BK - 1) / RTC_BK;
    const int kper = (KB + CLK - 1) / CLK;
    const int kb0 = rank * kper, kb1 = min(KB, kb0 + kper);
    const uint32_t b_bytes = (uint32_t)E * RTC_BK * 2;
    // Every CTA reads the same W_g slices; rotating the k-block order by the token
    // block spreads concurrent reads over different L2 lines instead of having all
    // CTAs request the same 32 KiB at once.
    const int nkb = kb1 - kb0;
    const int rot = nkb > 0 ? (int)(blockIdx.y % (unsigned)nkb) : 0;
    const uint32_t tmem_cols = E <= 32 ? 32 : E <= 64 ? 64 : E <= 128 ? 128 : 256;

    if (threadIdx.x == 0) {
        for (int s = 0; s < RTC_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tfull, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&mX);
        tma_prefetch_desc(&mW);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int i = 0; i < nkb; ++i, ++it) {
                const int kb = kb0 + (i + rot < nkb ? i + rot : i + rot - nkb);
                const uint32_t s = it % RTC_STAGES, ph = (it / RTC_STAGES) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, limit, abort_flag, 300)) { ok = false; break; }
                uint8_t *sa = ring + s * RTC_STAGE_BYTES;
                mbar_arrive_expect_tx(&full[s], RTC_A_BYTES + b_bytes);
                tma_load_2d(&mX, &full[s], sa, kb * RTC_BK, t0);
                tma_load_2d(&mW, &full[s], sa + RTC_A_BYTES, kb * RTC_BK, 0);
            }
            if (!ok) {
                const uint32_t first = it > RTC_STAGES ? it - RTC_STAGES : 0;
                for (uint32_t j = first; j < it; ++j) {
                    volatile int no_abort = 0;
                    mbar_wait(&full[j % RTC_STAGES], (j / RTC_STAGES) & 1, 10000000ull, &no_abort, 301);
                }
            }
        }
        __syncwarp(); // lanes 1-31 wait here for lane 0: the warp reconverges
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_bf16(RTC_BM, E);
            uint32_t it = 0;
            for (int i = 0; i < nkb; ++i, ++it) {
                const uint32_t s = it % RTC_STAGES, ph = (it / RTC_STAGES) & 1;
                if (!mbar_wait(&full[s], ph, limit, abort_flag, 310)) break;
                tc_fence_after();
                const uint32_t sa = smem_u32(ring + s * RTC_STAGE_BYTES);
                const uint32_t sb = sa + RTC_A_BYTES;
#pragma unroll
                for (int kk = 0; kk < RTC_BK / 16; ++kk)
                    umma_bf16_ss(tmem_base, umma_desc_sw128(sa + kk * 32),
                                 umma_desc_sw128(sb + kk * 32), idesc,
                                 (i > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&empty[s]);
            }
            umma_commit(tfull); // arrives once every MMA issued above has completed
        }
        __syncwarp();
    } else if (warp >= 4) {
        // Drain the accumulator: TMEM lane = token row, column = expert.
        const int q = warp & 3;
        const int row = q * 32 + lane;
        bool have = false;
        if (lane == 0) have = mbar_wait(tfull, 0, limit, abort_flag, 320);
        have = __shfl_sync(0xffffffffu, have ? 1 : 0, 0) != 0;
        __syncwarp();
        if (have) tc_fence_after();
        const bool empty_k = kb0 >= kb1;
        for (int c0 = 0; c0 < E; c0 += 32) {
            uint32_t v[32];
            if (have) {
                tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + c0, v);
                tmem_ld_wait();
            }
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (c0 + i < E) part[row * RTC_PART_LD + c0 + i] = (have && !empty_k) ? __uint_as_float(v[i]) : 0.f;
        }
    }
    tc_fence_before();
    cluster.sync();

    // ---- sum the cluster's partial logits and select: one warp per token -------
    const int tpc = RTC_BM / CLK; // tokens finalised by this CTA
    for (int jl = warp; jl < tpc; jl += RTC_THREADS / 32) {
        const int j = rank * tpc + jl;
        const int t = t0 + j;
        if (t >= p.N) break;
        float logit[EV];
#pragma unroll
        for (int v = 0; v < EV; ++v) {
            const int e = lane + 32 * v;
            float r = 0.f;
            if (e < E) {
                for (int c = 0; c < CLK; ++c) {
                    const float *remote = cluster.map_shared_rank(part, c);
                    r += remote[j * RTC_PART_LD + e];
                }
            }
            logit[v] = r;
        }
        router_select<EV>(p, t, logit, spbuf + warp * ROUTER_MAXV * 32, lane);
    }
    cluster.sync(); // partials stay alive until every reader is done
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols);
    }
}

}  // namespace moe
