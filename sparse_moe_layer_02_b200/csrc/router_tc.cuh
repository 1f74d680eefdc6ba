// Router logits on the tensor cores ("GLM-4.5 Group Router", How it works:
// r = x W_g^T in float32) for bf16 tokens and a bf16 or fp32 router matrix.
//
// bf16 W_g: bf16 x bf16 products are exact in fp32 and tcgen05 accumulates in
// fp32.  fp32 W_g: every element is split into three bf16 parts,
// w = w1 + w2 + w3 with w1 = bf16(w), w2 = bf16(w - w1), w3 = bf16(w - w1 - w2)
// (each residual is exact in fp32, and the split reproduces w to 2^-27 relative,
// finer than fp32 rounding), and x W_g^T is accumulated as three bf16 products:
// the large part in one set of fp32 accumulators, the two small parts in
// another.  Idle warps do the split into shared memory while the TMA fetches
// the tokens.
//
// One cluster of CLK CTAs per 128 tokens: CTA r multiplies the tokens' rows by
// W_g over the r-th slice of the hidden dimension (M = 128 tokens, N = E
// experts, K = 16 per instruction; 128 x E fp32 accumulators in TMEM, k-blocks
// rotating over several of them and summed in a fixed order at the end).  The
// partial logits go to shared memory; after a cluster barrier, warps take whole
// tokens, sum the CLK partial rows in rank order (distributed shared memory; a
// fixed order, so the result is deterministic) and run the same warp-shuffle
// selection as the CUDA-core router.  CLK = 1 for large batches; small batches
// split K over up to 16 CTAs so more SMs stream W_g.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "dispatch.cuh"
#include "router.cuh"

namespace moe {

constexpr int RTC_BM = 128;
constexpr int RTC_BK = 64;
constexpr int RTC_THREADS = 256;  // warp 0 TMA, warp 1 MMA, warps 2-7 split (fp32), 4-7 drain
constexpr int RTC_A_BYTES = RTC_BM * RTC_BK * 2;  // 16 KiB
constexpr int RTC_PART_LD = 257;                  // floats per token row of the partials
constexpr int RTC_MAXE_F32 = 192;                 // largest E of the fp32-W_g variant
constexpr int RTC_MAX_CLK = 16;                   // largest K-split cluster (non-portable size)
constexpr int RTC_MAX_KB = 24;                    // k-blocks per CTA above which K is split further

template <bool WF32> struct RtcCfg {
    static constexpr int STAGES = WF32 ? 2 : 4;
    static constexpr int B_PART = (WF32 ? RTC_MAXE_F32 : 256) * RTC_BK * 2; // one bf16 B tile
    static constexpr int B_BYTES = (WF32 ? 3 : 1) * B_PART;
    static constexpr int STAGE_BYTES = RTC_A_BYTES + B_BYTES;
    static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 256 +
                                (RTC_THREADS / 32) * ROUTER_MAXV * 32 * 4;
    static_assert(STAGE_BYTES % 1024 == 0, "stages stay 1024-byte aligned");
    static_assert(RTC_BM * RTC_PART_LD * 4 <= STAGES * STAGE_BYTES,
                  "partial logits reuse the operand ring");
};


// Split 8 fp32 router weights into three bf16 parts w = w1 + w2 + w3 (each part
// packed as 8 bf16 in a uint4).
__device__ __forceinline__ void split8(const float4 &u, const float4 &v, uint4 &q1, uint4 &q2,
                                       uint4 &q3) {
    const float w[8] = {u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w};
    uint32_t p1[4], p2[4], p3[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        float a1[2], a2[2], a3[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const float x0 = w[2 * h + q];
            const __nv_bfloat16 h1 = __float2bfloat16_rn(x0);
            const float r1 = x0 - __bfloat162float(h1);
            const __nv_bfloat16 h2 = __float2bfloat16_rn(r1);
            const float r2 = r1 - __bfloat162float(h2);
            a1[q] = __bfloat162float(h1);
            a2[q] = __bfloat162float(h2);
            a3[q] = r2;
        }
        p1[h] = pack_bf16x2(a1[0], a1[1]);
        p2[h] = pack_bf16x2(a2[0], a2[1]);
        p3[h] = pack_bf16x2(a3[0], a3[1]);
    }
    q1 = make_uint4(p1[0], p1[1], p1[2], p1[3]);
    q2 = make_uint4(p2[0], p2[1], p2[2], p2[3]);
    q3 = make_uint4(p3[0], p3[1], p3[2], p3[3]);
}

// The three parts of 8 weights written as one 16-byte chunk of each part's K-major
// tile with the 128-byte swizzle the MMA descriptor uses.
__device__ __forceinline__ void split_store(uint8_t *b0, int row, int chunk, const float4 &u,
                                            const float4 &v, int part_bytes) {
    uint4 q1, q2, q3;
    split8(u, v, q1, q2, q3);
    const int off = row * 128 + ((chunk ^ (row & 7)) << 4);
    *reinterpret_cast<uint4 *>(b0 + off) = q1;
    *reinterpret_cast<uint4 *>(b0 + part_bytes + off) = q2;
    *reinterpret_cast<uint4 *>(b0 + 2 * part_bytes + off) = q3;
}

// The same split of the whole fp32 W_g [E][D] into parts [3][E][D] in global memory,
// once per call, for batches of several token blocks: the router then loads the
// three parts by TMA instead of splitting them again in every token block.
// D % 8 == 0; one thread per 8 weights.
__global__ void __launch_bounds__(256) wg_split_kernel(const float *__restrict__ W, int E, int D,
                                                       __nv_bfloat16 *__restrict__ parts) {
    const size_t n8 = (size_t)E * D / 8;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8;
         i += (size_t)gridDim.x * blockDim.x) {
        const float4 u = __ldg(reinterpret_cast<const float4 *>(W) + 2 * i);
        const float4 v = __ldg(reinterpret_cast<const float4 *>(W) + 2 * i + 1);
        uint4 q1, q2, q3;
        split8(u, v, q1, q2, q3);
        uint4 *out = reinterpret_cast<uint4 *>(parts);
        out[i] = q1;
        out[n8 + i] = q2;
        out[2 * n8 + i] = q3;
    }
}

// Dispatch fused into the router for a batch of at most 128 tokens (one token
// block, so one cluster holds the whole routing): after selection, CTA 0 of the
// cluster runs the one-CTA dispatch on the routing just written, and then every
// CTA of the cluster copies its share of the token rows into the expert-sorted
// order.  on = 0: router only.
struct RtcFuse {
    DispatchParams dp;
    const uint8_t *x;
    uint8_t *x_perm;
    int row_bytes;
    int on;
};

template <int EV, bool WF32>
__global__ void __launch_bounds__(RTC_THREADS, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mW,
                     const RouterParams p, uint64_t limit, const __grid_constant__ RtcFuse fz) {
    using C = RtcCfg<WF32>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t *empty = full + C::STAGES;
    uint64_t *tfull = empty + C::STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tfull + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *spbuf = reinterpret_cast<float *>(smem + C::STAGES * C::STAGE_BYTES + 256);
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
    // Accumulators: the 512 TMEM columns hold NA = 512 / ecols copies of the
    // 128 x E logit tile.  Consecutive k-blocks rotate over NH of them (so each
    // sums only every NH-th k-block), and for an fp32 W_g the two small bf16 parts
    // of the split go to NL accumulators of their own, away from the large part.
    // Every tensor-core accumulation step rounds at the magnitude of its
    // accumulator; fewer steps per accumulator keep the logits closer to the
    // exact sum.  The partials are added in a fixed order at the drain.
    const uint32_t ecols = E <= 32 ? 32 : E <= 64 ? 64 : E <= 128 ? 128 : 256;
    const uint32_t tmem_cols = 512;
    const int NA = 512 / (int)ecols;
    const int NH = WF32 ? NA / 2 : NA;
    const int NL = WF32 ? NA / 2 : 0;
    // Every CTA reads the same W_g slices; rotating the k-block order by the token
    // block spreads concurrent reads over different L2 lines.
    const int nkb = kb1 > kb0 ? kb1 - kb0 : 0;
    const int rot = nkb > 0 ? (int)(blockIdx.y % (unsigned)nkb) : 0;
    auto kb_of = [&](int i) { return kb0 + (i + rot < nkb ? i + rot : i + rot - nkb); };
    constexpr int NCONV = 6; // warps 2-7 split fp32 W_g

    const bool presplit = WF32 && p.wg_parts != nullptr; // the three parts come by TMA (mW)
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], WF32 && !presplit ? 1 + NCONV : 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tfull, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&mX);
        if (!WF32 || presplit) tma_prefetch_desc(&mW);
    }
    // Nothing above reads or writes global memory or TMEM, so it may overlap the
    // previous kernel of the stream (programmatic launch); everything below follows it.
    grid_dep_wait();
    grid_dep_launch_dependents();
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
                const int kb = kb_of(i);
                const uint32_t s = it % C::STAGES, ph = (it / C::STAGES) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, limit, abort_flag, 300)) { ok = false; break; }
                uint8_t *sa = ring + s * C::STAGE_BYTES;
                const uint32_t wbytes = (uint32_t)E * RTC_BK * 2;
                mbar_arrive_expect_tx(&full[s], RTC_A_BYTES + (!WF32 ? wbytes : presplit ? 3 * wbytes : 0u));
                tma_load_2d(&mX, &full[s], sa, kb * RTC_BK, t0);
                if (!WF32) tma_load_2d(&mW, &full[s], sa + RTC_A_BYTES, kb * RTC_BK, 0);
                if (presplit)
                    for (int part_i = 0; part_i < 3; ++part_i)
                        tma_load_2d(&mW, &full[s], sa + RTC_A_BYTES + part_i * C::B_PART, kb * RTC_BK,
                                    part_i * E);
            }
            if (!ok) {
                const uint32_t first = it > (uint32_t)C::STAGES ? it - C::STAGES : 0;
                for (uint32_t j = first; j < it; ++j) {
                    volatile int no_abort = 0;
                    mbar_wait(&full[j % C::STAGES], (j / C::STAGES) & 1, 10000000ull, &no_abort, 301);
                }
            }
        }
        __syncwarp(); // lanes 1-31 wait here for lane 0: the warp reconverges
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_bf16(RTC_BM, E);
            uint32_t it = 0;
            for (int i = 0; i < nkb; ++i, ++it) {
                const uint32_t s = it % C::STAGES, ph = (it / C::STAGES) & 1;
                if (!mbar_wait(&full[s], ph, limit, abort_flag, 310)) break;
                tc_fence_after();
                const uint32_t sa = smem_u32(ring + s * C::STAGE_BYTES);
                const uint32_t sb = sa + RTC_A_BYTES;
                const uint32_t dh = tmem_base + (uint32_t)(i % NH) * ecols;
                const bool first_h = i < NH;
#pragma unroll
                for (int kk = 0; kk < RTC_BK / 16; ++kk) {
                    umma_bf16_ss(dh, umma_desc_sw128(sa + kk * 32), umma_desc_sw128(sb + kk * 32),
                                 idesc, (!first_h || kk > 0) ? 1u : 0u);
                    if (WF32) {
                        const uint32_t dl = tmem_base + (uint32_t)(NH + (NL > 0 ? i % NL : 0)) * ecols;
                        const bool first_l = i < NL;
#pragma unroll
                        for (int part_i = 1; part_i < 3; ++part_i)
                            umma_bf16_ss(dl, umma_desc_sw128(sa + kk * 32),
                                         umma_desc_sw128(sb + part_i * C::B_PART + kk * 32), idesc,
                                         (!first_l || kk > 0 || part_i > 1) ? 1u : 0u);
                    }
                }
                umma_commit(&empty[s]);
            }
            umma_commit(tfull); // arrives once every MMA issued above has completed
        }
        __syncwarp();
    } else if (WF32 && !presplit) {
        // Split fp32 W_g into three bf16 tiles per stage (warps 2-7).  A thread owns
        // up to SPLIT_IT 8-float pieces of a k-block.  The next k-block's pieces are
        // loaded into registers while the current ones are split and stored, so the
        // load latency is paid once per k-block rather than once per piece.
        constexpr int SPLIT_IT = (RTC_MAXE_F32 * 8 + NCONV * 32 - 1) / (NCONV * 32);
        const int cw = warp - 2, ct = cw * 32 + lane;
        const float *W = static_cast<const float *>(p.W_g);
        float4 ru[SPLIT_IT], rv[SPLIT_IT];
        auto fetch = [&](int kb) {
            const int k0 = kb * RTC_BK;
#pragma unroll
            for (int j = 0; j < SPLIT_IT; ++j) {
                const int item = ct + j * NCONV * 32;
                ru[j] = make_float4(0.f, 0.f, 0.f, 0.f);
                rv[j] = ru[j];
                if (item < E * 8) {
                    const int row = item >> 3, kk = k0 + (item & 7) * 8;
                    const float *src = W + (size_t)row * p.D + kk;
                    if (kk + 8 <= p.D) {
                        ru[j] = __ldg(reinterpret_cast<const float4 *>(src));
                        rv[j] = __ldg(reinterpret_cast<const float4 *>(src) + 1);
                    } else {
                        float t[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q) t[q] = kk + q < p.D ? src[q] : 0.f;
                        ru[j] = make_float4(t[0], t[1], t[2], t[3]);
                        rv[j] = make_float4(t[4], t[5], t[6], t[7]);
                    }
                }
            }
        };
        if (nkb > 0) fetch(kb_of(0));
        uint32_t it = 0;
        for (int i = 0; i < nkb; ++i, ++it) {
            const uint32_t s = it % C::STAGES, ph = (it / C::STAGES) & 1;
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&empty[s], ph ^ 1, limit, abort_flag, 330);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            uint8_t *b0 = ring + s * C::STAGE_BYTES + RTC_A_BYTES;
#pragma unroll
            for (int j = 0; j < SPLIT_IT; ++j) {
                const int item = ct + j * NCONV * 32;
                if (item < E * 8) split_store(b0, item >> 3, item & 7, ru[j], rv[j], C::B_PART);
            }
            fence_proxy_async_smem(); // generic-proxy stores -> visible to the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[s]);
            if (i + 1 < nkb) fetch(kb_of(i + 1));
        }
        __syncwarp();
    }
    if (warp >= 4) {
        // Drain the accumulator: TMEM lane = token row, column = expert.
        const int q = warp & 3;
        const int row = q * 32 + lane;
        bool have = false;
        if (lane == 0) have = mbar_wait(tfull, 0, limit, abort_flag, 320);
        have = __shfl_sync(0xffffffffu, have ? 1 : 0, 0) != 0;
        __syncwarp();
        if (have) tc_fence_after();
        // Accumulators written by this CTA (a CTA with fewer k-blocks than NH leaves
        // the others untouched); summed in a fixed order: large parts, then small.
        const int nh = nkb < NH ? nkb : NH;
        const int nl = nkb < NL ? nkb : NL;
        const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
        for (int c0 = 0; c0 < E; c0 += 32) {
            float hi[32], lo[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) hi[i] = lo[i] = 0.f;
            if (have) {
                for (int h = 0; h < nh; ++h) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(lane_base + (uint32_t)h * ecols + c0, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) hi[i] = h ? hi[i] + __uint_as_float(v[i]) : __uint_as_float(v[i]);
                }
                for (int l = 0; l < nl; ++l) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(lane_base + (uint32_t)(NH + l) * ecols + c0, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) lo[i] = l ? lo[i] + __uint_as_float(v[i]) : __uint_as_float(v[i]);
                }
            }
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (c0 + i < E) part[row * RTC_PART_LD + c0 + i] = have ? hi[i] + lo[i] : 0.f;
        }
    }
    tc_fence_before();
    cluster.sync();

    // ---- sum the cluster's partial logits and select: one warp per token -------
    // Token j of the block goes to CTA j % CLK, so a small batch spreads over the
    // whole cluster.  A lane loads the partials of its experts from every CTA of
    // the cluster before it adds any (all of them when CLK <= 4, else VB expert
    // slots x CLK ranks at a time), and adds them in rank order (deterministic).
    constexpr int VB = EV < 4 ? EV : 4;
    float bv[EV];
    load_bias<EV>(p, lane, bv);
    for (int jl = warp; rank + CLK * jl < RTC_BM; jl += RTC_THREADS / 32) {
        const int j = rank + CLK * jl;
        const int t = t0 + j;
        if (t >= p.N) break;
        float logit[EV];
        if (CLK <= 4) {
            float pv[EV][4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float *src = c < CLK ? cluster.map_shared_rank(part, c) + j * RTC_PART_LD : nullptr;
#pragma unroll
                for (int v = 0; v < EV; ++v) {
                    const int e = lane + 32 * v;
                    pv[v][c] = (c < CLK && e < E) ? src[e] : 0.f;
                }
            }
#pragma unroll
            for (int v = 0; v < EV; ++v) {
                float r = 0.f;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (c < CLK) r += pv[v][c];
                logit[v] = r;
            }
        } else {
#pragma unroll
            for (int v0 = 0; v0 < EV; v0 += VB) {
                float pv[VB][RTC_MAX_CLK];
#pragma unroll
                for (int c = 0; c < RTC_MAX_CLK; ++c) {
                    const float *src = c < CLK ? cluster.map_shared_rank(part, c) + j * RTC_PART_LD : nullptr;
#pragma unroll
                    for (int v = 0; v < VB; ++v) {
                        const int e = lane + 32 * (v0 + v);
                        pv[v][c] = (c < CLK && e < E) ? src[e] : 0.f;
                    }
                }
#pragma unroll
                for (int v = 0; v < VB; ++v) {
                    float r = 0.f;
#pragma unroll
                    for (int c = 0; c < RTC_MAX_CLK; ++c)
                        if (c < CLK) r += pv[v][c];
                    logit[v0 + v] = r;
                }
            }
        }
        router_select<EV>(p, t, logit, bv, spbuf + warp * ROUTER_MAXV * 32, lane);
    }
    cluster.sync(); // partials stay alive until every reader is done
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols);
    }
    if (fz.on) {
        // The routing of all tokens is in global memory and visible to the whole
        // cluster after the barrier above; the operand ring is free.
        static_assert(RTC_THREADS / 32 * DISPATCH_MAXE * 4 + 3 * DISPATCH_MAXE * 4 <=
                          RtcCfg<WF32>::STAGES * RtcCfg<WF32>::STAGE_BYTES,
                      "dispatch arrays fit the ring");
        if (rank == 0) {
            int *hist = reinterpret_cast<int *>(ring);
            int *cursor = hist + DISPATCH_MAXE;
            int *wsum = cursor + DISPATCH_MAXE;
            auto wcnt = reinterpret_cast<int(*)[DISPATCH_MAXE]>(wsum + DISPATCH_MAXE);
            dispatch_small_body<RTC_THREADS>(fz.dp, hist, cursor, wcnt, wsum);
        }
        cluster.sync(); // positions visible to every CTA of the cluster
        gather_items(fz.x, fz.x_perm, fz.dp, fz.row_bytes, rank * (RTC_THREADS / 32) + warp,
                     CLK * (RTC_THREADS / 32));
    }
}

}  // namespace moe
