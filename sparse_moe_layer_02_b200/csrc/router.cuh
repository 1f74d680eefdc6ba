// Router: fp32 logits, sigmoid, correction bias, group top-2 score, group keep,
// top-k and weights ("GLM-4.5 Group Router", How it works).
//
// One thread-block cluster handles 32 tokens.  CTA r of the cluster computes the
// logits of experts [r*TE, r*TE + TE) for those tokens on CUDA cores (fp32 FMA;
// bf16 and fp32 inputs are widened exactly, so every product is exact in fp32)
// and keeps them in its shared memory.  After a cluster barrier each warp takes
// whole tokens and reads the token's E logits from all CTAs of the cluster
// through distributed shared memory; selection then runs in the warp's
// registers with shuffles: lane l holds experts l, l+32, l+64, ...
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace moe {

namespace cg = cooperative_groups;

constexpr int ROUTER_TM = 32;       // tokens per cluster
constexpr int ROUTER_KC = 32;       // K chunk staged in shared memory
constexpr int ROUTER_THREADS = 128; // 4 warps
constexpr int ROUTER_MAXV = 16;     // experts per lane: E <= 512
constexpr int ROUTER_MAXG = 64;     // groups

struct RouterParams {
    const void *x;
    const void *W_g;
    const float *b;
    int N, D, E, G, tg, k, norm;
    float alpha;
    int32_t *topk_idx;
    float *topk_w;
};

// (value, index) comparison: larger value wins, ties go to the lower index.
__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
    return v > bv || (v == bv && i < bi);
}

__device__ __forceinline__ void warp_argmax(float &v, int &i) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        float ov = __shfl_xor_sync(0xffffffffu, v, off);
        int oi = __shfl_xor_sync(0xffffffffu, i, off);
        if (better(ov, oi, v, i)) {
            v = ov;
            i = oi;
        }
    }
}

template <typename XT, typename WT, int TE>
__global__ void __launch_bounds__(ROUTER_THREADS)
    router_kernel(const RouterParams p) {
    constexpr int EPT = TE / 8; // experts per thread in the logits tile
    __shared__ float xs[ROUTER_TM][ROUTER_KC + 1];
    __shared__ float ws[TE][ROUTER_KC + 1];
    __shared__ float logit[ROUTER_TM][TE];
    __shared__ float spbuf[4][ROUTER_MAXV * 32];

    cg::cluster_group cluster = cg::this_cluster();
    const int CL = gridDim.x;
    const int rank = blockIdx.x;
    const int t0 = blockIdx.y * ROUTER_TM;
    const int e0 = rank * TE;
    const int tid = threadIdx.x;
    const int ty = tid >> 3, tx = tid & 7;

    const XT *x = static_cast<const XT *>(p.x);
    const WT *W = static_cast<const WT *>(p.W_g);

    // ---- logits tile [32 tokens x TE experts], fp32 accumulation -------------
    float acc0[EPT], acc1[EPT];
#pragma unroll
    for (int j = 0; j < EPT; ++j) acc0[j] = acc1[j] = 0.f;

    for (int k0 = 0; k0 < p.D; k0 += ROUTER_KC) {
        for (int i = tid; i < ROUTER_TM * ROUTER_KC; i += ROUTER_THREADS) {
            const int r = i / ROUTER_KC, c = i % ROUTER_KC;
            const int t = t0 + r, kk = k0 + c;
            xs[r][c] = (t < p.N && kk < p.D) ? to_f32(x[(size_t)t * p.D + kk]) : 0.f;
        }
        for (int i = tid; i < TE * ROUTER_KC; i += ROUTER_THREADS) {
            const int r = i / ROUTER_KC, c = i % ROUTER_KC;
            const int e = e0 + r, kk = k0 + c;
            ws[r][c] = (e < p.E && kk < p.D) ? to_f32(W[(size_t)e * p.D + kk]) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < ROUTER_KC; ++kk) {
            const float a0 = xs[ty][kk], a1 = xs[ty + 16][kk];
#pragma unroll
            for (int j = 0; j < EPT; ++j) {
                const float w = ws[tx + 8 * j][kk];
                acc0[j] = fmaf(a0, w, acc0[j]);
                acc1[j] = fmaf(a1, w, acc1[j]);
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
        logit[ty][tx + 8 * j] = acc0[j];
        logit[ty + 16][tx + 8 * j] = acc1[j];
    }
    cluster.sync();

    // ---- selection: one warp per token --------------------------------------
    const int warp = tid >> 5, lane = tid & 31;
    const int E = p.E, G = p.G, m = E / G;
    const int V = (E + 31) >> 5;
    float *sp_w = spbuf[warp];
    for (int j = rank + CL * warp; j < ROUTER_TM; j += CL * 4) {
        const int t = t0 + j;
        if (t >= p.N) break;
        float s[ROUTER_MAXV], sp[ROUTER_MAXV];
#pragma unroll
        for (int v = 0; v < ROUTER_MAXV; ++v) {
            const int e = lane + 32 * v;
            s[v] = 0.f;
            sp[v] = -INFINITY;
            if (v < V && e < E) {
                const float *remote = cluster.map_shared_rank(&logit[0][0], e / TE);
                const float r = remote[j * TE + (e % TE)];
                s[v] = 1.0f / (1.0f + expf(-r));
                sp[v] = s[v] + p.b[e];
            }
        }
        // Candidate mask over this lane's experts (bit v).
        uint32_t cand = 0;
        if (G > 1) {
#pragma unroll
            for (int v = 0; v < ROUTER_MAXV; ++v)
                if (v < V && lane + 32 * v < E) sp_w[lane + 32 * v] = sp[v];
            __syncwarp();
            // Group score = sum of the two largest s' of the group (lane g, g+32).
            float gs[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int g = lane + 32 * h;
                if (g < G) {
                    float b1 = -INFINITY, b2 = -INFINITY;
                    for (int q = g * m; q < (g + 1) * m; ++q) {
                        const float v = sp_w[q];
                        if (v > b1) {
                            b2 = b1;
                            b1 = v;
                        } else if (v > b2) {
                            b2 = v;
                        }
                    }
                    gs[h] = b1 + b2;
                }
            }
            __syncwarp();
            uint64_t kept = 0;
            for (int r = 0; r < p.tg; ++r) {
                float bv = -INFINITY;
                int bi = 0x7fffffff;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int g = lane + 32 * h;
                    if (g < G && !((kept >> g) & 1ull) && better(gs[h], g, bv, bi)) {
                        bv = gs[h];
                        bi = g;
                    }
                }
                warp_argmax(bv, bi);
                kept |= 1ull << bi;
            }
#pragma unroll
            for (int v = 0; v < ROUTER_MAXV; ++v) {
                const int e = lane + 32 * v;
                if (v < V && e < E && ((kept >> (e / m)) & 1ull)) cand |= 1u << v;
            }
        } else {
#pragma unroll
            for (int v = 0; v < ROUTER_MAXV; ++v)
                if (v < V && lane + 32 * v < E) cand |= 1u << v;
        }
        // Top-k by s' among candidates; lane r keeps the r-th pick.
        int my_e = -1;
        float my_s = 0.f;
        for (int r = 0; r < p.k; ++r) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int v = 0; v < ROUTER_MAXV; ++v) {
                if ((cand >> v) & 1u) {
                    const int e = lane + 32 * v;
                    if (better(sp[v], e, bv, bi)) {
                        bv = sp[v];
                        bi = e;
                    }
                }
            }
            warp_argmax(bv, bi);
            const int owner = bi & 31, vw = bi >> 5;
            float sv = 0.f;
#pragma unroll
            for (int v = 0; v < ROUTER_MAXV; ++v)
                if (v == vw) sv = s[v];
            sv = __shfl_sync(0xffffffffu, sv, owner);
            if (lane == owner) cand &= ~(1u << vw);
            if (lane == r) {
                my_e = bi;
                my_s = sv;
            }
        }
        // Weights from the raw scores of the chosen set.
        float sum = (lane < p.k) ? my_s : 0.f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane < p.k) {
            const float w = p.norm ? p.alpha * my_s / (sum + 1e-20f) : p.alpha * my_s;
            p.topk_idx[(size_t)t * p.k + lane] = my_e;
            p.topk_w[(size_t)t * p.k + lane] = w;
        }
    }
    cluster.sync(); // keep this CTA's logits alive until every reader is done
}

}  // namespace moe
