// Router: fp32 logits, sigmoid, correction bias, group top-2 score, group keep,
// top-k and weights ("GLM-4.5 Group Router", How it works).
//
// One thread-block cluster of ROUTER_CL CTAs handles 32 tokens.  CTA r of the
// cluster computes partial logits of all E experts for those tokens over the
// r-th slice of the hidden dimension D, on CUDA cores in fp32 (bf16 and fp32
// inputs are widened exactly, so every product is exact in fp32), and keeps the
// 32 x E partial tile in its shared memory.  After a cluster barrier, warp w of
// CTA r takes token j = r + ROUTER_CL * w: lane l sums expert l, l+32, ...
// over the ROUTER_CL partial tiles in rank order (distributed shared memory, a
// fixed order, so the result is deterministic) and selection then runs in the
// warp's registers with shuffles.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace moe {

namespace cg = cooperative_groups;

constexpr int ROUTER_TM = 32;        // tokens per cluster
constexpr int ROUTER_CL = 8;         // CTAs per cluster = K slices
constexpr int ROUTER_KC = 32;        // K chunk staged in shared memory
constexpr int ROUTER_THREADS = 256;  // 8 warps
constexpr int ROUTER_MAXV = 16;      // experts per lane: E <= 512
constexpr int ROUTER_MAXG = 64;      // groups

struct RouterParams {
    const void *x;
    const void *W_g;
    const float *b;
    int N, D, E, G, tg, k, norm;
    float alpha;
    int32_t *topk_idx;
    float *topk_w;
    // fp32 W_g already split into three bf16 parts [3][E][D] (null: the tensor-core
    // router splits it itself, per token block)
    const void *wg_parts;
    // Test hook (null on the hot path): receives every token's fp32 selection
    // scores s' = sigmoid(r) + b [N][E], before any group masking.
    float *dbg_sp;
};

// Dynamic shared memory of router_kernel<EV>: x chunk, W chunk, partial logits,
// per-warp s' rows for the group stage.
__host__ __device__ constexpr int router_smem_bytes(int EV) {
    return (ROUTER_TM * (ROUTER_KC + 1) + 32 * EV * (ROUTER_KC + 1) + ROUTER_TM * 32 * EV +
            (ROUTER_THREADS / 32) * ROUTER_MAXV * 32) * 4;
}

// Unsigned key with the order of the floats: a larger float has a larger key
// (-inf included, -0 equal to +0); NaN maps to 0, below every number, so it is
// never preferred to a number.
__device__ __forceinline__ uint32_t order_key(float v) {
    if (v != v) return 0u;
    const uint32_t b = __float_as_uint(v == 0.f ? 0.f : v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Warp-wide pick of the best (key, id) pair: the largest key, and among the lanes
// holding it the smallest id.  Lanes with nothing to offer pass key 0 and id
// 0xffffffff.  Two redux.sync reductions instead of a shuffle butterfly.
__device__ __forceinline__ uint32_t warp_pick(uint32_t key, uint32_t id) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, key);
    return __reduce_min_sync(0xffffffffu, key == m ? id : 0xffffffffu);
}

// The float of an order_key (key 0, a NaN's, reads as -inf: never preferred).
__device__ __forceinline__ float key_value(uint32_t key) {
    if (key == 0u) return -INFINITY;
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Each lane's correction bias for its experts lane, lane + 32, ... (0 past E),
// loaded once per warp before its tokens.
template <int EV>
__device__ __forceinline__ void load_bias(const RouterParams &p, int lane, float (&bv)[EV]) {
#pragma unroll
    for (int v = 0; v < EV; ++v) {
        const int e = lane + 32 * v;
        bv[v] = e < p.E ? p.b[e] : 0.f;
    }
}

// Selection for one token by one warp ("GLM-4.5 Group Router", How it works):
// lane l holds the fp32 logits of experts l, l+32, ...  s = sigmoid(r),
// s' = s + b; with n_group > 1 a group scores the sum of its two largest s' and
// the topk_group best groups are kept (others are -inf); the k largest s' among
// the kept experts are chosen (ties to the lower id) and their weights are
// alpha * s / (sum of the chosen s + 1e-20), or alpha * s without normalisation.
// sp_w is a per-warp scratch row of 32 * ROUTER_MAXV floats in shared memory; bv
// the lane's bias values (load_bias).
template <int EV>
__device__ __forceinline__ void router_select(const RouterParams &p, int t, const float (&logit)[EV],
                                              const float (&bv)[EV], float *sp_w, int lane) {
    const int E = p.E, G = p.G, m = E / G;
    float s[EV], sp[EV];
#pragma unroll
    for (int v = 0; v < EV; ++v) {
        const int e = lane + 32 * v;
        s[v] = 0.f;
        sp[v] = -INFINITY;
        if (e < E) {
            s[v] = 1.0f / (1.0f + expf(-logit[v]));
            sp[v] = s[v] + bv[v];
            if (p.dbg_sp) p.dbg_sp[(size_t)t * E + e] = sp[v];
        }
    }
    // Candidate mask over this lane's experts (bit v).
    uint32_t cand = 0;
    if (G > 1 && m == 32 && E % 32 == 0) {
        // Group g is exactly the slot v = g of every lane: its two largest s'
        // (equal values both count) by warp reductions on order keys, in
        // registers.  The same values as the scan below, so the same sum.
        float gs[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int g = 0; g < EV; ++g) {
            if (g < G) {
                const uint32_t k1 = order_key(sp[g]);
                const uint32_t m1 = __reduce_max_sync(0xffffffffu, k1);
                const uint32_t holder = __reduce_min_sync(0xffffffffu, k1 == m1 ? (uint32_t)lane : 32u);
                const uint32_t m2 = __reduce_max_sync(0xffffffffu, (uint32_t)lane == holder ? 0u : k1);
                const float score = key_value(m1) + key_value(m2);
                if (lane == g) gs[0] = score;
            }
        }
        uint64_t kept = 0;
        const uint32_t gk = order_key(gs[0]);
        for (int r = 0; r < p.tg; ++r) {
            const bool mine = lane < G && !((kept >> lane) & 1ull);
            const uint32_t win = warp_pick(mine ? gk : 0u, mine ? (uint32_t)lane : 0xffffffffu);
            if (win < 64u) kept |= 1ull << win;
        }
#pragma unroll
        for (int v = 0; v < EV; ++v)
            if (lane + 32 * v < E && ((kept >> v) & 1ull)) cand |= 1u << v;
    } else if (G > 1) {
#pragma unroll
        for (int v = 0; v < EV; ++v)
            if (lane + 32 * v < E) sp_w[lane + 32 * v] = sp[v];
        __syncwarp();
        // Group score = sum of the two largest s' of the group (lanes own g, g+32).
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
        const uint32_t gk[2] = {order_key(gs[0]), order_key(gs[1])};
        for (int r = 0; r < p.tg; ++r) {
            uint32_t bk = 0, bi = 0xffffffffu;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int g = lane + 32 * h;
                if (g < G && !((kept >> g) & 1ull) && (bi == 0xffffffffu || gk[h] > bk)) {
                    bk = gk[h];
                    bi = g;
                }
            }
            const uint32_t win = warp_pick(bk, bi);
            if (win < 64u) kept |= 1ull << win;
        }
#pragma unroll
        for (int v = 0; v < EV; ++v) {
            const int e = lane + 32 * v;
            if (e < E && ((kept >> (e / m)) & 1ull)) cand |= 1u << v;
        }
    } else {
#pragma unroll
        for (int v = 0; v < EV; ++v)
            if (lane + 32 * v < E) cand |= 1u << v;
    }
    // Top-k by s' among candidates; lane r keeps the r-th pick.  A lane's own
    // experts rise with v, so its first maximal key is its smallest id.
    uint32_t key[EV];
#pragma unroll
    for (int v = 0; v < EV; ++v) key[v] = order_key(sp[v]);
    int my_e = -1;
    float my_s = 0.f;
    for (int r = 0; r < p.k; ++r) {
        uint32_t bk = 0, bi = 0xffffffffu;
#pragma unroll
        for (int v = 0; v < EV; ++v) {
            if (((cand >> v) & 1u) && (bi == 0xffffffffu || key[v] > bk)) {
                bk = key[v];
                bi = lane + 32 * v;
            }
        }
        const int win = (int)warp_pick(bk, bi);
        const int owner = win & 31, vw = win >> 5;
        float sv = 0.f;
#pragma unroll
        for (int v = 0; v < EV; ++v)
            if (v == vw) sv = s[v];
        sv = __shfl_sync(0xffffffffu, sv, owner);
        if (lane == owner) cand &= ~(1u << vw);
        if (lane == r) {
            my_e = win;
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

// One step of the loss-free balancer ("GLM-4.5 Group Router", How it works: the
// bias is updated from expert load during training, at rate 0.001, then 0).  The
// rule is the plainest reading of the loss-free balancing the page cites: every
// expert's bias moves by `rate` towards the mean load, b_e += rate * sign(mean -
// load_e), the comparison made exactly in integers (total - E * load_e).  Loads
// count the routed (token, slot) pairs; the sentinel E counts for nobody, other
// out-of-range ids are reported.  One CTA of BIAS_THREADS threads, E <= 512.
constexpr int BIAS_THREADS = 512;

__global__ void __launch_bounds__(BIAS_THREADS)
    bias_update_kernel(const int32_t *topk_idx, int n_ids, int E, float rate, float *b,
                       int32_t *loads_out) {
    __shared__ int hist[512];
    __shared__ long long total;
    for (int e = threadIdx.x; e < E; e += BIAS_THREADS) hist[e] = 0;
    if (threadIdx.x == 0) total = 0;
    __syncthreads();
    int mine = 0;
    for (int i = threadIdx.x; i < n_ids; i += BIAS_THREADS) {
        const int e = topk_idx[i];
        if (e >= 0 && e < E) {
            atomicAdd(&hist[e], 1);
            ++mine;
        } else if (e != E) {
            record_error(DEV_BAD_INDEX, 12);
        }
    }
    atomicAdd(reinterpret_cast<unsigned long long *>(&total), (unsigned long long)mine);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += BIAS_THREADS) {
        const long long diff = total - (long long)E * hist[e];
        const float step = diff > 0 ? rate : (diff < 0 ? -rate : 0.f);
        b[e] = b[e] + step;
        if (loads_out) loads_out[e] = hist[e];
    }
}

// EV = experts per lane (E <= 32 * EV); each thread accumulates 4 tokens x EV experts.
template <typename XT, typename WT, int EV>
__global__ void __launch_bounds__(ROUTER_THREADS)
    router_kernel(const RouterParams p) {
    extern __shared__ float rsm[];
    float(*xs)[ROUTER_KC + 1] = reinterpret_cast<float(*)[ROUTER_KC + 1]>(rsm);
    float(*ws)[ROUTER_KC + 1] =
        reinterpret_cast<float(*)[ROUTER_KC + 1]>(rsm + ROUTER_TM * (ROUTER_KC + 1));
    float *part = rsm + ROUTER_TM * (ROUTER_KC + 1) + 32 * EV * (ROUTER_KC + 1); // [TM][32*EV]
    float *spbuf = part + ROUTER_TM * 32 * EV; // [8 warps][MAXV*32]
    constexpr int EP = 32 * EV;                // padded expert count

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = blockIdx.x;
    const int t0 = blockIdx.y * ROUTER_TM;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = p.E;

    // K slice of this CTA (a multiple of the chunk size).
    const int kper = ((p.D + ROUTER_CL * ROUTER_KC - 1) / (ROUTER_CL * ROUTER_KC)) * ROUTER_KC;
    const int kbeg = rank * kper, kend = min(p.D, kbeg + kper);

    const XT *x = static_cast<const XT *>(p.x);
    const WT *W = static_cast<const WT *>(p.W_g);

    // ---- partial logits [32 tokens x E] over [kbeg, kend) ----------------------
    // thread: tokens warp + 8*i (i < 4), experts lane + 32*j (j < EV)
    float acc[4][EV];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < EV; ++j) acc[i][j] = 0.f;

    // Register-staged double buffering: the next chunk's loads are in flight
    // while the current chunk is multiplied out of shared memory.
    constexpr int XPT = ROUTER_TM * ROUTER_KC / ROUTER_THREADS; // 4
    constexpr int WPT = EP * ROUTER_KC / ROUTER_THREADS;        // 4 * EV
    float xr[XPT], wr[WPT];
    auto load_chunk = [&](int k0) {
#pragma unroll
        for (int q = 0; q < XPT; ++q) {
            const int i = tid + ROUTER_THREADS * q;
            const int r = i / ROUTER_KC, c = i % ROUTER_KC;
            const int t = t0 + r, kk = k0 + c;
            xr[q] = (t < p.N && kk < kend) ? to_f32(x[(size_t)t * p.D + kk]) : 0.f;
        }
#pragma unroll
        for (int q = 0; q < WPT; ++q) {
            const int i = tid + ROUTER_THREADS * q;
            const int r = i / ROUTER_KC, c = i % ROUTER_KC;
            const int kk = k0 + c;
            wr[q] = (r < E && kk < kend) ? to_f32(W[(size_t)r * p.D + kk]) : 0.f;
        }
    };
    // Clusters of different token blocks read the same W_g columns; rotating the
    // chunk order by the token block keeps them on different L2 lines.
    const int nch = kend > kbeg ? (kend - kbeg + ROUTER_KC - 1) / ROUTER_KC : 0;
    const int rot = nch > 0 ? (int)(blockIdx.y % (unsigned)nch) : 0;
    auto chunk_k0 = [&](int i) {
        const int c = i + rot < nch ? i + rot : i + rot - nch;
        return kbeg + c * ROUTER_KC;
    };
    if (nch > 0) load_chunk(chunk_k0(0));
    for (int ci = 0; ci < nch; ++ci) {
#pragma unroll
        for (int q = 0; q < XPT; ++q) {
            const int i = tid + ROUTER_THREADS * q;
            xs[i / ROUTER_KC][i % ROUTER_KC] = xr[q];
        }
#pragma unroll
        for (int q = 0; q < WPT; ++q) {
            const int i = tid + ROUTER_THREADS * q;
            ws[i / ROUTER_KC][i % ROUTER_KC] = wr[q];
        }
        __syncthreads();
        if (ci + 1 < nch) load_chunk(chunk_k0(ci + 1));
#pragma unroll 4
        for (int kk = 0; kk < ROUTER_KC; ++kk) {
            float a[4], w[EV];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = xs[warp + 8 * i][kk];
#pragma unroll
            for (int j = 0; j < EV; ++j) w[j] = ws[lane + 32 * j][kk];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < EV; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < EV; ++j) part[(warp + 8 * i) * EP + lane + 32 * j] = acc[i][j];
    cluster.sync();

    // ---- reduce over the cluster's K slices, then select: one warp per token ----
    const int j = rank + ROUTER_CL * warp; // token of this warp (32 = CL * 4 tokens per cluster)
    const int t = t0 + j;
    if (warp < ROUTER_TM / ROUTER_CL && t < p.N) {
        float bv[EV];
        load_bias<EV>(p, lane, bv);
        float logit[EV];
#pragma unroll
        for (int v = 0; v < EV; ++v) {
            const int e = lane + 32 * v;
            float r = 0.f;
            if (e < E) {
#pragma unroll
                for (int c = 0; c < ROUTER_CL; ++c) {
                    const float *remote = cluster.map_shared_rank(part, c);
                    r += remote[j * EP + e];
                }
            }
            logit[v] = r;
        }
        router_select<EV>(p, t, logit, bv, spbuf + warp * ROUTER_MAXV * 32, lane);
    }
    cluster.sync(); // keep this CTA's partials alive until every reader is done
}

}  // namespace moe
