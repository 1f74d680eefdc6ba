// fp32 expert path on CUDA cores (no TF32: fp32 products and fp32 accumulation),
// for fp32 layers such as the tiny fully-fp32 configuration.  Same dispatch and
// same arithmetic as the tensor-core path ("GLM-4.5 MoE Forward", How it works):
//   gate_up  h[r, c]  = SiLU(x_r . W_gate[c]) * (x_r . W_up[c])   (fp32 h, optional limits)
//   down     slot[r]  = w_r * (h_r . W_down rows)                 (fp32 slot)
//            y[n]     = (h_sh . W_sh_down rows)                    (shared, into y)
//   combine  y[n]    <- sum_j slot[pos(n, j)] + y[n]               (slot order)
#pragma once

#include "common.cuh"

namespace moe {

constexpr int SIMT_T = 32;  // rows x cols per block
constexpr int SIMT_KC = 32; // K chunk

enum SimtMode { SIMT_GATEUP_R = 0, SIMT_GATEUP_S = 1, SIMT_DOWN_R = 2, SIMT_DOWN_S = 3 };

struct SimtArgs {
    const float *x, *gate_up, *down, *sh_gate, *sh_up, *sh_down;
    const int32_t *perm_tok, *counts, *tile_off, *meta, *pos_of;
    const float *w_perm;
    float *h_perm, *h_sh, *slot, *y;
    int N, D, E, d, d_sh, k;
    float gate_max, up_max; // SwiGLU limits (+infinity = plain SwiGLU)
};

__device__ __forceinline__ int expert_of_row(const int32_t *tile_off, int E, int row) {
    const int mt = row / 128;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tile_off[mid] <= mt) lo = mid; else hi = mid - 1;
    }
    return lo;
}

template <int MODE>
__global__ void __launch_bounds__(256) simt_expert_kernel(const SimtArgs a) {
    constexpr bool GATEUP = (MODE == SIMT_GATEUP_R || MODE == SIMT_GATEUP_S);
    constexpr bool ROUTED = (MODE == SIMT_GATEUP_R || MODE == SIMT_DOWN_R);
    __shared__ float As[SIMT_T][SIMT_KC + 1];
    __shared__ float B0[SIMT_T][SIMT_KC + 1];
    __shared__ float B1[GATEUP ? SIMT_T : 1][SIMT_KC + 1];

    const int r0 = blockIdx.x * SIMT_T, c0 = blockIdx.y * SIMT_T;
    const int rows = ROUTED ? a.meta[1] : a.N;
    if (r0 >= rows) return;
    const int ncols = GATEUP ? (ROUTED ? a.d : a.d_sh) : a.D;
    const int K = GATEUP ? a.D : (ROUTED ? a.d : a.d_sh);
    const int e = ROUTED ? expert_of_row(a.tile_off, a.E, r0) : 0;
    // Rows of expert e at or beyond seg_end are padding (no token).
    const int seg_end = ROUTED ? a.tile_off[e] * 128 + a.counts[e] : rows;

    // A rows and B matrices of this block.
    const float *Bm0, *Bm1 = nullptr;
    if (MODE == SIMT_GATEUP_R) {
        Bm0 = a.gate_up + (size_t)e * 2 * a.d * a.D;
        Bm1 = Bm0 + (size_t)a.d * a.D;
    } else if (MODE == SIMT_GATEUP_S) {
        Bm0 = a.sh_gate;
        Bm1 = a.sh_up;
    } else if (MODE == SIMT_DOWN_R) {
        Bm0 = a.down + (size_t)e * a.D * a.d;
    } else {
        Bm0 = a.sh_down;
    }

    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    float g[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, u[2][2] = {{0.f, 0.f}, {0.f, 0.f}};

    for (int k0 = 0; k0 < K; k0 += SIMT_KC) {
        for (int i = tid; i < SIMT_T * SIMT_KC; i += 256) {
            const int r = i / SIMT_KC, kk = i % SIMT_KC;
            const int gr = r0 + r, gk = k0 + kk;
            float av = 0.f;
            if (gr < rows && gk < K) {
                if (MODE == SIMT_GATEUP_R) {
                    av = gr < seg_end ? a.x[(size_t)a.perm_tok[gr] * a.D + gk] : 0.f;
                } else if (MODE == SIMT_GATEUP_S) {
                    av = a.x[(size_t)gr * a.D + gk];
                } else if (MODE == SIMT_DOWN_R) {
                    av = a.h_perm[(size_t)gr * a.d + gk];
                } else {
                    av = a.h_sh[(size_t)gr * a.d_sh + gk];
                }
            }
            As[r][kk] = av;
            const int gc = c0 + r;
            const bool bok = gc < ncols && gk < K;
            B0[r][kk] = bok ? Bm0[(size_t)gc * K + gk] : 0.f;
            if (GATEUP) B1[r][kk] = bok ? Bm1[(size_t)gc * K + gk] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < SIMT_KC; ++kk) {
            const float a0 = As[ty][kk], a1 = As[ty + 16][kk];
            const float b0 = B0[tx][kk], b1 = B0[tx + 16][kk];
            g[0][0] = fmaf(a0, b0, g[0][0]);
            g[0][1] = fmaf(a0, b1, g[0][1]);
            g[1][0] = fmaf(a1, b0, g[1][0]);
            g[1][1] = fmaf(a1, b1, g[1][1]);
            if (GATEUP) {
                const float v0 = B1[tx][kk], v1 = B1[tx + 16][kk];
                u[0][0] = fmaf(a0, v0, u[0][0]);
                u[0][1] = fmaf(a0, v1, u[0][1]);
                u[1][0] = fmaf(a1, v0, u[1][0]);
                u[1][1] = fmaf(a1, v1, u[1][1]);
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r = r0 + ty + 16 * i;
        if (r >= rows) continue;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int c = c0 + tx + 16 * j;
            if (c >= ncols) continue;
            if (MODE == SIMT_GATEUP_R) {
                a.h_perm[(size_t)r * a.d + c] = swiglu_f(g[i][j], u[i][j], a.gate_max, a.up_max);
            } else if (MODE == SIMT_GATEUP_S) {
                a.h_sh[(size_t)r * a.d_sh + c] = swiglu_f(g[i][j], u[i][j], a.gate_max, a.up_max);
            } else if (MODE == SIMT_DOWN_R) {
                if (r < seg_end) a.slot[(size_t)r * a.D + c] = a.w_perm[r] * g[i][j];
            } else {
                a.y[(size_t)r * a.D + c] = g[i][j];
            }
        }
    }
}

// y[n, c] = (sum over slots j in order of slot[pos(n, j), c]) + y[n, c].
__global__ void __launch_bounds__(256) simt_combine_kernel(const SimtArgs a) {
    const size_t total = (size_t)a.N * a.D;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (size_t)gridDim.x * blockDim.x) {
        const int n = (int)(i / a.D), c = (int)(i % a.D);
        float s = 0.f;
        for (int j = 0; j < a.k; ++j) {
            const int p = a.pos_of[(size_t)n * a.k + j];
            if (p >= 0) s += a.slot[(size_t)p * a.D + c];
        }
        a.y[i] = s + a.y[i];
    }
}

}  // namespace moe
