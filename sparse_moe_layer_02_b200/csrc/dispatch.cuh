// Token dispatch ("GLM-4.5 MoE Forward", How it works: token-choice dispatch,
// every token goes to exactly its k routed experts; an id equal to E is the
// sentinel of the GLM-5 experts' forward and goes nowhere).
//
// The N*k (token, slot) pairs are sorted by (expert, token, slot) into
// expert-contiguous segments, each padded to a multiple of the tile height (128
// rows, or 32 for the decode kernels) so every tile belongs to one expert:
//   1. count:   per-chunk expert histograms (shared-memory atomics)
//   2. scan:    per-expert totals, per-chunk bases, tile prefix
//   3. scatter: stable positions (warp match + per-warp counts), inverse map,
//               per-row token id and routing weight
//   4. gather:  copy each token's row of x to its permuted rows (bf16 path)
#pragma once

#include "common.cuh"

namespace moe {

constexpr int DISPATCH_CHUNK = 1024;
constexpr int DISPATCH_THREADS = 256;
constexpr int DISPATCH_MAXE = 512;
constexpr int TILE_M = 128;

struct DispatchParams {
    const int32_t *topk_idx; // [N*k]
    const float *topk_w;     // [N*k]
    int N, k, E, nchunks;
    int tile_rows;       // rows per tile of the permuted layout (128, or 32 for decode)
    int32_t *chunk_hist; // [nchunks][E] counts, then absolute bases
    int32_t *counts;     // [E]
    int32_t *tile_off;   // [E+1] prefix of tiles per expert
    int32_t *meta;       // [0] done counter, [1] padded rows, [2] routed m-tiles
    int32_t *pos_of;     // [N*k] permuted row of each (token, slot), -1 if none
    int32_t *perm_tok;   // [rows_max] token of each permuted row (padding rows: unset)
    float *w_perm;       // [rows_max] routing weight of each permuted row (padding rows: unset)
};

__global__ void __launch_bounds__(DISPATCH_THREADS) dispatch_count_kernel(const DispatchParams p) {
    __shared__ int hist[DISPATCH_MAXE];
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int total = p.N * p.k;
    const int base = blockIdx.x * DISPATCH_CHUNK;
    for (int i = base + threadIdx.x; i < min(base + DISPATCH_CHUNK, total); i += blockDim.x) {
        const int e = p.topk_idx[i];
        if (e >= 0 && e < p.E)
            atomicAdd(&hist[e], 1);
        else if (e != p.E)
            record_error(DEV_BAD_INDEX, 10);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < p.E; e += blockDim.x)
        p.chunk_hist[(size_t)blockIdx.x * p.E + e] = hist[e];
}

// One CTA of DISPATCH_MAXE threads (thread e owns expert e).
__global__ void __launch_bounds__(DISPATCH_MAXE) dispatch_scan_kernel(const DispatchParams p) {
    __shared__ int wsum[DISPATCH_MAXE / 32];
    const int e = threadIdx.x;
    const int lane = e & 31, warp = e >> 5;
    int total = 0;
    if (e < p.E) {
        for (int c = 0; c < p.nchunks; ++c) {
            int *h = &p.chunk_hist[(size_t)c * p.E + e];
            const int v = *h;
            *h = total; // exclusive within the expert
            total += v;
        }
        p.counts[e] = total;
    }
    const int tiles = (e < p.E) ? (total + p.tile_rows - 1) / p.tile_rows : 0;
    // Block-wide exclusive scan of tiles.
    int v = tiles;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += n;
    }
    if (lane == 31) wsum[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = (lane < DISPATCH_MAXE / 32) ? wsum[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += n;
        }
        if (lane < DISPATCH_MAXE / 32) wsum[lane] = w;
    }
    __syncthreads();
    const int incl = v + (warp > 0 ? wsum[warp - 1] : 0);
    const int excl = incl - tiles;
    if (e < p.E) {
        p.tile_off[e] = excl;
        const int row0 = excl * p.tile_rows;
        for (int c = 0; c < p.nchunks; ++c) p.chunk_hist[(size_t)c * p.E + e] += row0;
    }
    if (e == p.E - 1) {
        p.tile_off[p.E] = incl;
        p.meta[0] = 0;
        p.meta[1] = incl * p.tile_rows;
        p.meta[2] = incl;
    }
}

__global__ void __launch_bounds__(DISPATCH_THREADS) dispatch_scatter_kernel(const DispatchParams p) {
    constexpr int NW = DISPATCH_THREADS / 32;
    __shared__ int cursor[DISPATCH_MAXE];
    __shared__ int wcnt[NW][DISPATCH_MAXE];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < p.E; e += DISPATCH_THREADS) {
        cursor[e] = p.chunk_hist[(size_t)blockIdx.x * p.E + e];
#pragma unroll
        for (int w = 0; w < NW; ++w) wcnt[w][e] = 0;
    }
    __syncthreads();
    const int total = p.N * p.k;
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int round = 0; round < DISPATCH_CHUNK / DISPATCH_THREADS; ++round) {
        const int i = blockIdx.x * DISPATCH_CHUNK + round * DISPATCH_THREADS + tid;
        const bool valid = i < total;
        int key = -1;
        if (valid) {
            const int e = p.topk_idx[i];
            key = (e >= 0 && e < p.E) ? e : -1;
        }
        const uint32_t peers = __match_any_sync(0xffffffffu, key);
        const int rank = __popc(peers & lt_mask);
        if (key >= 0 && rank == 0) wcnt[warp][key] = __popc(peers);
        __syncthreads();
        int pos = -1;
        if (key >= 0) {
            pos = cursor[key] + rank;
            for (int w = 0; w < warp; ++w) pos += wcnt[w][key];
        }
        __syncthreads();
        for (int e = tid; e < p.E; e += DISPATCH_THREADS) {
            int add = 0;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                add += wcnt[w][e];
                wcnt[w][e] = 0;
            }
            cursor[e] += add;
        }
        if (valid) {
            p.pos_of[i] = pos;
            if (pos >= 0) {
                p.perm_tok[pos] = i / p.k;
                p.w_perm[pos] = p.topk_w[i];
            }
        }
        __syncthreads();
    }
}

// Whole dispatch (count, scan, scatter) in one CTA for batches of at most
// DISPATCH_SMALL_IDS ids, as at decode: same results as the three kernels above
// (stable positions ordered by expert, then token, then slot).
constexpr int DISPATCH_SMALL_IDS = 2048;
constexpr int DISPATCH_SMALL_THREADS = 512;

// Body of the one-CTA dispatch for NT threads (NT >= E: thread e owns expert e in
// the scan); shared arrays hist[DISPATCH_MAXE], cursor[DISPATCH_MAXE],
// wcnt[NT/32][DISPATCH_MAXE], wsum[NT/32].
template <int NT>
__device__ __forceinline__ void dispatch_small_body(const DispatchParams &p, int *hist, int *cursor,
                                                    int (*wcnt)[DISPATCH_MAXE], int *wsum) {
    constexpr int NW = NT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int total = p.N * p.k;
    for (int e = tid; e < p.E; e += NT) {
        hist[e] = 0;
#pragma unroll
        for (int w = 0; w < NW; ++w) wcnt[w][e] = 0;
    }
    __syncthreads();
    for (int i = tid; i < total; i += NT) {
        const int e = p.topk_idx[i];
        if (e >= 0 && e < p.E)
            atomicAdd(&hist[e], 1);
        else if (e != p.E)
            record_error(DEV_BAD_INDEX, 11);
    }
    __syncthreads();
    // exclusive scan of tiles per expert (thread e owns expert e; E <= NT)
    const int e = tid;
    const int cnt = e < p.E ? hist[e] : 0;
    const int tiles = (cnt + p.tile_rows - 1) / p.tile_rows;
    int v = tiles;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += n;
    }
    if (lane == 31) wsum[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = lane < NW ? wsum[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += n;
        }
        if (lane < NW) wsum[lane] = w;
    }
    __syncthreads();
    const int incl = v + (warp > 0 ? wsum[warp - 1] : 0);
    const int excl = incl - tiles;
    if (e < p.E) {
        p.counts[e] = cnt;
        p.tile_off[e] = excl;
        cursor[e] = excl * p.tile_rows;
    }
    if (e == p.E - 1) {
        p.tile_off[p.E] = incl;
        p.meta[0] = 0;
        p.meta[1] = incl * p.tile_rows;
        p.meta[2] = incl;
    }
    __syncthreads();
    // stable positions, NT ids per round
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int base = 0; base < total; base += NT) {
        const int i = base + tid;
        const bool valid = i < total;
        int key = -1;
        if (valid) {
            const int ee = p.topk_idx[i];
            key = (ee >= 0 && ee < p.E) ? ee : -1;
        }
        const uint32_t peers = __match_any_sync(0xffffffffu, key);
        const int rank = __popc(peers & lt_mask);
        if (key >= 0 && rank == 0) wcnt[warp][key] = __popc(peers);
        __syncthreads();
        int pos = -1;
        if (key >= 0) {
            pos = cursor[key] + rank;
            for (int w = 0; w < warp; ++w) pos += wcnt[w][key];
        }
        __syncthreads();
        for (int ee = tid; ee < p.E; ee += NT) {
            int add = 0;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                add += wcnt[w][ee];
                wcnt[w][ee] = 0;
            }
            cursor[ee] += add;
        }
        if (valid) {
            p.pos_of[i] = pos;
            if (pos >= 0) {
                p.perm_tok[pos] = i / p.k;
                p.w_perm[pos] = p.topk_w[i];
            }
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(DISPATCH_SMALL_THREADS) dispatch_small_kernel(const DispatchParams p) {
    constexpr int NW = DISPATCH_SMALL_THREADS / 32;
    __shared__ int hist[DISPATCH_MAXE];
    __shared__ int cursor[DISPATCH_MAXE];
    __shared__ int wcnt[NW][DISPATCH_MAXE];
    __shared__ int wsum[NW];
    dispatch_small_body<DISPATCH_SMALL_THREADS>(p, hist, cursor, wcnt, wsum);
}

// Copy each token's row of x to its k permuted rows (x_perm[pos_of[n, j]]).  A
// warp takes one 2 KiB piece of one token's row: the piece is read once (x is
// usually larger than L2, and the permuted order would otherwise re-read each row
// k times) and written k times, with 16-byte vectors, four per lane in flight.
// Padding rows stay unwritten: an MMA output row depends only on its own operand
// row, and padding rows' outputs are never stored or read.  row_bytes is a
// multiple of 16.
// One warp per item (token n, 2 KiB piece); items item0, item0 + step, ...
__device__ __forceinline__ void gather_items(const uint8_t *__restrict__ x, uint8_t *__restrict__ x_perm,
                                             const DispatchParams &p, int row_bytes, int item0,
                                             int step) {
    const int lane = threadIdx.x & 31;
    const int nvec = row_bytes >> 4;
    const int pieces = (nvec + 127) / 128;
    for (int item = item0; item < p.N * pieces; item += step) {
        const int n = item / pieces;
        const int v0 = (item - n * pieces) * 128;
        const int my_pos = lane < p.k ? p.pos_of[(size_t)n * p.k + lane] : -1;
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)n * row_bytes);
        uint4 r[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int v = v0 + lane + 32 * u;
            if (v < nvec) r[u] = src[v];
        }
        for (int j = 0; j < p.k; ++j) {
            const int pos = __shfl_sync(0xffffffffu, my_pos, j);
            if (pos < 0) continue;
            uint4 *dst = reinterpret_cast<uint4 *>(x_perm + (size_t)pos * row_bytes);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int v = v0 + lane + 32 * u;
                if (v < nvec) dst[v] = r[u];
            }
        }
    }
}

__global__ void __launch_bounds__(256) dispatch_gather_kernel(const uint8_t *__restrict__ x,
                                                              uint8_t *__restrict__ x_perm,
                                                              const DispatchParams p,
                                                              int row_bytes) {
    gather_items(x, x_perm, p, row_bytes, (blockIdx.x * blockDim.x + threadIdx.x) >> 5,
                 (gridDim.x * blockDim.x) >> 5);
}

}  // namespace moe
