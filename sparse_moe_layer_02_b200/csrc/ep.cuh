// Expert parallelism over peer memory ("GLM-5.3-Flash Module 02", the sections on
// expert placement and popularity: experts are spread over devices, and each
// token's hidden state travels to the devices holding its top-k experts and
// back).  P ranks, one per GPU; rank q holds experts [q*E/P, (q+1)*E/P) and its
// own batch of tokens.  Every rank owns one "symmetric" buffer of the same
// layout, mapped into every other rank's address space; all exchange is plain
// stores and atomics into the peers' buffers (NVLink / NVSwitch peer memory), no
// collective library call.
//
// One forward, epoch e (a call counter, the same on every rank), parity e & 1:
//   count   dense local dispatch of the rank's (token, slot) pairs by expert (the
//           single-device dispatch kernels with one-row tiles); its per-expert
//           counts and token count go into row `rank` of every rank's count
//           matrix, then flag[rank] = e is released into every rank.
//   send    wait (bounded) for all P flags; from the P x E counts every rank
//           derives every receiver's layout: expert-major, 128-row padded
//           segments, sources in rank order inside a segment, each source's
//           pairs in its (token, slot) order.  Each token row piece is stored
//           into the owners' receive buffers with {source rank, pair id, weight};
//           each stored (row, piece) adds 1 to the receiver's arrival counter.
//   experts the receiver's grouped gate_up + down (the single-device prefill
//           kernels) start once all its rows have arrived; the down epilogue
//           stores each routed row, scaled by its weight, into the source rank's
//           slot buffer at the pair id and adds 1 per (row, column block) to that
//           rank's return counter.  The shared expert runs on the rank's own
//           tokens in the same launches (fp32 output).
//   combine wait (bounded) for every returned row, then y = slots in slot order
//           + shared output, as on a single device.
// Counters are reset one epoch after their last use (the count phase of epoch
// e clears the counters of parity (e+1) & 1, whose last readers ran in epoch e-1
// and whose next writers wait for this rank's flag of epoch e+1).
//
// Every row is computed by the same kernels, from the same operand row and
// weights in the same k-block order, as on a single device, so the output equals
// the single-device prefill path's bit for bit.
#pragma once

#include "common.cuh"
#include "dispatch.cuh"
#include "gemm_sm100.cuh"

namespace moe {

constexpr int EP_TILE = 128;         // rows per tile of the receive layout
constexpr int EP_PIECE_VEC = 128;    // 16-byte vectors per piece of a token row (2 KiB)

// Byte offsets inside every rank's symmetric buffer (the same on all ranks).
struct EpSym {
    size_t cnt;       // int32 [2][P][E + 1]: per parity, row r = rank r's counts, then its N
    size_t flag;      // uint32 [2][P]: epoch of rank r's published counts
    size_t ctr;       // uint32 [4]: arrivals by parity, then returns by parity
    size_t recv_x;    // bf16 [rows_cap][D]: rows received for this rank's experts
    size_t recv_meta; // int4 [rows_cap]: {source rank or -1, pair id, weight bits, 0}
    size_t slot;      // bf16 [N_cap * k][D]: returned weighted rows of this rank's pairs
    size_t total;
    int rows_cap;
};

inline size_t ep_align(size_t v) { return (v + 255) / 256 * 256; }

// Layout of the symmetric buffer for P ranks of at most N_cap tokens each.
inline bool ep_sym_layout(int P, int N_cap, int D, int E, int k, EpSym &S) {
    if (P < 1 || P > EP_MAX_RANKS || N_cap < 0 || D <= 0 || E <= 0 || E % P || k <= 0) return false;
    const size_t pairs_all = (size_t)P * N_cap * k;
    const size_t rows = (pairs_all + (size_t)(E / P) * (EP_TILE - 1) + EP_TILE - 1) / EP_TILE * EP_TILE;
    if (rows > (size_t)INT32_MAX / 2) return false;
    S.rows_cap = (int)rows;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = ep_align(off + bytes);
        return at;
    };
    S.cnt = take((size_t)2 * P * (E + 1) * 4);
    S.flag = take((size_t)2 * P * 4);
    S.ctr = take(4 * 4);
    S.recv_x = take(rows * D * 2);
    S.recv_meta = take(rows * 16);
    S.slot = take((size_t)N_cap * k * D * 2);
    S.total = off;
    return true;
}

struct EpParams {
    int P, rank, E, E_loc, k, N, D;
    uint32_t epoch;
    uint8_t *sym[EP_MAX_RANKS]; // every rank's symmetric buffer, as mapped on this device
    EpSym S;
    const uint8_t *x;           // [N][D] bf16, this rank's tokens
    const int32_t *topk_idx;    // [N*k]
    const float *topk_w;        // [N*k]
    const int32_t *counts;      // [E] dense dispatch: pairs per expert
    const int32_t *dense_off;   // [E+1] dense dispatch: exclusive prefix of counts
    const int32_t *pos_of;      // [N*k] dense dispatch: position, -1 if none
    int32_t *dest_base;         // [E] receiver row of dense position 0 of expert e
    int32_t *rcounts;           // [E_loc] rows received per local expert
    int32_t *rtile_off;         // [E_loc+1] tile prefix of the receive layout
    int32_t *rmeta;             // [16] [0] down tiles done, [1] rows, [2] tiles,
                                //      [3] arrival target, [4] return target,
                                //      [5] 1 if the count exchange timed out
    int32_t *pair_pos;          // [N*k] pair id if routed, else -1 (combine rows)
    int down_nb;                // column blocks of the down kernel (ceil(D / 256))
    uint64_t wait_limit_ns;
};

__device__ __forceinline__ int32_t *ep_cnt(const EpParams &p, int q, int parity) {
    return reinterpret_cast<int32_t *>(p.sym[q] + p.S.cnt) + (size_t)parity * p.P * (p.E + 1);
}
__device__ __forceinline__ uint32_t *ep_flag(const EpParams &p, int q, int parity) {
    return reinterpret_cast<uint32_t *>(p.sym[q] + p.S.flag) + parity * p.P;
}
__device__ __forceinline__ uint32_t *ep_ctr(const EpParams &p, int q) {
    return reinterpret_cast<uint32_t *>(p.sym[q] + p.S.ctr);
}

__device__ __forceinline__ void st_release_sys_u32(uint32_t *ptr, uint32_t v) {
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}

// count phase (one CTA): publish this rank's per-expert counts and token count
// into every rank's count matrix, then release its flag there.
__global__ void __launch_bounds__(512) ep_publish_kernel(const EpParams p) {
    const int par = p.epoch & 1;
    if (threadIdx.x == 0) {
        uint32_t *c = ep_ctr(p, p.rank);
        c[par ^ 1] = 0;       // arrivals of the other parity
        c[2 + (par ^ 1)] = 0; // returns of the other parity
    }
    for (int q = 0; q < p.P; ++q) {
        int32_t *row = ep_cnt(p, q, par) + (size_t)p.rank * (p.E + 1);
        for (int e = threadIdx.x; e <= p.E; e += blockDim.x) row[e] = e < p.E ? p.counts[e] : p.N;
    }
    __threadfence_system();
    __syncthreads();
    if (threadIdx.x < p.P) st_release_sys_u32(ep_flag(p, threadIdx.x, par) + p.rank, p.epoch);
}

// send phase, step 1 (one CTA of 512 threads, E <= 512): wait for every rank's
// counts, then derive this rank's send offsets and its receive layout.
__global__ void __launch_bounds__(512) ep_layout_kernel(const EpParams p) {
    __shared__ int tiles[DISPATCH_MAXE];
    __shared__ int fail;
    __shared__ int red[2];
    const int par = p.epoch & 1, tid = threadIdx.x;
    if (tid == 0) {
        fail = 0;
        red[0] = red[1] = 0;
    }
    __syncthreads();
    if (tid < p.P) {
        const uint32_t *f = ep_flag(p, p.rank, par) + tid;
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_sys_u32(f) != p.epoch) {
            if (globaltimer_ns() - t0 > p.wait_limit_ns) {
                record_error(DEV_TIMEOUT, 140);
                atomicExch(&fail, 1);
                break;
            }
            __nanosleep(64);
        }
    }
    __syncthreads();
    const int32_t *cnt = ep_cnt(p, p.rank, par);
    const int e = tid;
    int R = 0, pre = 0;
    if (e < p.E && !fail) {
        for (int r = 0; r < p.P; ++r) {
            const int c = cnt[(size_t)r * (p.E + 1) + e];
            R += c;
            if (r < p.rank) pre += c;
        }
    }
    if (e < p.E) tiles[e] = (R + EP_TILE - 1) / EP_TILE;
    __syncthreads();
    // receiver q's segments: experts q*E_loc .. in order, each padded to tiles
    const int q = e < p.E ? e / p.E_loc : 0, first = q * p.E_loc;
    int tprefix = 0;
    if (e < p.E) {
        for (int e2 = first; e2 < e; ++e2) tprefix += tiles[e2];
        // a receiver whose rows would not fit its buffer (a rank past N_cap): give up
        if (e - first == p.E_loc - 1 && (long)(tprefix + tiles[e]) * EP_TILE > p.S.rows_cap) {
            record_error(DEV_BAD_INDEX, 142);
            atomicExch(&fail, 1);
        }
    }
    __syncthreads();
    if (e < p.E && !fail) {
        p.dest_base[e] = tprefix * EP_TILE + pre - p.dense_off[e];
        if (q == p.rank) {
            const int el = e - first;
            p.rcounts[el] = R;
            p.rtile_off[el] = tprefix;
            if (el == p.E_loc - 1) {
                p.rtile_off[p.E_loc] = tprefix + tiles[e];
                p.rmeta[1] = (tprefix + tiles[e]) * EP_TILE;
                p.rmeta[2] = tprefix + tiles[e];
            }
            atomicAdd(&red[0], R);
            // padding rows of this segment go nowhere when the down kernel stores
            int4 *meta = reinterpret_cast<int4 *>(p.sym[p.rank] + p.S.recv_meta);
            for (int r = tprefix * EP_TILE + R; r < (tprefix + tiles[e]) * EP_TILE; ++r)
                meta[r] = make_int4(-1, 0, 0, 0);
        }
        atomicAdd(&red[1], cnt[(size_t)p.rank * (p.E + 1) + e]);
    }
    if (fail && e < p.E_loc) {
        p.rcounts[e] = 0;
        p.rtile_off[e] = 0;
        if (e == p.E_loc - 1) p.rtile_off[p.E_loc] = 0;
    }
    if (tid == 0) {
        p.rmeta[0] = 0;
        if (fail) p.rmeta[1] = p.rmeta[2] = 0;
    }
    __syncthreads();
    if (tid == 0) {
        const int pieces = ((p.D * 2 / 16) + EP_PIECE_VEC - 1) / EP_PIECE_VEC;
        p.rmeta[3] = red[0] * pieces;      // (row, piece) stores this rank receives
        p.rmeta[4] = red[1] * p.down_nb;   // (row, column block) stores it gets back
        p.rmeta[5] = fail;                 // nothing is sent on a failed exchange
    }
}

// send phase, step 2: one warp per 2 KiB piece of a token row (as the
// single-device gather), stored into the receive buffers of the ranks owning
// the token's experts; piece 0 also stores each pair's {source, pair, weight}.
__global__ void __launch_bounds__(256) ep_send_kernel(const EpParams p) {
    if (p.rmeta[5]) return;
    const int lane = threadIdx.x & 31;
    const int row_bytes = p.D * 2;
    const int nvec = row_bytes >> 4;
    const int pieces = (nvec + EP_PIECE_VEC - 1) / EP_PIECE_VEC;
    const int par = p.epoch & 1;
    for (int item = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; item < p.N * pieces;
         item += (gridDim.x * blockDim.x) >> 5) {
        const int n = item / pieces;
        const int piece = item - n * pieces;
        const int v0 = piece * EP_PIECE_VEC;
        int q = -1, row = 0;
        if (lane < p.k) {
            const int i = n * p.k + lane;
            const int pos = p.pos_of[i];
            const int e = p.topk_idx[i];
            if (pos >= 0) {
                q = e / p.E_loc;
                row = p.dest_base[e] + pos;
            }
            if (piece == 0) {
                p.pair_pos[i] = pos >= 0 ? i : -1;
                if (pos >= 0) {
                    int4 *meta = reinterpret_cast<int4 *>(p.sym[q] + p.S.recv_meta);
                    meta[row] = make_int4(p.rank, i, __float_as_int(p.topk_w[i]), 0);
                }
            }
        }
        const uint4 *src = reinterpret_cast<const uint4 *>(p.x + (size_t)n * row_bytes);
        uint4 r[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int v = v0 + lane + 32 * u;
            if (v < nvec) r[u] = src[v];
        }
        for (int j = 0; j < p.k; ++j) {
            const int qj = __shfl_sync(0xffffffffu, q, j);
            const int rowj = __shfl_sync(0xffffffffu, row, j);
            if (qj < 0) continue;
            uint4 *dst = reinterpret_cast<uint4 *>(p.sym[qj] + p.S.recv_x + (size_t)rowj * row_bytes);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int v = v0 + lane + 32 * u;
                if (v < nvec) dst[v] = r[u];
            }
        }
        uint32_t *ctr[EP_MAX_RANKS];
#pragma unroll
        for (int t = 0; t < EP_MAX_RANKS; ++t) ctr[t] = t < p.P ? ep_ctr(p, t) + par : nullptr;
        warp_count_rows(ctr, q, p.P);
    }
}

// combine phase: wait (bounded) until every row this rank's pairs get back has
// been stored, then y = sum of the k slots in slot order + shared output.
__global__ void __launch_bounds__(256, 2) ep_combine_kernel(const EpParams p, const GemmArgs g) {
    __shared__ int fail;
    if (threadIdx.x == 0) {
        fail = 0;
        const uint32_t *c = ep_ctr(p, p.rank) + 2 + (p.epoch & 1);
        const uint32_t target = (uint32_t)p.rmeta[4];
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_sys_u32(c) < target) {
            if (globaltimer_ns() - t0 > p.wait_limit_ns) {
                record_error(DEV_TIMEOUT, 141);
                fail = 1;
                break;
            }
            __nanosleep(128);
        }
    }
    __syncthreads();
    if (fail) return;
    const int warp = threadIdx.x >> 5;
    combine_rows(g, blockIdx.x * 8 + warp, gridDim.x * 8, threadIdx.x & 31);
}

}  // namespace moe
