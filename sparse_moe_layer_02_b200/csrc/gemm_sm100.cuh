// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Both kernels are persistent (one CTA per SM, static round-robin over tiles) and
// warp-specialised, 192 threads:
//   warp 0      TMA producer: A tile 128 x 64 and B tile 256 x 64 (bf16, 128-byte
//               swizzle) per stage into a 4-stage shared-memory ring
//   warp 1      allocates 512 TMEM columns and issues tcgen05.mma (M=128, N=256,
//               K=16, bf16 in, fp32 accumulate) from one thread; two 256-column
//               accumulators alternate so the epilogue of one tile overlaps the
//               main loop of the next
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//               32*(w%4) .. +31, i.e. one output row per thread), math, stores
//
// gate_up ("GLM-4.5 MoE Forward": E_i(x) = W_down (SiLU(W_gate x) (.) W_up x);
// gate_up_proj[i] is (2 d_moe, D), gate rows first): one tile = 128 permuted
// token rows x 128 intermediate columns; B stacks 128 gate rows and the matching
// 128 up rows, so accumulator columns 0..127 hold the gate and 128..255 the up
// projection of the same columns and the epilogue writes h = SiLU(gate) * up in
// bf16.  The shared expert's tiles (A = x itself, B = its gate/up matrices) follow
// the routed tiles in the same launch.
//
// down: one tile = 128 rows x 256 output columns of W_down (D x d_moe).  Routed
// tiles scale each row by its routing weight; each epilogue warp stages 32 rows x
// 32 columns of bf16 per-slot partials in shared memory and writes them with one
// TMA store (the permuted rows of a tile are contiguous in the slot buffer).  The
// shared expert's tiles store their fp32 output.  Every tile bumps a done counter.
// The combine is the next launch (combine_kernel): row n of y = the k slot
// partials summed in slot order plus the shared expert's output at scale 1,
// written once in bf16 (deterministic: no atomics on the output).
#pragma once

#include "common.cuh"

namespace moe {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BN = 256;
constexpr int GEMM_BK = 64;
// Four 48 KiB stages: the most that fit beside the store staging.  The main loop
// is sensitive to the depth (three stages made gate_up 7 % slower).
constexpr int GEMM_STAGES = 4;
constexpr int GEMM_THREADS = 192;
constexpr int GEMM_A_BYTES = GEMM_BM * GEMM_BK * 2;  // 16 KiB
constexpr int GEMM_B_BYTES = GEMM_BN * GEMM_BK * 2;  // 32 KiB
constexpr int GEMM_STAGE_BYTES = GEMM_A_BYTES + GEMM_B_BYTES;
constexpr int GEMM_TMEM_COLS = 512;
constexpr int GEMM_MAXE = 512;
// Shared memory: 1024 alignment slack + ring + barriers/flags + tile table, then
// (1024-aligned) the down epilogue's store staging: per epilogue warp two buffers
// of 32 rows x 32 bf16 columns.
constexpr int GEMM_OUT_BOX = 32;                                   // rows and columns of a store box
constexpr int GEMM_OUT_BUF = GEMM_OUT_BOX * GEMM_OUT_BOX * 2;     // 2 KiB
constexpr int GEMM_STG_OFF =
    (GEMM_STAGES * GEMM_STAGE_BYTES + 256 + 2 * (GEMM_MAXE + 1) * 4 + 1023) / 1024 * 1024;
constexpr int GEMM_SMEM_BYTES = 1024 + GEMM_STG_OFF + 4 * 2 * GEMM_OUT_BUF;
static_assert(GEMM_SMEM_BYTES <= 232448, "shared memory");

enum GemmKind { GEMM_GATE_UP = 0, GEMM_DOWN = 1 };
enum GemmTiles {
    GEMM_ALL_TILES = 0,   // one-CTA kernel: every tile; pair kernel: every full pair
    GEMM_TAIL_TILES = 1,  // one-CTA kernel: the odd last m-tile of each expert
    GEMM_PAIR_PAD = 2,    // pair kernel: every m-tile, an odd last one with an empty half
    GEMM_ODD_EXPERTS = 3, // one-CTA kernel: every tile of the experts with an odd m-tile count
    GEMM_EVEN_EXPERTS = 4 // pair kernel: every tile of the experts with an even m-tile count
};

constexpr int EP_MAX_RANKS = 8; // ranks of an expert-parallel group

__device__ __forceinline__ uint32_t ld_acquire_sys_u32(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Adds 1 to ctr[key] for every lane of the calling (converged) warp with key in
// [0, nkeys), one atomic per distinct key, after the earlier stores of every lane
// of the warp are visible system-wide (they may be in another GPU's memory): each
// lane fences its own stores, the warp barrier orders all lanes before the
// leaders' atomics.
__device__ __forceinline__ void warp_count_rows(uint32_t *const *ctr, int key, int nkeys) {
    __threadfence_system();
    __syncwarp();
    const bool ok = key >= 0 && key < nkeys;
    const uint32_t same = __match_any_sync(0xffffffffu, ok ? key : -1);
    if (ok && (__ffs(same) - 1) == (int)(threadIdx.x & 31)) atomicAdd(ctr[key], (uint32_t)__popc(same));
}

struct GemmArgs {
    const int32_t *tile_off; // [E+1]
    int32_t *meta;           // [0] routed tiles done (down), [2] routed m-tiles
    int E, N, k;
    int nb_r, nb_s;      // n-blocks per routed / shared m-tile
    int mt_s;            // shared m-tiles
    int kb_r, kb_s;      // k-blocks of routed / shared tiles
    int b_rows_per_e;    // rows of one expert in the routed B map (2d or D)
    int up_off;          // gate_up: row offset of the up half (d)
    // outputs
    __nv_bfloat16 *out_r; // gate_up: h_perm [rows, ld_r]; down: slot [rows, ld_r]
    int ld_r, ncols_r;
    __nv_bfloat16 *out_s; // gate_up: h_sh [N, ld_s]; down: y [N, ld_s]
    int ld_s, ncols_s;
    const float *w_perm;   // down: routing weight per permuted row
    const int32_t *pos_of; // down: [N*k] permuted row of (n, j), -1 if none
    const __nv_bfloat16 *slot; // down: slot partials (same as out_r)
    float *osh;                // down: shared expert output [N, ld_s] fp32
    uint64_t wait_limit_ns;
    int never_signal;
    float gate_max, up_max; // gate_up: SwiGLU limits (+infinity = plain SwiGLU)
    int tma_out;            // down: routed rows stored by TMA through the mOut map
    // Tiles taken by the one-CTA kernel: GEMM_ALL_TILES, or GEMM_TAIL_TILES = only
    // the last m-tile of every expert with an odd m-tile count (and the last shared
    // m-tile when their count is odd), the tiles the CTA-pair kernel leaves over.
    int mode;
    // Expert parallelism (all null / 0 for a single-device layer).  The routed
    // rows are other ranks' tokens received into this rank's buffer.
    const uint32_t *ep_wait_ctr;    // gate_up: rows arrived (this epoch) ...
    const int32_t *ep_wait_target;  // ... must reach *ep_wait_target before any load
    const int4 *ep_meta;            // down: per routed row {source rank or -1, pair id, w bits, 0}
    int ep_P;                       // down: ranks; > 0 selects the expert-parallel epilogue
    __nv_bfloat16 *ep_out[EP_MAX_RANKS]; // down: every rank's slot buffer (rows by pair id)
    uint32_t *ep_ret[EP_MAX_RANKS];      // down: every rank's returned-rows counter (this epoch)
};

struct TileCoord {
    bool valid; // false: the odd half of a padded pair tile (no rows; nothing loaded or stored)
    bool shared;
    int e;     // routed expert
    int a_row; // row coordinate in the A map
    int nb;    // n-block
    int kb;    // k-blocks
};

// Exclusive prefix over the experts (one warp): out[e] = sum_{j < e} f(j) for
// e in [0, E], with f(j) from expert j's m-tile count m (tile prefix tile_off):
// kind 0 the full pairs m / 2, kind 1 the odd tail m % 2, kind 2 the pairs
// including a half-empty last one, (m + 1) / 2, kind 3 all m-tiles of an odd
// count (0 for even), kind 4 the pairs of an even count (0 for odd).
__device__ __forceinline__ void warp_expert_prefix(const int *tile_off, int E, int *out, int kind,
                                                   int lane) {
    int carry = 0;
    for (int base = 0; base <= E; base += 32) {
        const int e = base + lane;
        int v = 0;
        if (e < E) {
            const int m = tile_off[e + 1] - tile_off[e];
            v = kind == 1 ? (m & 1)
                : kind == 2 ? ((m + 1) >> 1)
                : kind == 3 ? ((m & 1) ? m : 0)
                : kind == 4 ? ((m & 1) ? 0 : (m >> 1))
                : (m >> 1);
        }
        int incl = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += n;
        }
        if (e <= E) out[e] = carry + incl - v;
        carry += __shfl_sync(0xffffffffu, incl, 31);
    }
}

// Largest e in [0, E) with pre[e] * nb <= t (pre non-decreasing, pre[0] = 0).
__device__ __forceinline__ int find_expert(const int *pre, int E, int nb, int t) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pre[mid] * nb <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// s_aux: the tail prefix (warp_expert_prefix with odd = 1) in GEMM_TAIL_TILES mode.
__device__ __forceinline__ TileCoord decode_tile(int t, int routed_tiles, const GemmArgs &a,
                                                 const int *s_tile_off, const int *s_aux) {
    TileCoord c;
    if (t < routed_tiles) {
        if (a.mode == GEMM_TAIL_TILES) {
            // one odd tail m-tile per listed expert, its n-blocks consecutive
            const int e = find_expert(s_aux, a.E, a.nb_r, t);
            c.nb = t - s_aux[e] * a.nb_r;
            c.valid = true;
            c.shared = false;
            c.e = e;
            c.a_row = (s_tile_off[e + 1] - 1) * GEMM_BM;
            c.kb = a.kb_r;
            return c;
        }
        // Expert-major order: expert e owns tiles [tile_off[e] * nb_r, tile_off[e+1] * nb_r),
        // n-block-major inside, so the m-tiles that read the same weight tile are
        // neighbours in the round-robin and run at the same time (one HBM read,
        // the others hit L2).  GEMM_ODD_EXPERTS numbers only the odd-count experts'
        // tiles, through their prefix s_aux, in the same order.
        const int *pre = a.mode == GEMM_ODD_EXPERTS ? s_aux : s_tile_off;
        const int lo = find_expert(pre, a.E, a.nb_r, t);
        const int mte = s_tile_off[lo + 1] - s_tile_off[lo];
        const int local = t - pre[lo] * a.nb_r;
        c.nb = local / mte;
        const int mt = s_tile_off[lo] + (local - c.nb * mte);
        c.valid = true;
        c.shared = false;
        c.e = lo;
        c.a_row = mt * GEMM_BM;
        c.kb = a.kb_r;
    } else {
        const int t2 = t - routed_tiles;
        int mt;
        if (a.mode == GEMM_TAIL_TILES) {
            mt = a.mt_s - 1;
            c.nb = t2;
        } else {
            mt = t2 / a.nb_s;
            c.nb = t2 - mt * a.nb_s;
        }
        c.valid = true;
        c.shared = true;
        c.e = -1;
        c.a_row = mt * GEMM_BM;
        c.kb = a.kb_s;
    }
    return c;
}

__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Store 32 consecutive fp32 values as bf16 (cols [col, col+32) of a row), only the
// 8-column pieces that lie below ncols (ncols % 8 == 0).
__device__ __forceinline__ void store_row_chunk_bf16(__nv_bfloat16 *row_ptr, int col, int ncols,
                                                     const float (&v)[32]) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
    uint4 *dst = reinterpret_cast<uint4 *>(row_ptr + col);
#pragma unroll
    for (int q = 0; q < 4; ++q)
        if (col + 8 * q < ncols) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
}

// Adds the eight bf16 values of w into acc (fp32).
__device__ __forceinline__ void acc_bf16x8(float (&acc)[8], const uint4 &w) {
    float lo, hi;
    unpack_bf16x2(w.x, lo, hi); acc[0] += lo; acc[1] += hi;
    unpack_bf16x2(w.y, lo, hi); acc[2] += lo; acc[3] += hi;
    unpack_bf16x2(w.z, lo, hi); acc[4] += lo; acc[5] += hi;
    unpack_bf16x2(w.w, lo, hi); acc[6] += lo; acc[7] += hi;
}

// y[n] = sum_{j<k} slot[pos(n, j)] (slot order) + osh[n], one warp per row, each
// lane U 8-column pieces at a time.  The slot rows are fetched eight slots at a
// time before any of them is added, so 8 U slot loads and the shared row are in
// flight per lane (the loop is bound by load latency); the adds then run in slot
// order (a missing slot adds +0).  U = 2 keeps a thread at 128 registers, so two
// 256-thread CTAs fit on an SM; with U = 4 (228 registers, one CTA per SM) the
// combine ran 20-26 % slower.
template <int U = 2>
__device__ __forceinline__ void combine_rows(const GemmArgs &a, int gwarp, int nwarps, int lane) {
    const int pieces = a.ncols_s / 8;
    for (int n = gwarp; n < a.N; n += nwarps) {
        const int my_pos = lane < a.k ? a.pos_of[(size_t)n * a.k + lane] : -1;
        for (int pbase = 0; pbase < pieces; pbase += 32 * U) {
            const int p0 = pbase + lane;
            float4 o[U][2];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int pc = p0 + 32 * u;
                if (pc < pieces) {
                    const float4 *op = reinterpret_cast<const float4 *>(a.osh + (size_t)n * a.ld_s + pc * 8);
                    o[u][0] = __ldcg(op);
                    o[u][1] = __ldcg(op + 1);
                }
            }
            float sum[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int h = 0; h < 8; ++h) sum[u][h] = 0.f;
            for (int jb = 0; jb < a.k; jb += 8) {
                uint4 w[8][U];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const int j = jb + jj;
                    const int p = __shfl_sync(0xffffffffu, my_pos, j & 31);
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int pc = p0 + 32 * u;
                        w[jj][u] = make_uint4(0u, 0u, 0u, 0u);
                        if (j < a.k && p >= 0 && pc < pieces)
                            w[jj][u] = __ldcg(reinterpret_cast<const uint4 *>(
                                a.slot + (size_t)p * a.ld_r + pc * 8));
                    }
                }
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
#pragma unroll
                    for (int u = 0; u < U; ++u) acc_bf16x8(sum[u], w[jj][u]);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int pc = p0 + 32 * u;
                if (pc < pieces) {
                    const float4 o0 = o[u][0], o1 = o[u][1];
                    const uint4 out = make_uint4(pack_bf16x2(sum[u][0] + o0.x, sum[u][1] + o0.y),
                                                 pack_bf16x2(sum[u][2] + o0.z, sum[u][3] + o0.w),
                                                 pack_bf16x2(sum[u][4] + o1.x, sum[u][5] + o1.y),
                                                 pack_bf16x2(sum[u][6] + o1.z, sum[u][7] + o1.w));
                    *reinterpret_cast<uint4 *>(a.out_s + (size_t)n * a.ld_s + pc * 8) = out;
                }
            }
        }
    }
}

// The combine, launched after the down kernel: one warp per row of y (see
// combine_rows).  As the down kernel's own final phase (six warps per SM) it ran
// 0.26-0.64 ms slower on the prefill workloads.
constexpr int COMBINE_THREADS = 256;

__global__ void __launch_bounds__(COMBINE_THREADS, 2) combine_kernel(const GemmArgs g) {
    constexpr int W = COMBINE_THREADS / 32;
    // Every down tile has been counted (the launch follows the down kernel on the
    // stream, so this holds at once; the bounded check reports a tile that never
    // completed instead of combining stale slots).
    __shared__ int failed;
    if (threadIdx.x == 0) {
        failed = 0;
        const int target = g.meta[2] * g.nb_r + g.mt_s * g.nb_s + (g.never_signal ? 1 : 0);
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_gpu(&g.meta[0]) < target) {
            if (globaltimer_ns() - t0 > g.wait_limit_ns) {
                record_error(DEV_TIMEOUT, 122);
                failed = 1;
                break;
            }
            __nanosleep(256);
        }
    }
    __syncthreads();
    if (failed) return;
    combine_rows(g, blockIdx.x * W + (threadIdx.x >> 5), gridDim.x * W, threadIdx.x & 31);
}

// Epilogue of one tile for the 32 rows of TMEM lane quadrant q (thread `lane`
// owns row q * 32 + lane of the tile): gate_up writes h = SwiGLU(gate, up) in
// bf16; down writes the routed rows scaled by their routing weight (bf16 slot
// partials, by TMA through mOut or per thread) or the shared expert's fp32 rows.
// tbase: the accumulator's TMEM address at this warp's lane quadrant.  stg /
// nstore: this warp's two store staging buffers and the boxes staged so far.
template <int KIND>
__device__ __forceinline__ void epilogue_tile(const GemmArgs &a, const CUtensorMap &mOut,
                                              const TileCoord &c, uint32_t tbase, int q, int lane,
                                              uint8_t *stg, uint32_t &nstore) {
    const int row = q * 32 + lane;
    if (KIND == GEMM_GATE_UP) {
        __nv_bfloat16 *out = c.shared ? a.out_s : a.out_r;
        const int ld = c.shared ? a.ld_s : a.ld_r;
        const int ncols = c.shared ? a.ncols_s : a.ncols_r;
        const int grow = c.a_row + row;
        const bool row_ok = c.shared ? (grow < a.N) : true;
        __nv_bfloat16 *row_ptr = out + (size_t)grow * ld;
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
            uint32_t g[32], u[32];
            tmem_ld_32x32b_x32(tbase + ch * 32, g);
            tmem_ld_32x32b_x32(tbase + 128 + ch * 32, u);
            tmem_ld_wait();
            const int col = c.nb * 128 + ch * 32;
            if (row_ok && col < ncols) {
                float h[32];
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    h[i] = swiglu_f(__uint_as_float(g[i]), __uint_as_float(u[i]),
                                    a.gate_max, a.up_max);
                store_row_chunk_bf16(row_ptr, col, ncols, h);
            }
        }
    } else if (!c.shared && a.tma_out) {
        // Routed rows are contiguous in the slot buffer: each 32-column chunk
        // of this warp's 32 rows is staged in shared memory and written by
        // one TMA store (full lines, off the epilogue threads' critical path).
        const float wr = a.w_perm[c.a_row + row];
#pragma unroll 1
        for (int ch = 0; ch < 8; ++ch) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tbase + ch * 32, v);
            tmem_ld_wait();
            const int col = c.nb * GEMM_BN + ch * 32;
            if (col < a.ncols_r) {
                uint8_t *buf = stg + (nstore & 1) * GEMM_OUT_BUF;
                if (lane == 0) bulk_wait_group_read<1>(); // the box staged 2 ago left buf
                __syncwarp();
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(wr * __uint_as_float(v[2 * i]),
                                        wr * __uint_as_float(v[2 * i + 1]));
                const uint4 u[4] = {make_uint4(pk[0], pk[1], pk[2], pk[3]),
                                    make_uint4(pk[4], pk[5], pk[6], pk[7]),
                                    make_uint4(pk[8], pk[9], pk[10], pk[11]),
                                    make_uint4(pk[12], pk[13], pk[14], pk[15])};
                uint4 *dst = reinterpret_cast<uint4 *>(buf + lane * (GEMM_OUT_BOX * 2));
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    // rotate the pieces across lanes (fewer bank conflicts); the
                    // selects keep the data in registers
                    const int p = (j + lane) & 3;
                    const uint4 val = p == 0 ? u[0] : p == 1 ? u[1] : p == 2 ? u[2] : u[3];
                    dst[p] = val;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&mOut, buf, col, c.a_row + q * 32);
                    bulk_commit_group();
                }
                ++nstore;
            }
        }
    } else if (!c.shared) {
        const int grow = c.a_row + row;
        float wr;
        __nv_bfloat16 *row_ptr;
        int src = 0;
        if (a.ep_P > 0) {
            // the row goes back to its token's rank, at the token's pair id;
            // padding rows carry source -1 and are not stored
            const int4 m = a.ep_meta[grow];
            src = (m.x >= 0 && m.x < a.ep_P) ? m.x : -1;
            wr = __int_as_float(m.z);
            row_ptr = src >= 0 ? a.ep_out[src] + (size_t)m.y * a.ld_r : nullptr;
        } else {
            wr = a.w_perm[grow];
            row_ptr = a.out_r + (size_t)grow * a.ld_r;
        }
#pragma unroll 1
        for (int ch = 0; ch < 8; ++ch) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tbase + ch * 32, v);
            tmem_ld_wait();
            const int col = c.nb * GEMM_BN + ch * 32;
            if (row_ptr && col < a.ncols_r) {
                float o[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = wr * __uint_as_float(v[i]);
                store_row_chunk_bf16(row_ptr, col, a.ncols_r, o);
            }
        }
        if (a.ep_P > 0) warp_count_rows(a.ep_ret, src, a.ep_P);
    } else {
        // shared expert: fp32 output rows, added last by combine_kernel
        const int n = c.a_row + row;
        float *row_ptr = a.osh + (size_t)n * a.ld_s;
#pragma unroll 1
        for (int ch = 0; ch < 8; ++ch) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tbase + ch * 32, v);
            tmem_ld_wait();
            const int col = c.nb * GEMM_BN + ch * 32;
            if (n < a.N && col < a.ncols_s) {
#pragma unroll
                for (int qv = 0; qv < 8; ++qv)
                    if (col + 4 * qv < a.ncols_s)
                        reinterpret_cast<float4 *>(row_ptr + col)[qv] =
                            make_float4(__uint_as_float(v[4 * qv]), __uint_as_float(v[4 * qv + 1]),
                                        __uint_as_float(v[4 * qv + 2]), __uint_as_float(v[4 * qv + 3]));
            }
        }
    }
}

// mOut (down with tma_out): the slot rows [rows, D] bf16, box 32 x 32, no swizzle.
template <int KIND>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap mA_r,
                        const __grid_constant__ CUtensorMap mB_r,
                        const __grid_constant__ CUtensorMap mA_s,
                        const __grid_constant__ CUtensorMap mB_s0,
                        const __grid_constant__ CUtensorMap mB_s1,
                        const __grid_constant__ CUtensorMap mOut, const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + GEMM_STAGES * GEMM_STAGE_BYTES);
    uint64_t *empty = full + GEMM_STAGES;
    uint64_t *tfull = empty + GEMM_STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *s_tile_off = reinterpret_cast<int *>(smem + GEMM_STAGES * GEMM_STAGE_BYTES + 256);
    int *s_aux = s_tile_off + (GEMM_MAXE + 1);

    const int warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < GEMM_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&mA_r);
        tma_prefetch_desc(&mB_r);
        tma_prefetch_desc(&mA_s);
        tma_prefetch_desc(&mB_s0);
        if (KIND == GEMM_GATE_UP) tma_prefetch_desc(&mB_s1);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, GEMM_TMEM_COLS);
        tmem_relinquish();
    }
    for (int i = threadIdx.x; i <= a.E; i += blockDim.x) s_tile_off[i] = a.tile_off[i];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    if (a.mode == GEMM_TAIL_TILES || a.mode == GEMM_ODD_EXPERTS) {
        if (warp == 2)
            warp_expert_prefix(s_tile_off, a.E, s_aux, a.mode == GEMM_TAIL_TILES ? 1 : 3, lane);
        __syncthreads();
    }

    const uint64_t limit = a.wait_limit_ns;
    if (a.ep_wait_ctr) {
        // Expert parallelism: other ranks write the routed rows; start once all of
        // them have arrived (bounded wait), and make the rows visible to TMA.
        if (threadIdx.x == 0) {
            const uint32_t target = (uint32_t)*a.ep_wait_target;
            const uint64_t t0 = globaltimer_ns();
            while (ld_acquire_sys_u32(a.ep_wait_ctr) < target) {
                if (globaltimer_ns() - t0 > limit) {
                    record_error(DEV_TIMEOUT, 104);
                    *abort_flag = 1;
                    break;
                }
                __nanosleep(128);
            }
            fence_proxy_async_global();
        }
        __syncthreads();
    }
    const bool tails = a.mode == GEMM_TAIL_TILES, odd_only = a.mode == GEMM_ODD_EXPERTS;
    const int routed_tiles = (tails || odd_only ? s_aux[a.E] : a.meta[2]) * a.nb_r;
    // the shared expert counts as one more expert: its last m-tile, or all of its
    // m-tiles, belong here when its m-tile count is odd
    const int shared_tiles = tails ? ((a.mt_s & 1) ? a.nb_s : 0)
                                   : odd_only ? ((a.mt_s & 1) ? a.mt_s * a.nb_s : 0)
                                              : a.mt_s * a.nb_s;
    const int total_tiles = *abort_flag ? 0 : routed_tiles + shared_tiles;

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                const TileCoord c = decode_tile(t, routed_tiles, a, s_tile_off, s_aux);
                const CUtensorMap *mA = c.shared ? &mA_s : &mA_r;
                // Tiles of one n-block (same weight tile) start at the same k-block and
                // share each weight line as it arrives; the n-blocks of one m-tile
                // (same token tile) start at different k-blocks, so they do not all
                // request the same token lines at the same time.
                const int rot = c.nb % c.kb;
                for (int i = 0; i < c.kb; ++i, ++it) {
                    const int kb = i + rot < c.kb ? i + rot : i + rot - c.kb;
                    const uint32_t s = it % GEMM_STAGES, ph = (it / GEMM_STAGES) & 1;
                    if (!mbar_wait(&empty[s], ph ^ 1, limit, abort_flag, 100)) { ok = false; break; }
                    uint8_t *sa = ring + s * GEMM_STAGE_BYTES;
                    uint8_t *sb = sa + GEMM_A_BYTES;
                    mbar_arrive_expect_tx(&full[s], GEMM_STAGE_BYTES);
                    const int kx = kb * GEMM_BK;
                    tma_load_2d(mA, &full[s], sa, kx, c.a_row);
                    if (KIND == GEMM_GATE_UP) {
                        if (c.shared) {
                            tma_load_2d(&mB_s0, &full[s], sb, kx, c.nb * 128);
                            tma_load_2d(&mB_s1, &full[s], sb + GEMM_B_BYTES / 2, kx, c.nb * 128);
                        } else {
                            const int r0 = c.e * a.b_rows_per_e + c.nb * 128;
                            tma_load_2d(&mB_r, &full[s], sb, kx, r0);
                            tma_load_2d(&mB_r, &full[s], sb + GEMM_B_BYTES / 2, kx, r0 + a.up_off);
                        }
                    } else {
                        if (c.shared)
                            tma_load_2d(&mB_s0, &full[s], sb, kx, c.nb * GEMM_BN);
                        else
                            tma_load_2d(&mB_r, &full[s], sb, kx, c.e * a.b_rows_per_e + c.nb * GEMM_BN);
                    }
                }
            }
            if (!ok) {
                // Let copies already issued land before the CTA's memory goes away.
                const uint32_t first = it > GEMM_STAGES ? it - GEMM_STAGES : 0;
                for (uint32_t j = first; j < it; ++j) {
                    volatile int no_abort = 0;
                    mbar_wait(&full[j % GEMM_STAGES], (j / GEMM_STAGES) & 1, 10000000ull, &no_abort, 101);
                }
            }
        }
        __syncwarp(); // lanes 1-31 wait here for lane 0: the warp reconverges
    } else if (warp == 1) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(GEMM_BM, GEMM_BN);
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++tc) {
                const TileCoord c = decode_tile(t, routed_tiles, a, s_tile_off, s_aux);
                const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
                if (!mbar_wait(&tempty[acc], aph ^ 1, limit, abort_flag, 110)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * GEMM_BN;
                for (int i = 0; i < c.kb; ++i, ++it) {
                    const uint32_t s = it % GEMM_STAGES, ph = (it / GEMM_STAGES) & 1;
                    if (!mbar_wait(&full[s], ph, limit, abort_flag, 111)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(ring + s * GEMM_STAGE_BYTES);
                    const uint32_t sb = sa + GEMM_A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < GEMM_BK / 16; ++kk)
                        umma_bf16_ss(d_tmem, umma_desc_sw128(sa + kk * 32),
                                     umma_desc_sw128(sb + kk * 32), idesc,
                                     (i > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[s]);
                }
                if (!ok) break;
                umma_commit(&tfull[acc]);
            }
            // Drain: wait until every MMA issued by this thread has completed.
            umma_commit(drain);
            volatile int no_abort = 0;
            mbar_wait(drain, 0, 100000000ull, &no_abort, 112);
        }
        __syncwarp();
    } else {
        // ------------------------------ epilogue ---------------------------------
        const int q = warp & 3;          // TMEM lane quadrant of this warp (rows q*32 + lane)
        const int ep_tid = threadIdx.x - 64;
        uint8_t *stg = smem + GEMM_STG_OFF + q * 2 * GEMM_OUT_BUF; // this warp's two store buffers
        uint32_t nstore = 0;             // store boxes this warp has staged
        uint32_t tc = 0;
        for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++tc) {
            const TileCoord c = decode_tile(t, routed_tiles, a, s_tile_off, s_aux);
            const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
            // After an abort every wait fails at once; the loop still walks the same
            // tiles in every epilogue warp so the named barriers stay matched.
            // One lane waits; the result is made warp-uniform before the
            // warp-collective TMEM loads.
            bool have = false;
            if (lane == 0) have = mbar_wait(&tfull[acc], aph, limit, abort_flag, 121);
            have = __shfl_sync(0xffffffffu, have ? 1 : 0, 0) != 0;
            __syncwarp();
            if (have) {
            tc_fence_after();
            const uint32_t tbase = tmem_base + acc * GEMM_BN + ((uint32_t)(q * 32) << 16);

            epilogue_tile<KIND>(a, mOut, c, tbase, q, lane, stg, nstore);
            // Release the accumulator.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            }  // have
            if (KIND == GEMM_DOWN) {
                // Count the finished tile (combine_kernel checks the count).
                __threadfence();
                named_bar_sync(1, 128);
                if (ep_tid == 0 && have) atomicAdd(&a.meta[0], 1);
            }
        }
    }

    if (KIND == GEMM_DOWN && warp >= 2 && lane == 0) bulk_wait_group<0>(); // stores done
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, GEMM_TMEM_COLS);
    }
    // Launched with programmatic serialization after the pair kernel (which reads
    // and writes none of this launch's rows), this launch starts on the SMs the
    // pair kernel frees and does not finish before it: the next kernel on the
    // stream then sees both.  Without that launch attribute this returns at once.
    grid_dep_wait();
}

}  // namespace moe

namespace moe {

// ---------------------------------------------------------------------------
// The same grouped GEMMs on CTA pairs (cta_group::2).  A cluster of two CTAs
// (the two SMs of a TPC) takes a pair tile: two consecutive m-tiles of one
// expert (or of the shared expert) times one n-block.  CTA r loads its own 128
// token rows (m-tile 2p + r) and half of the weight tile: gate_up the gate rows
// (r = 0) or the matching up rows (r = 1), down the first or second 128 of the
// 256 output features.  One thread of CTA 0 issues M = 256, N = 256, K = 16
// MMAs over both CTAs' shared memory, and each CTA's TMEM receives the
// accumulators of its own 128 rows: the same tile layout, so the same epilogue
// as the one-CTA kernel.  Per k-block each SM loads 32 KiB instead of 48 KiB
// for the same MMA work, so the ring holds six stages instead of four.
//
// Barriers: CTA 0's full[s] counts the bytes of both CTAs' loads (each CTA's
// TMA completes on it; CTA 0 announces the total); every MMA batch's commit
// arrives on empty[s] of both CTAs and the last one of a tile on tfull[acc] of
// both; the eight epilogue warps of the pair release an accumulator on CTA 0's
// tempty[acc].  An expert with an odd number of m-tiles either leaves its last
// m-tile to the one-CTA kernel in GEMM_TAIL_TILES mode (as does the shared
// expert's last m-tile when their count is odd), or, in GEMM_PAIR_PAD mode, runs
// it here as a pair whose second half has no rows (its MMA rows are wasted), or,
// in GEMM_EVEN_EXPERTS mode, runs wholly on the one-CTA kernel (GEMM_ODD_EXPERTS)
// while this kernel takes the experts with an even count.  Measured on the
// prefill configurations, only the last split beat the one-CTA kernel alone, and
// only for the down GEMM, where it is the default; gate_up stays on one SM.
// ---------------------------------------------------------------------------
constexpr int PAIR_STAGES = 6;
constexpr int PAIR_A_BYTES = GEMM_BM * GEMM_BK * 2;  // 16 KiB: this CTA's 128 rows
constexpr int PAIR_B_BYTES = 128 * GEMM_BK * 2;      // 16 KiB: this CTA's half of the 256 columns
constexpr int PAIR_STAGE_BYTES = PAIR_A_BYTES + PAIR_B_BYTES;
constexpr int PAIR_STG_OFF =
    (PAIR_STAGES * PAIR_STAGE_BYTES + 256 + 2 * (GEMM_MAXE + 1) * 4 + 1023) / 1024 * 1024;
constexpr int PAIR_SMEM_BYTES = 1024 + PAIR_STG_OFF + 4 * 2 * GEMM_OUT_BUF;
static_assert(PAIR_SMEM_BYTES <= 232448, "shared memory");

// Pair tile t for CTA `rank` of the pair: routed pairs first (expert-major,
// n-block-major inside, so pairs that read the same weight tile run together),
// then the shared expert's full pairs.  s_pair: prefix of m-tile pairs per expert.
__device__ __forceinline__ TileCoord decode_pair(int t, int routed_tiles, const GemmArgs &a,
                                                 const int *s_tile_off, const int *s_pair,
                                                 int rank) {
    TileCoord c;
    if (t < routed_tiles) {
        const int e = find_expert(s_pair, a.E, a.nb_r, t);
        const int pe = s_pair[e + 1] - s_pair[e];
        const int local = t - s_pair[e] * a.nb_r;
        c.nb = local / pe;
        const int p = local - c.nb * pe;
        const int mt = s_tile_off[e] + 2 * p + rank;
        c.valid = mt < s_tile_off[e + 1];
        c.shared = false;
        c.e = e;
        c.a_row = mt * GEMM_BM;
        c.kb = a.kb_r;
    } else {
        const int t2 = t - routed_tiles;
        const int mp = t2 / a.nb_s;
        c.nb = t2 - mp * a.nb_s;
        c.valid = 2 * mp + (int)rank < a.mt_s;
        c.shared = true;
        c.e = -1;
        c.a_row = (2 * mp + rank) * GEMM_BM;
        c.kb = a.kb_s;
    }
    return c;
}

// Maps as grouped_gemm_kernel, with 128-row boxes for every B operand.
template <int KIND>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap mA_r,
                             const __grid_constant__ CUtensorMap mB_r,
                             const __grid_constant__ CUtensorMap mA_s,
                             const __grid_constant__ CUtensorMap mB_s0,
                             const __grid_constant__ CUtensorMap mB_s1,
                             const __grid_constant__ CUtensorMap mOut, const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + PAIR_STAGES * PAIR_STAGE_BYTES);
    uint64_t *empty = full + PAIR_STAGES;
    uint64_t *tfull = empty + PAIR_STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *s_tile_off = reinterpret_cast<int *>(smem + PAIR_STAGES * PAIR_STAGE_BYTES + 256);
    int *s_pair = s_tile_off + (GEMM_MAXE + 1);
    // GEMM_PAIR_PAD: every m-tile runs here; an expert's odd last m-tile (and the
    // shared expert's) forms a pair with an empty half, whose rows CTA 1 neither
    // loads nor stores (its MMA rows are wasted).  Otherwise only full pairs run here.
    const bool pad = a.mode == GEMM_PAIR_PAD;

    const int warp = warp_id(), lane = lane_id();
    const uint32_t rank = cluster_ctarank();
    const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < PAIR_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 8);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&mA_r);
        tma_prefetch_desc(&mB_r);
        tma_prefetch_desc(&mA_s);
        tma_prefetch_desc(&mB_s0);
        if (KIND == GEMM_GATE_UP) tma_prefetch_desc(&mB_s1);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, GEMM_TMEM_COLS);
        tmem_relinquish_pair();
    }
    for (int i = threadIdx.x; i <= a.E; i += blockDim.x) s_tile_off[i] = a.tile_off[i];
    __syncthreads();
    const bool even_only = a.mode == GEMM_EVEN_EXPERTS;
    if (warp == 2) warp_expert_prefix(s_tile_off, a.E, s_pair, pad ? 2 : even_only ? 4 : 0, lane);
    tc_fence_before();
    // Both CTAs' barriers are initialised and their TMEM allocated before either
    // CTA's loads, MMAs or arrivals can reach the other.
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const uint64_t limit = a.wait_limit_ns;
    const int routed_tiles = s_pair[a.E] * a.nb_r;
    const int shared_pairs = even_only ? ((a.mt_s & 1) ? 0 : a.mt_s >> 1)
                                       : (pad ? a.mt_s + 1 : a.mt_s) >> 1;
    const int total_tiles = routed_tiles + shared_pairs * a.nb_s;
    // The one-CTA launch that follows (the other experts' tiles) may start on the
    // SMs this launch frees as its CTAs finish.
    grid_dep_launch_dependents();

    if (warp == 0) {
        // ------------------------------ TMA producer (both CTAs) ------------------
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            const uint32_t full0 = mapa_shared(smem_u32(full), 0); // CTA 0's full[0]
            for (int t = cid; t < total_tiles && ok; t += ncl) {
                const TileCoord c = decode_pair(t, routed_tiles, a, s_tile_off, s_pair, rank);
                // bytes CTA 0 announces: both CTAs' operands less an empty half's rows
                const bool full_pair = rank ? c.valid
                                            : decode_pair(t, routed_tiles, a, s_tile_off, s_pair, 1).valid;
                const uint32_t pair_bytes = 2 * PAIR_STAGE_BYTES - (full_pair ? 0 : PAIR_A_BYTES);
                const CUtensorMap *mA = c.shared ? &mA_s : &mA_r;
                const CUtensorMap *mB;
                int brow;
                if (KIND == GEMM_GATE_UP) {
                    if (c.shared) {
                        mB = rank ? &mB_s1 : &mB_s0;
                        brow = c.nb * 128;
                    } else {
                        mB = &mB_r;
                        brow = c.e * a.b_rows_per_e + (rank ? a.up_off : 0) + c.nb * 128;
                    }
                } else {
                    mB = c.shared ? &mB_s0 : &mB_r;
                    brow = (c.shared ? 0 : c.e * a.b_rows_per_e) + c.nb * GEMM_BN + rank * 128;
                }
                const int rot = c.nb % c.kb;
                for (int i = 0; i < c.kb; ++i, ++it) {
                    const int kb = i + rot < c.kb ? i + rot : i + rot - c.kb;
                    const uint32_t s = it % PAIR_STAGES, ph = (it / PAIR_STAGES) & 1;
                    if (!mbar_wait_cl(&empty[s], ph ^ 1, limit, abort_flag, 140)) { ok = false; break; }
                    uint8_t *sa = ring + s * PAIR_STAGE_BYTES;
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], pair_bytes);
                    const uint32_t fb = full0 + s * 8;
                    const int kx = kb * GEMM_BK;
                    if (c.valid) tma_load_2d_pair(mA, fb, sa, kx, c.a_row);
                    tma_load_2d_pair(mB, fb, sa + PAIR_A_BYTES, kx, brow);
                }
            }
            if (!ok && rank == 0) {
                // Let copies already issued land before the pair's memory goes away.
                const uint32_t first = it > PAIR_STAGES ? it - PAIR_STAGES : 0;
                for (uint32_t j = first; j < it; ++j) {
                    volatile int no_abort = 0;
                    mbar_wait(&full[j % PAIR_STAGES], (j / PAIR_STAGES) & 1, 10000000ull, &no_abort, 141);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------ MMA issuer (CTA 0) -------------------------
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(2 * GEMM_BM, GEMM_BN);
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int t = cid; t < total_tiles && ok; t += ncl, ++tc) {
                const TileCoord c = decode_pair(t, routed_tiles, a, s_tile_off, s_pair, 0);
                const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
                if (!mbar_wait_cl(&tempty[acc], aph ^ 1, limit, abort_flag, 150)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * GEMM_BN;
                for (int i = 0; i < c.kb; ++i, ++it) {
                    const uint32_t s = it % PAIR_STAGES, ph = (it / PAIR_STAGES) & 1;
                    if (!mbar_wait_cl(&full[s], ph, limit, abort_flag, 151)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(ring + s * PAIR_STAGE_BYTES);
                    const uint32_t sb = sa + PAIR_A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < GEMM_BK / 16; ++kk)
                        umma_bf16_ss_pair(d_tmem, umma_desc_sw128(sa + kk * 32),
                                          umma_desc_sw128(sb + kk * 32), idesc,
                                          (i > 0 || kk > 0) ? 1u : 0u);
                    umma_commit_pair_mc(&empty[s], 0x3);
                }
                if (!ok) break;
                umma_commit_pair_mc(&tfull[acc], 0x3);
            }
            // Drain: wait until every MMA issued by this thread has completed.
            umma_commit_pair(drain);
            volatile int no_abort = 0;
            mbar_wait(drain, 0, 100000000ull, &no_abort, 152);
        }
        __syncwarp();
    } else {
        // ------------------------------ epilogue (both CTAs) -----------------------
        const int q = warp & 3;
        const int ep_tid = threadIdx.x - 64;
        uint8_t *stg = smem + PAIR_STG_OFF + q * 2 * GEMM_OUT_BUF;
        uint32_t nstore = 0;
        uint32_t tc = 0;
        const uint32_t tempty0 = mapa_shared(smem_u32(tempty), 0); // CTA 0's tempty[0]
        for (int t = cid; t < total_tiles; t += ncl, ++tc) {
            const TileCoord c = decode_pair(t, routed_tiles, a, s_tile_off, s_pair, rank);
            const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
            bool have = false;
            if (lane == 0) have = mbar_wait_cl(&tfull[acc], aph, limit, abort_flag, 160);
            have = __shfl_sync(0xffffffffu, have ? 1 : 0, 0) != 0;
            __syncwarp();
            if (have) {
                tc_fence_after();
                const uint32_t tbase = tmem_base + acc * GEMM_BN + ((uint32_t)(q * 32) << 16);
                if (c.valid) epilogue_tile<KIND>(a, mOut, c, tbase, q, lane, stg, nstore);
                // Release the accumulator to the pair's MMA issuer.
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(tempty0 + acc * 8);
            }
            if (KIND == GEMM_DOWN) {
                // Count the finished m-tile (combine_kernel checks the count).
                __threadfence();
                named_bar_sync(1, 128);
                if (ep_tid == 0 && have && c.valid) atomicAdd(&a.meta[0], 1);
            }
        }
    }

    if (KIND == GEMM_DOWN && warp >= 2 && lane == 0) bulk_wait_group<0>(); // stores done
    tc_fence_before();
    // Neither CTA leaves while the pair's MMAs may still read its shared memory or
    // the other CTA may still arrive on its barriers.
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, GEMM_TMEM_COLS);
    }
}

}  // namespace moe
