// C-ABI entry points of libmoe: argument checks, workspace planning, TMA
// descriptor encoding and kernel launches.  Declarations and the contract of
// every entry point are in include/moe.h.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstring>
#include <mutex>

#include "moe.h"
#include "common.cuh"
#include "dispatch.cuh"
#include "ep.cuh"
#include "gemm_decode_sm100.cuh"
#include "gemm_sm100.cuh"
#include "router.cuh"
#include "router_tc.cuh"
#include "simt_f32.cuh"

namespace moe {
namespace {

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;
// bf16 layers with at most this many tokens take the decode kernels (weights as
// the 128-row MMA operand, 32-token tiles); larger ones the 128-row token tiles.
constexpr int kDecodeMaxTokens = 256;
uint64_t g_wait_limit_ns = kDefaultWaitLimitNs;
int g_never_signal = 0;
// Prefill expert GEMMs on CTA pairs: 0 never, 1 full pairs with the odd last
// m-tiles on the one-CTA kernel, 2 every m-tile in pairs, odd ones with an empty
// half, 3 the even-count experts on pairs and the odd-count ones on the one-CTA
// kernel, 4 the same for the down GEMM only; -1 selects kDefaultPairMode (a test
// and tuning hook).
constexpr int kDefaultPairMode = 4;
int g_pair_mode = -1;
// Test hook: device buffer receiving the router's selection scores s' (null: off).
float *g_dbg_sp = nullptr;
size_t g_dbg_sp_n = 0;

std::atomic<unsigned long long> g_launches{0};
constexpr int kMaxProfEvents = 16;
void *g_prof_events[kMaxProfEvents];
int g_prof_n = 0;

// Records the caller's profiling events (if any) at kernel boundaries of one call.
struct Profiler {
    cudaStream_t st;
    int next = 0;
    bool capturing = false;
    explicit Profiler(cudaStream_t s, bool active = true) : st(s) {
        if (!active) return;
        if (g_prof_n > 0) {
            cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
            capturing = cudaStreamIsCapturing(st, &cs) == cudaSuccess &&
                        cs == cudaStreamCaptureStatusActive;
        }
        mark();
    }
    void mark() {
        if (next < g_prof_n && g_prof_events[next]) {
            cudaEvent_t ev = static_cast<cudaEvent_t>(g_prof_events[next]);
            // Under stream capture an external record becomes an event-record node of
            // the graph (a plain record would only order the capture).
            const cudaError_t e = capturing
                                      ? cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal)
                                      : cudaEventRecord(ev, st);
            if (e != cudaSuccess) cudaGetLastError(); // profiling never fails the call
        }
        ++next;
    }
};

constexpr int kMaxDevices = 64;
struct DeviceInfo {
    bool ready;
    int sms;
    int major, minor;
    bool gemm_attr_set;
    bool dec_attr_set;
    bool pair_attr_set;
    int pair_max_clusters; // co-resident CTA pairs of the pair kernels (0: unusable)
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

int current_device_info(DeviceInfo **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.ready) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MOE_ERR_CUDA;
        d.sms = prop.multiProcessorCount;
        d.major = prop.major;
        d.minor = prop.minor;
        d.ready = true;
    }
    *out = &d;
    return MOE_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int check_router_shape(int N, int D, int E, int G, int tg, int k) {
    if (N < 0 || N > 65535 * ROUTER_TM || D <= 0 || E <= 0 || E > DISPATCH_MAXE)
        return MOE_ERR_SHAPE;
    if (G <= 0 || G > ROUTER_MAXG || E % G != 0) return MOE_ERR_SHAPE;
    if (G > 1 && E / G < 2) return MOE_ERR_SHAPE;
    if (tg <= 0 || tg > G) return MOE_ERR_SHAPE;
    if (k <= 0 || k > 32 || k > tg * (E / G)) return MOE_ERR_SHAPE;
    return MOE_OK;
}

// ---------------------------------------------------------------------------
// Workspace layout (every region 256-byte aligned).
// ---------------------------------------------------------------------------
struct WsLayout {
    size_t chunk_hist, counts, tile_off, meta, pos_of, perm_tok, w_perm;
    size_t x_perm, h_perm, h_sh, slot, osh, wg_parts, total, total_with_parts;
    int nchunks;
    size_t rows_max;
    bool decode;
    int tile_rows;
};

// with_wg_parts: also reserve the three bf16 parts of an fp32 router matrix
// (moe_layer_forward's split-once path); moe_forward never uses them.
bool plan_workspace(int N, int D, int E, int d, int d_sh, int k, int dtype, WsLayout &L,
                    bool with_wg_parts = false) {
    if (N < 0 || D <= 0 || E <= 0 || d <= 0 || d_sh <= 0 || k <= 0) return false;
    if (dtype != MOE_F32 && dtype != MOE_BF16) return false;
    const size_t es = dtype == MOE_BF16 ? 2 : 4;
    const size_t nk = (size_t)N * (size_t)k;
    if (nk > (size_t)INT32_MAX / 2) return false;
    L.decode = dtype == MOE_BF16 && N <= kDecodeMaxTokens;
    L.tile_rows = L.decode ? DEC_TT : TILE_M;
    // Every non-empty expert pads its segment by at most tile_rows - 1 rows.
    const size_t busy = std::min<size_t>((size_t)E, std::max<size_t>(nk, 1));
    L.rows_max = round_up(nk + (size_t)(L.tile_rows - 1) * busy, TILE_M);
    if (L.rows_max > (size_t)INT32_MAX / 2) return false;
    L.nchunks = (int)((nk + DISPATCH_CHUNK - 1) / DISPATCH_CHUNK);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = round_up(off + bytes, 256);
        return at;
    };
    L.chunk_hist = take((size_t)std::max(L.nchunks, 1) * E * 4);
    L.counts = take((size_t)E * 4);
    L.tile_off = take((size_t)(E + 1) * 4);
    L.meta = take(16 * 4);
    L.pos_of = take(nk * 4);
    L.perm_tok = take(L.rows_max * 4);
    L.w_perm = take(L.rows_max * 4);
    L.x_perm = take(dtype == MOE_BF16 ? L.rows_max * D * es : 0);
    L.h_perm = take(L.rows_max * d * es);
    L.h_sh = take((size_t)N * d_sh * es);
    L.slot = take(L.rows_max * D * es);
    // fp32 output of the shared expert, combined with the slots (prefill kernels)
    L.osh = take(dtype == MOE_BF16 && !L.decode ? (size_t)N * D * 4 : 0);
    L.total = off;
    // the router matrix split into three bf16 parts (moe_layer_forward, fp32 W_g)
    L.wg_parts = take(with_wg_parts ? (size_t)3 * E * D * 2 : 0);
    L.total_with_parts = off;
    return true;
}

// ---------------------------------------------------------------------------
// TMA descriptors
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D bf16 map over a row-major [rows, cols] matrix with row stride ld elements;
// box = 64 columns (128 bytes, the swizzle span) x box_rows rows, 128-byte swizzle,
// out-of-range elements read as zero.
bool make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint64_t ld,
              uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * 2};
    cuuint32_t box[2] = {GEMM_BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D bf16 map for TMA stores of the down epilogue: box 32 columns x 32 rows,
// no swizzle (the staging buffer holds the box row-major).
bool make_map_out(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint64_t ld) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * 2};
    cuuint32_t box[2] = {GEMM_OUT_BOX, GEMM_OUT_BOX};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int launch_status() {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launched(Profiler &prof) {
    const int rc = launch_status();
    prof.mark();
    return rc;
}

int current_device_index() {
    int dev = 0;
    return cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices ? dev : -1;
}

// cudaLaunchKernelEx; a launch refused with the programmatic-serialization attribute
// (always the last one) is repeated without it.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(cudaLaunchConfig_t cfg, void (*kernel)(KArgs...), Args &&...args) {
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
    if (e != cudaSuccess && cfg.numAttrs > 0 &&
        cfg.attrs[cfg.numAttrs - 1].id == cudaLaunchAttributeProgrammaticStreamSerialization) {
        cudaGetLastError();
        --cfg.numAttrs;
        e = cudaLaunchKernelEx(&cfg, kernel, args...);
    }
    return e;
}

template <typename XT, typename WT, int EV>
int launch_router_t(const RouterParams &p, cudaStream_t st) {
    constexpr int smem = router_smem_bytes(EV);
    static bool attr_set[kMaxDevices] = {}; // function attributes are set per device
    const int dev = current_device_index();
    if (dev < 0) return MOE_ERR_CUDA;
    if (!attr_set[dev]) {
        std::lock_guard<std::mutex> lk(g_mu);
        if (cudaFuncSetAttribute(router_kernel<XT, WT, EV>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ROUTER_CL, (p.N + ROUTER_TM - 1) / ROUTER_TM, 1);
    cfg.blockDim = dim3(ROUTER_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ROUTER_CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, router_kernel<XT, WT, EV>, p) != cudaSuccess) return MOE_ERR_CUDA;
    return launch_status();
}

template <typename XT, typename WT>
int launch_router_x(const RouterParams &p, cudaStream_t st) {
    if (p.E <= 32) return launch_router_t<XT, WT, 1>(p, st);
    if (p.E <= 64) return launch_router_t<XT, WT, 2>(p, st);
    if (p.E <= 128) return launch_router_t<XT, WT, 4>(p, st);
    if (p.E <= 256) return launch_router_t<XT, WT, 8>(p, st);
    return launch_router_t<XT, WT, 16>(p, st);
}

template <int EV, bool WF32>
int launch_router_tc_t(const CUtensorMap &mX, const CUtensorMap &mW, const RouterParams &p, int clk,
                       const RtcFuse &fz, bool pdl, cudaStream_t st) {
    constexpr int smem = RtcCfg<WF32>::SMEM;
    // largest cluster size this kernel can be launched with, per device (the
    // attributes are set per device)
    static int max_clk_of[kMaxDevices] = {};
    const int dev = current_device_index();
    if (dev < 0) return MOE_ERR_CUDA;
    int &max_clk = max_clk_of[dev];
    if (!max_clk) {
        std::lock_guard<std::mutex> lk(g_mu);
        if (cudaFuncSetAttribute(router_tc_kernel<EV, WF32>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return MOE_ERR_CUDA;
        max_clk = 8;
        if (cudaFuncSetAttribute(router_tc_kernel<EV, WF32>,
                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
            cudaLaunchConfig_t q = {};
            q.gridDim = dim3(RTC_MAX_CLK, 1, 1);
            q.blockDim = dim3(RTC_THREADS, 1, 1);
            q.dynamicSmemBytes = smem;
            cudaLaunchAttribute qa[1];
            qa[0].id = cudaLaunchAttributeClusterDimension;
            qa[0].val.clusterDim.x = RTC_MAX_CLK;
            qa[0].val.clusterDim.y = 1;
            qa[0].val.clusterDim.z = 1;
            q.attrs = qa;
            q.numAttrs = 1;
            int clusters = 0;
            if (cudaOccupancyMaxActiveClusters(&clusters, router_tc_kernel<EV, WF32>, &q) ==
                    cudaSuccess &&
                clusters > 0)
                max_clk = RTC_MAX_CLK;
        }
        cudaGetLastError(); // a refused query is not an error of this call
    }
    if (clk > max_clk) clk = max_clk;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(clk, (p.N + RTC_BM - 1) / RTC_BM, 1);
    cfg.blockDim = dim3(RTC_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = clk;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    if (launch_ex(cfg, router_tc_kernel<EV, WF32>, mX, mW, p, g_wait_limit_ns, fz) != cudaSuccess)
        return MOE_ERR_CUDA;
    return launch_status();
}

// Tensor-core router for bf16 x with a bf16 W_g (16 <= E <= 256) or an fp32 W_g
// (16 <= E <= 192, three-way bf16 split); E % 16 == 0.
// pdl: launch with programmatic stream serialization (the fused decode path).
template <bool WF32>
int launch_router_tc(const RouterParams &p, int sms, const RtcFuse &fz, bool pdl, cudaStream_t st) {
    CUtensorMap mX, mW;
    if (!make_map(&mX, p.x, p.D, p.N, p.D, RTC_BM)) return MOE_ERR_CUDA;
    if (WF32 && p.wg_parts) {
        // the three bf16 parts [3E, D]; a box is one part's E rows
        if (!make_map(&mW, p.wg_parts, p.D, 3 * (uint64_t)p.E, p.D, p.E)) return MOE_ERR_CUDA;
    } else if (WF32) {
        mW = mX; // unused: the fp32 matrix is read and split by the kernel's own warps
    } else if (!make_map(&mW, p.W_g, p.D, p.E, p.D, p.E)) {
        return MOE_ERR_CUDA;
    }
    const int tblocks = (p.N + RTC_BM - 1) / RTC_BM;
    // K-split cluster size: a power of two (so it divides the 128 tokens of a
    // block) chosen to put about one CTA on every SM, and large enough that no
    // CTA accumulates more than RTC_MAX_KB k-blocks of the hidden dimension: the
    // tensor core rounds toward zero at every accumulation step, so shorter
    // chains (their partials summed in fp32 in rank order) keep the logits
    // closer to the exact sum.  At most 16 (8 where the device cannot
    // co-schedule 16-CTA clusters of this kernel).
    const int KB = (p.D + RTC_BK - 1) / RTC_BK;
    int clk = 1;
    while (clk < RTC_MAX_CLK && (2 * clk * tblocks <= sms || (KB + clk - 1) / clk > RTC_MAX_KB))
        clk *= 2;
    if (p.E <= 32) return launch_router_tc_t<1, WF32>(mX, mW, p, clk, fz, pdl, st);
    if (p.E <= 64) return launch_router_tc_t<2, WF32>(mX, mW, p, clk, fz, pdl, st);
    if (p.E <= 128) return launch_router_tc_t<4, WF32>(mX, mW, p, clk, fz, pdl, st);
    return launch_router_tc_t<8, WF32>(mX, mW, p, clk, fz, pdl, st);
}

// after_pair: launched right after a pair kernel that touches none of this
// launch's rows, with programmatic stream serialization, so it fills the SMs the
// pair kernel frees (the kernel waits for the pair kernel before it exits).
template <int KIND>
int launch_gemm(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &a2,
                const CUtensorMap &a3, const CUtensorMap &a4, const CUtensorMap &a5,
                const GemmArgs &args, int grid, bool cooperative, cudaStream_t st,
                bool after_pair = false) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = GEMM_SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = cooperative ? 1 : 0;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_pair && !cooperative ? 2 : 1;
    if (launch_ex(cfg, grouped_gemm_kernel<KIND>, a0, a1, a2, a3, a4, a5, args) != cudaSuccess)
        return MOE_ERR_CUDA;
    return launch_status();
}

template <int KIND>
int launch_gemm_pair(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &a2,
                     const CUtensorMap &a3, const CUtensorMap &a4, const CUtensorMap &a5,
                     const GemmArgs &args, int clusters, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters, 1, 1);
    cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = PAIR_SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, grouped_gemm_pair_kernel<KIND>, a0, a1, a2, a3, a4, a5, args) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    return launch_status();
}

// A non-cooperative launch uses programmatic stream serialization: the kernel
// waits for its predecessor before touching global memory.
template <int KIND>
int launch_decode(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &a2,
                  const CUtensorMap &a3, const CUtensorMap &a4, const DecArgs &args, int grid,
                  bool cooperative, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(DEC_THREADS, 1, 1);
    cfg.dynamicSmemBytes = dec_smem_bytes<KIND>();
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = cooperative ? 1 : 0;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = cooperative ? 1 : 2;
    if (launch_ex(cfg, grouped_gemm_decode_kernel<KIND>, a0, a1, a2, a3, a4, args) != cudaSuccess)
        return MOE_ERR_CUDA;
    return launch_status();
}

int ensure_decode_attrs(DeviceInfo *dev) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (dev->dec_attr_set) return MOE_OK;
    if (cudaFuncSetAttribute(grouped_gemm_decode_kernel<GEMM_GATE_UP>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dec_smem_bytes<GEMM_GATE_UP>()) != cudaSuccess ||
        cudaFuncSetAttribute(grouped_gemm_decode_kernel<GEMM_DOWN>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dec_smem_bytes<GEMM_DOWN>()) != cudaSuccess)
        return MOE_ERR_CUDA;
    dev->dec_attr_set = true;
    return MOE_OK;
}

int ensure_gemm_attrs(DeviceInfo *dev) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (dev->gemm_attr_set) return MOE_OK;
    if (cudaFuncSetAttribute(grouped_gemm_kernel<GEMM_GATE_UP>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GEMM_SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(grouped_gemm_kernel<GEMM_DOWN>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GEMM_SMEM_BYTES) != cudaSuccess)
        return MOE_ERR_CUDA;
    dev->gemm_attr_set = true;
    return MOE_OK;
}

// Shared-memory attributes of the pair kernels and the number of CTA pairs that
// can be co-resident (0 if the device cannot run them; the one-CTA kernels then
// take every tile).
int ensure_pair_attrs(DeviceInfo *dev) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (dev->pair_attr_set) return MOE_OK;
    dev->pair_max_clusters = 0;
    if (cudaFuncSetAttribute(grouped_gemm_pair_kernel<GEMM_GATE_UP>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PAIR_SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(grouped_gemm_pair_kernel<GEMM_DOWN>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PAIR_SMEM_BYTES) != cudaSuccess)
        return MOE_ERR_CUDA;
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(2 * dev->sms, 1, 1);
    q.blockDim = dim3(GEMM_THREADS, 1, 1);
    q.dynamicSmemBytes = PAIR_SMEM_BYTES;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 2;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.attrs = qa;
    q.numAttrs = 1;
    int c1 = 0, c2 = 0;
    if (cudaOccupancyMaxActiveClusters(&c1, grouped_gemm_pair_kernel<GEMM_GATE_UP>, &q) ==
            cudaSuccess &&
        cudaOccupancyMaxActiveClusters(&c2, grouped_gemm_pair_kernel<GEMM_DOWN>, &q) == cudaSuccess)
        dev->pair_max_clusters = std::min(c1, c2);
    cudaGetLastError(); // a refused query only disables the pair kernels
    dev->pair_attr_set = true;
    return MOE_OK;
}

// The router launch.  With fz (bf16 layers of at most 128 tokens whose logits run
// on the tensor cores) the dispatch and gather of the forward run inside the
// router kernel; *fused tells whether they did.
// wg_parts_ws: optional scratch of 3 * E * D bf16 for splitting an fp32 W_g once per
// call (used when the batch has several token blocks).
int router_impl(const void *x, int x_dtype, const void *W_g, int wg_dtype, const float *b, int N,
                int D, int E, int n_group, int topk_group, int k, int norm_topk_prob, float alpha,
                int32_t *topk_idx, float *topk_w, void *stream, const RtcFuse *fz, bool *fused,
                void *wg_parts_ws = nullptr) {
    if (fused) *fused = false;
    int rc = check_router_shape(N, D, E, n_group, topk_group, k);
    if (rc != MOE_OK) return rc;
    if ((x_dtype != MOE_F32 && x_dtype != MOE_BF16) || (wg_dtype != MOE_F32 && wg_dtype != MOE_BF16))
        return MOE_ERR_DTYPE;
    if (N == 0) return MOE_OK;
    if (!x || !W_g || !b || !topk_idx || !topk_w) return MOE_ERR_ARG;
    if (!aligned16(x) || !aligned16(W_g) || !aligned16(b) || !aligned16(topk_idx) ||
        !aligned16(topk_w))
        return MOE_ERR_ARG;
    DeviceInfo *dev = nullptr;
    if ((rc = current_device_info(&dev)) != MOE_OK) return rc;
    if (dev->major != 10) return MOE_ERR_NO_DEVICE;
    RouterParams p;
    p.x = x;
    p.W_g = W_g;
    p.b = b;
    p.N = N;
    p.D = D;
    p.E = E;
    p.G = n_group;
    p.tg = topk_group;
    p.k = k;
    p.norm = norm_topk_prob ? 1 : 0;
    p.alpha = alpha;
    p.topk_idx = topk_idx;
    p.topk_w = topk_w;
    p.wg_parts = nullptr;
    p.dbg_sp = nullptr;
    if (g_dbg_sp) {
        if (g_dbg_sp_n < (size_t)N * E) return MOE_ERR_ARG;
        p.dbg_sp = g_dbg_sp;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    RtcFuse off = {};
    const bool tc = x_dtype == MOE_BF16 && E % 16 == 0 && E >= 16 && D % 8 == 0 &&
                    ((wg_dtype == MOE_BF16 && E <= 256) || (wg_dtype == MOE_F32 && E <= RTC_MAXE_F32));
    if (tc) {
        const bool fuse = fz && fz->on && N <= RTC_BM && E <= RTC_THREADS;
        if (fused) *fused = fuse;
        if (wg_dtype == MOE_F32 && wg_parts_ws && N > RTC_BM) {
            // split W_g once instead of in every token block
            const size_t n8 = (size_t)E * D / 8;
            const int grid = (int)std::min<size_t>((n8 + 255) / 256, (size_t)dev->sms * 8);
            wg_split_kernel<<<grid, 256, 0, st>>>(static_cast<const float *>(W_g), E, D,
                                                  static_cast<__nv_bfloat16 *>(wg_parts_ws));
            if ((rc = launch_status()) != MOE_OK) return rc;
            p.wg_parts = wg_parts_ws;
        }
        const RtcFuse &f = fuse ? *fz : off;
        return wg_dtype == MOE_BF16 ? launch_router_tc<false>(p, dev->sms, f, fuse, st)
                                    : launch_router_tc<true>(p, dev->sms, f, fuse, st);
    }
    if (x_dtype == MOE_F32 && wg_dtype == MOE_F32) return launch_router_x<float, float>(p, st);
    if (x_dtype == MOE_BF16 && wg_dtype == MOE_F32) return launch_router_x<__nv_bfloat16, float>(p, st);
    if (x_dtype == MOE_BF16 && wg_dtype == MOE_BF16)
        return launch_router_x<__nv_bfloat16, __nv_bfloat16>(p, st);
    return launch_router_x<float, __nv_bfloat16>(p, st);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

int moe_version(void) { return 100; }

const char *moe_status_string(int status) {
    switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_ARG: return "invalid argument (null or misaligned pointer, bad flag)";
    case MOE_ERR_SHAPE: return "invalid or unsupported sizes";
    case MOE_ERR_DTYPE: return "unsupported dtype combination";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait ran out";
    case MOE_ERR_BAD_INDEX: return "topk_idx held an expert id outside [0, E]";
    case MOE_ERR_NO_DEVICE: return "no sm_100 device is current";
    default: return "unknown status";
    }
}

int moe_debug_set_wait_limit_ns(uint64_t ns) {
    g_wait_limit_ns = ns ? ns : kDefaultWaitLimitNs;
    return MOE_OK;
}

int moe_debug_never_signal(int on) {
    g_never_signal = on ? 1 : 0;
    return MOE_OK;
}

int moe_debug_set_pair_mode(int mode) {
    if (mode < -1 || mode > 4) return MOE_ERR_ARG;
    g_pair_mode = mode;
    return MOE_OK;
}

int moe_debug_capture_scores(float *buf, size_t n_floats) {
    if (buf && (!aligned16(buf) || n_floats == 0)) return MOE_ERR_ARG;
    g_dbg_sp = buf;
    g_dbg_sp_n = buf ? n_floats : 0;
    return MOE_OK;
}

int moe_profile_set_events(void *const *events, int n) {
    if (n < 0 || n > kMaxProfEvents || (n > 0 && !events)) return MOE_ERR_ARG;
    for (int i = 0; i < n; ++i) g_prof_events[i] = events[i];
    g_prof_n = n;
    return MOE_OK;
}

unsigned long long moe_launch_count(void) { return g_launches.load(); }

int moe_router(const void *x, int x_dtype, const void *W_g, int wg_dtype, const float *b, int N,
               int D, int E, int n_group, int topk_group, int k, int norm_topk_prob, float alpha,
               int32_t *topk_idx, float *topk_w, void *stream) {
    return moe::router_impl(x, x_dtype, W_g, wg_dtype, b, N, D, E, n_group, topk_group, k,
                            norm_topk_prob, alpha, topk_idx, topk_w, stream, nullptr, nullptr);
}

int moe_bias_update(const int32_t *topk_idx, int N, int k, int E, float rate, float *b,
                    int32_t *loads_out, void *stream) {
    if (N < 0 || k <= 0 || k > 32 || E <= 0 || E > 512) return MOE_ERR_SHAPE;
    if ((size_t)N * k > (size_t)INT32_MAX) return MOE_ERR_SHAPE;
    if (rate != rate) return MOE_ERR_ARG;
    if (!b || (N > 0 && !topk_idx)) return MOE_ERR_ARG;
    int rc;
    moe::DeviceInfo *dev = nullptr;
    if ((rc = moe::current_device_info(&dev)) != MOE_OK) return rc;
    if (dev->major != 10) return MOE_ERR_NO_DEVICE;
    moe::bias_update_kernel<<<1, moe::BIAS_THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
        topk_idx, N * k, E, rate, b, loads_out);
    return moe::launch_status();
}

size_t moe_forward_workspace(int N, int D, int E, int d_moe, int d_sh, int k, int dtype) {
    WsLayout L;
    if (!plan_workspace(N, D, E, d_moe, d_sh, k, dtype, L)) return 0;
    return L.total;
}

size_t moe_layer_forward_workspace(int N, int D, int E, int d_moe, int d_sh, int k, int dtype,
                                   int wg_dtype) {
    if (wg_dtype != MOE_F32 && wg_dtype != MOE_BF16) return 0;
    WsLayout L;
    if (!plan_workspace(N, D, E, d_moe, d_sh, k, dtype, L, wg_dtype == MOE_F32)) return 0;
    return L.total_with_parts;
}

}  // extern "C"

namespace moe {
namespace {

// Validates the forward's arguments (nothing is launched on an error) and plans
// its workspace.
int check_forward(const void *x, const void *gate_up, const void *down, const void *sh_gate,
                  const void *sh_up, const void *sh_down, const int32_t *topk_idx,
                  const float *topk_w, int N, int D, int E, int d_moe, int d_sh, int k, int dtype,
                  const void *y, const void *workspace, size_t ws_bytes, WsLayout &L) {
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_DTYPE;
    if (N < 0 || D <= 0 || E <= 0 || E > DISPATCH_MAXE || d_moe <= 0 || d_sh <= 0 || k <= 0 ||
        k > 32)
        return MOE_ERR_SHAPE;
    if (dtype == MOE_BF16 && (D % 8 || d_moe % 8 || d_sh % 8)) return MOE_ERR_SHAPE;
    if (dtype == MOE_F32 && (D % 4)) return MOE_ERR_SHAPE;
    if (!plan_workspace(N, D, E, d_moe, d_sh, k, dtype, L)) return MOE_ERR_SHAPE;
    if (N == 0) return MOE_OK;
    const void *ptrs[] = {x, gate_up, down, sh_gate, sh_up, sh_down, topk_idx, topk_w, y};
    for (const void *q : ptrs)
        if (!q || !aligned16(q)) return MOE_ERR_ARG;
    if (!workspace || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MOE_ERR_WORKSPACE;
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

// Dispatch fields of the workspace (the same for the standalone and the fused dispatch).
DispatchParams dispatch_params(const WsLayout &L, uint8_t *ws, const int32_t *topk_idx,
                               const float *topk_w, int N, int k, int E) {
    DispatchParams dp;
    dp.topk_idx = topk_idx;
    dp.topk_w = topk_w;
    dp.N = N;
    dp.k = k;
    dp.E = E;
    dp.nchunks = L.nchunks;
    dp.tile_rows = L.tile_rows;
    dp.chunk_hist = reinterpret_cast<int32_t *>(ws + L.chunk_hist);
    dp.counts = reinterpret_cast<int32_t *>(ws + L.counts);
    dp.tile_off = reinterpret_cast<int32_t *>(ws + L.tile_off);
    dp.meta = reinterpret_cast<int32_t *>(ws + L.meta);
    dp.pos_of = reinterpret_cast<int32_t *>(ws + L.pos_of);
    dp.perm_tok = reinterpret_cast<int32_t *>(ws + L.perm_tok);
    dp.w_perm = reinterpret_cast<float *>(ws + L.w_perm);
    return dp;
}

// The forward after routing.  prof_in: the caller's profiler (its marks continue);
// dispatched: the router already ran the dispatch and gather (fused path).
int forward_impl(const void *x, const void *gate_up, const void *down, const void *sh_gate,
                 const void *sh_up, const void *sh_down, const int32_t *topk_idx,
                 const float *topk_w, int N, int D, int E, int d_moe, int d_sh, int k, int dtype,
                 float gate_max, float up_max, void *y, void *workspace, size_t ws_bytes,
                 void *stream, Profiler *prof_in = nullptr, bool dispatched = false) {
    WsLayout L;
    int rc = check_forward(x, gate_up, down, sh_gate, sh_up, sh_down, topk_idx, topk_w, N, D, E,
                           d_moe, d_sh, k, dtype, y, workspace, ws_bytes, L);
    if (rc != MOE_OK || N == 0) return rc;
    DeviceInfo *dev = nullptr;
    if ((rc = current_device_info(&dev)) != MOE_OK) return rc;
    if (dev->major != 10) return MOE_ERR_NO_DEVICE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    Profiler prof_own(st, prof_in == nullptr);
    Profiler &prof = prof_in ? *prof_in : prof_own;

    const DispatchParams dp = dispatch_params(L, ws, topk_idx, topk_w, N, k, E);

    if (dispatched) {
        // count, scan, scatter (and the gather below) ran inside the router kernel
        prof.mark();
        prof.mark();
        prof.mark();
    } else if ((size_t)N * k <= DISPATCH_SMALL_IDS) {
        // one CTA does count, scan and scatter (the three profiling marks coincide)
        dispatch_small_kernel<<<1, DISPATCH_SMALL_THREADS, 0, st>>>(dp);
        if ((rc = launched(prof)) != MOE_OK) return rc;
        prof.mark();
        prof.mark();
    } else {
        dispatch_count_kernel<<<L.nchunks, DISPATCH_THREADS, 0, st>>>(dp);
        if ((rc = launched(prof)) != MOE_OK) return rc;
        dispatch_scan_kernel<<<1, DISPATCH_MAXE, 0, st>>>(dp);
        if ((rc = launched(prof)) != MOE_OK) return rc;
        dispatch_scatter_kernel<<<L.nchunks, DISPATCH_THREADS, 0, st>>>(dp);
        if ((rc = launched(prof)) != MOE_OK) return rc;
    }

    if (dtype == MOE_F32) {
        SimtArgs a;
        a.x = static_cast<const float *>(x);
        a.gate_up = static_cast<const float *>(gate_up);
        a.down = static_cast<const float *>(down);
        a.sh_gate = static_cast<const float *>(sh_gate);
        a.sh_up = static_cast<const float *>(sh_up);
        a.sh_down = static_cast<const float *>(sh_down);
        a.perm_tok = dp.perm_tok;
        a.counts = dp.counts;
        a.tile_off = dp.tile_off;
        a.meta = dp.meta;
        a.pos_of = dp.pos_of;
        a.w_perm = dp.w_perm;
        a.h_perm = reinterpret_cast<float *>(ws + L.h_perm);
        a.h_sh = reinterpret_cast<float *>(ws + L.h_sh);
        a.slot = reinterpret_cast<float *>(ws + L.slot);
        a.y = static_cast<float *>(y);
        a.N = N;
        a.D = D;
        a.E = E;
        a.d = d_moe;
        a.d_sh = d_sh;
        a.k = k;
        a.gate_max = gate_max;
        a.up_max = up_max;
        const int rblocks = (int)(L.rows_max / SIMT_T);
        const int nblocks = (N + SIMT_T - 1) / SIMT_T;
        simt_expert_kernel<SIMT_GATEUP_R><<<dim3(rblocks, (d_moe + 31) / 32), 256, 0, st>>>(a);
        if ((rc = launched(prof)) != MOE_OK) return rc;
        simt_expert_kernel<SIMT_GATEUP_S><<<dim3(nblocks, (d_sh + 31) / 32), 256, 0, st>>>(a);
        if ((rc = launched(prof)) != MOE_OK) return rc;
        simt_expert_kernel<SIMT_DOWN_R><<<dim3(rblocks, (D + 31) / 32), 256, 0, st>>>(a);
        if ((rc = launched(prof)) != MOE_OK) return rc;
        simt_expert_kernel<SIMT_DOWN_S><<<dim3(nblocks, (D + 31) / 32), 256, 0, st>>>(a);
        if ((rc = launched(prof)) != MOE_OK) return rc;
        const size_t total = (size_t)N * D;
        const int cblocks = (int)std::min<size_t>((total + 255) / 256, (size_t)dev->sms * 16);
        simt_combine_kernel<<<cblocks, 256, 0, st>>>(a);
        return launched(prof);
    }

    // ---- bf16 tensor-core path ----
    uint8_t *x_perm = ws + L.x_perm;
    if (dispatched) {
        prof.mark();
    } else {
        const int items = N * ((D * 2 / 16 + 127) / 128); // 2 KiB pieces of token rows
        const int grid = std::min((items + 7) / 8, dev->sms * 16);
        dispatch_gather_kernel<<<grid, 256, 0, st>>>(static_cast<const uint8_t *>(x), x_perm, dp,
                                                    D * 2);
        if ((rc = launched(prof)) != MOE_OK) return rc;
    }
    __nv_bfloat16 *h_perm = reinterpret_cast<__nv_bfloat16 *>(ws + L.h_perm);
    __nv_bfloat16 *h_sh = reinterpret_cast<__nv_bfloat16 *>(ws + L.h_sh);
    __nv_bfloat16 *slot = reinterpret_cast<__nv_bfloat16 *>(ws + L.slot);

    if (L.decode) {
        if ((rc = ensure_decode_attrs(dev)) != MOE_OK) return rc;
        CUtensorMap mgu, mx_perm, msg, msu, mx, mdn, mh_perm, msd, mh_sh;
        const bool ok =
            make_map(&mgu, gate_up, D, (uint64_t)E * 2 * d_moe, D, 64) &&
            make_map(&mx_perm, x_perm, D, L.rows_max, D, DEC_TT) &&
            make_map(&msg, sh_gate, D, d_sh, D, 64) && make_map(&msu, sh_up, D, d_sh, D, 64) &&
            make_map(&mx, x, D, N, D, DEC_TT) &&
            make_map(&mdn, down, d_moe, (uint64_t)E * D, d_moe, DEC_BM) &&
            make_map(&mh_perm, h_perm, d_moe, L.rows_max, d_moe, DEC_TT) &&
            make_map(&msd, sh_down, d_sh, D, d_sh, DEC_BM) &&
            make_map(&mh_sh, h_sh, d_sh, N, d_sh, DEC_TT);
        if (!ok) return MOE_ERR_CUDA;
        const int tt_max = (int)(L.rows_max / DEC_TT);
        DecArgs g = {};
        g.tile_off = dp.tile_off;
        g.counts = dp.counts;
        g.meta = dp.meta;
        g.E = E;
        g.N = N;
        g.k = k;
        g.tt_s = (N + DEC_TT - 1) / DEC_TT;
        g.wait_limit_ns = g_wait_limit_ns;
        g.never_signal = g_never_signal;
        g.gate_max = gate_max;
        g.up_max = up_max;
        // gate_up + SwiGLU: 64 features x 32 tokens per tile
        g.nb_r = (d_moe + 63) / 64;
        g.nb_s = (d_sh + 63) / 64;
        g.kb_r = g.kb_s = (D + DEC_BK - 1) / DEC_BK;
        g.a_rows_per_e = 2 * d_moe;
        g.up_off = d_moe;
        g.out_r = h_perm;
        g.ld_r = g.ncols_r = d_moe;
        g.out_s = h_sh;
        g.ld_s = g.ncols_s = d_sh;
        int max_tiles = tt_max * g.nb_r + g.tt_s * g.nb_s;
        rc = launch_decode<GEMM_GATE_UP>(mgu, mx_perm, msg, msu, mx, g,
                                         std::min(dev->sms, max_tiles), false, st);
        prof.mark();
        if (rc != MOE_OK) return rc;
        // down + weighted slot partials + shared expert + combine: 128 features x 32 tokens
        g.nb_r = g.nb_s = (D + DEC_BM - 1) / DEC_BM;
        g.kb_r = (d_moe + DEC_BK - 1) / DEC_BK;
        g.kb_s = (d_sh + DEC_BK - 1) / DEC_BK;
        g.a_rows_per_e = D;
        g.up_off = 0;
        g.out_r = slot;
        g.ld_r = g.ncols_r = D;
        g.out_s = static_cast<__nv_bfloat16 *>(y);
        g.ld_s = g.ncols_s = D;
        g.w_perm = dp.w_perm;
        g.pos_of = dp.pos_of;
        g.slot = slot;
        max_tiles = tt_max * g.nb_r + g.tt_s * g.nb_s;
        rc = launch_decode<GEMM_DOWN>(mdn, mh_perm, msd, msd, mh_sh, g,
                                      std::min(dev->sms, max_tiles), true, st);
        prof.mark();
        prof.mark(); // the combine ran inside the down kernel
        return rc;
    }

    if ((rc = ensure_gemm_attrs(dev)) != MOE_OK) return rc;
    // CTA pairs by default for the down GEMM only, split by expert parity (mode
    // 4): on the configurations measured (two to four m-tiles per expert on
    // average) that made down 2-5 % faster, while gate_up on pairs was as often
    // slower as faster.  Splitting an expert's m-tiles between the two launches
    // (mode 1) streams its weights from HBM twice; padding odd m-tiles (mode 2)
    // wastes half an MMA tile.
    const int pair_mode = g_pair_mode < 0 ? kDefaultPairMode : g_pair_mode;
    bool pair = pair_mode >= 1;
    if (pair) {
        if ((rc = ensure_pair_attrs(dev)) != MOE_OK) return rc;
        pair = dev->pair_max_clusters > 0;
    }
    // padded pairs take every m-tile (no one-CTA launch); only if pairs can run
    const bool pad = pair && pair_mode == 2;
    // modes 3 and 4: the experts with an even m-tile count (and the shared expert
    // if its count is even) run wholly on pairs, the others wholly on the one-CTA
    // kernel, so no expert's weights are streamed by both launches; mode 4 does
    // this for the down GEMM only and runs gate_up on the one-CTA kernel
    const bool by_parity = pair && (pair_mode == 3 || pair_mode == 4);
    const bool pair_gu = pair && pair_mode != 4;
    const int pair_tiles_mode = pad ? GEMM_PAIR_PAD : by_parity ? GEMM_EVEN_EXPERTS : GEMM_ALL_TILES;
    const int rest_tiles_mode = by_parity ? GEMM_ODD_EXPERTS : GEMM_TAIL_TILES;
    CUtensorMap mx_perm, mgu, mx, msg, msu, mh_perm, mdn, mh_sh, msd, mdn2, msd2;
    bool ok = make_map(&mx_perm, x_perm, D, L.rows_max, D, 128) &&
              make_map(&mgu, gate_up, D, (uint64_t)E * 2 * d_moe, D, 128) &&
              make_map(&mx, x, D, N, D, 128) && make_map(&msg, sh_gate, D, d_sh, D, 128) &&
              make_map(&msu, sh_up, D, d_sh, D, 128) &&
              make_map(&mh_perm, h_perm, d_moe, L.rows_max, d_moe, 128) &&
              make_map(&mdn, down, d_moe, (uint64_t)E * D, d_moe, GEMM_BN) &&
              make_map(&mh_sh, h_sh, d_sh, N, d_sh, 128) &&
              make_map(&msd, sh_down, d_sh, D, d_sh, GEMM_BN) &&
              (!pair || (make_map(&mdn2, down, d_moe, (uint64_t)E * D, d_moe, 128) &&
                         make_map(&msd2, sh_down, d_sh, D, d_sh, 128)));
    if (!ok) return MOE_ERR_CUDA;

    const int mt_s = (N + GEMM_BM - 1) / GEMM_BM;
    const int mt_r_max = (int)(L.rows_max / GEMM_BM);
    GemmArgs g = {};
    g.tile_off = dp.tile_off;
    g.meta = dp.meta;
    g.E = E;
    g.N = N;
    g.k = k;
    g.mt_s = mt_s;
    g.wait_limit_ns = g_wait_limit_ns;
    g.never_signal = g_never_signal;
    g.gate_max = gate_max;
    g.up_max = up_max;
    // Launch sizes: the pair kernels take at most one pair tile per cluster; the
    // tail launch has at most one m-tile per expert (and one shared m-tile).
    const int pair_bound_mt = (mt_r_max + 1) / 2 + (mt_s + 1) / 2 + (pad ? E : 0);
    const int tail_bound_mt = std::min(E, mt_r_max) + 1;

    // gate_up + SwiGLU
    g.nb_r = (d_moe + 127) / 128;
    g.nb_s = (d_sh + 127) / 128;
    g.kb_r = g.kb_s = (D + GEMM_BK - 1) / GEMM_BK;
    g.b_rows_per_e = 2 * d_moe;
    g.up_off = d_moe;
    g.out_r = h_perm;
    g.ld_r = d_moe;
    g.ncols_r = d_moe;
    g.out_s = h_sh;
    g.ld_s = d_sh;
    g.ncols_s = d_sh;
    int max_tiles = mt_r_max * g.nb_r + mt_s * g.nb_s;
    g.mode = GEMM_ALL_TILES;
    if (pair_gu) {
        const int nbm = std::max(g.nb_r, g.nb_s);
        g.mode = pair_tiles_mode;
        rc = launch_gemm_pair<GEMM_GATE_UP>(mx_perm, mgu, mx, msg, msu, mx, g,
                                            std::min(dev->pair_max_clusters,
                                                     std::max(1, pair_bound_mt * nbm)), st);
        if (rc != MOE_OK) return rc;
        g.mode = rest_tiles_mode;
        if (!by_parity) max_tiles = tail_bound_mt * nbm;
    }
    if (!pad) {
        rc = launch_gemm<GEMM_GATE_UP>(mx_perm, mgu, mx, msg, msu, mx, g,
                                       std::min(dev->sms, max_tiles), false, st, pair_gu);
        if (rc != MOE_OK) return rc;
    }
    prof.mark();

    // down + weighted slot partials + shared expert + combine
    g.mode = GEMM_ALL_TILES;
    g.nb_r = g.nb_s = (D + GEMM_BN - 1) / GEMM_BN;
    g.kb_r = (d_moe + GEMM_BK - 1) / GEMM_BK;
    g.kb_s = (d_sh + GEMM_BK - 1) / GEMM_BK;
    g.b_rows_per_e = D;
    g.up_off = 0;
    g.out_r = slot;
    g.ld_r = D;
    g.ncols_r = D;
    g.out_s = static_cast<__nv_bfloat16 *>(y);
    g.ld_s = D;
    g.ncols_s = D;
    g.w_perm = dp.w_perm;
    g.pos_of = dp.pos_of;
    g.slot = slot;
    g.osh = reinterpret_cast<float *>(ws + L.osh);
    g.tma_out = 1;
    CUtensorMap mslot;
    if (!make_map_out(&mslot, slot, D, L.rows_max, D)) return MOE_ERR_CUDA;
    max_tiles = mt_r_max * g.nb_r + mt_s * g.nb_s;
    if (pair) {
        g.mode = pair_tiles_mode;
        rc = launch_gemm_pair<GEMM_DOWN>(mh_perm, mdn2, mh_sh, msd2, msd2, mslot, g,
                                         std::min(dev->pair_max_clusters,
                                                  std::max(1, pair_bound_mt * g.nb_r)), st);
        if (rc != MOE_OK) return rc;
        g.mode = rest_tiles_mode;
        if (!by_parity) max_tiles = tail_bound_mt * g.nb_r;
    }
    if (!pad) {
        rc = launch_gemm<GEMM_DOWN>(mh_perm, mdn, mh_sh, msd, msd, mslot, g,
                                    std::min(dev->sms, max_tiles), false, st, pair);
        if (rc != MOE_OK) return rc;
    }
    prof.mark();
    // y = slots in slot order + shared output, at many warps per SM
    combine_kernel<<<std::min((N + 7) / 8, dev->sms * 16), COMBINE_THREADS, 0, st>>>(g);
    return launched(prof);
}

}  // namespace
}  // namespace moe

extern "C" {

int moe_forward(const void *x, const void *gate_up, const void *down, const void *sh_gate,
                const void *sh_up, const void *sh_down, const int32_t *topk_idx,
                const float *topk_w, int N, int D, int E, int d_moe, int d_sh, int k, int dtype,
                void *y, void *workspace, size_t ws_bytes, void *stream) {
    return forward_impl(x, gate_up, down, sh_gate, sh_up, sh_down, topk_idx, topk_w, N, D, E,
                        d_moe, d_sh, k, dtype, INFINITY, INFINITY, y, workspace, ws_bytes, stream);
}

int moe_forward_clamped(const void *x, const void *gate_up, const void *down, const void *sh_gate,
                        const void *sh_up, const void *sh_down, const int32_t *topk_idx,
                        const float *topk_w, int N, int D, int E, int d_moe, int d_sh, int k,
                        int dtype, float gate_max, float up_max, void *y, void *workspace,
                        size_t ws_bytes, void *stream) {
    if (gate_max != gate_max || up_max != up_max || up_max < 0.f) return MOE_ERR_ARG;
    return forward_impl(x, gate_up, down, sh_gate, sh_up, sh_down, topk_idx, topk_w, N, D, E,
                        d_moe, d_sh, k, dtype, gate_max, up_max, y, workspace, ws_bytes, stream);
}

int moe_layer_forward(const void *x, const void *W_g, int wg_dtype, const float *b, int N, int D,
                      int E, int n_group, int topk_group, int k, int norm_topk_prob, float alpha,
                      const void *gate_up, const void *down, const void *sh_gate, const void *sh_up,
                      const void *sh_down, int d_moe, int d_sh, int dtype, int32_t *topk_idx,
                      float *topk_w, void *y, void *workspace, size_t ws_bytes, void *stream) {
    using namespace moe;
    int rc = check_router_shape(N, D, E, n_group, topk_group, k);
    if (rc != MOE_OK) return rc;
    if (wg_dtype != MOE_F32 && wg_dtype != MOE_BF16) return MOE_ERR_DTYPE;
    WsLayout L;
    if ((rc = check_forward(x, gate_up, down, sh_gate, sh_up, sh_down, topk_idx, topk_w, N, D, E,
                            d_moe, d_sh, k, dtype, y, workspace, ws_bytes, L)) != MOE_OK)
        return rc;
    if (N == 0) return MOE_OK;
    // The split-once scratch for an fp32 W_g is used when the workspace covers it
    // (moe_layer_forward_workspace); with moe_forward_workspace bytes the router
    // splits W_g in every token block instead (the same routing, bit for bit).
    WsLayout Lp;
    plan_workspace(N, D, E, d_moe, d_sh, k, dtype, Lp, wg_dtype == MOE_F32);
    void *wg_parts_ws = wg_dtype == MOE_F32 && ws_bytes >= Lp.total_with_parts
                            ? static_cast<void *>(static_cast<uint8_t *>(workspace) + Lp.wg_parts)
                            : nullptr;
    if (!W_g || !b || !aligned16(W_g) || !aligned16(b)) return MOE_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    Profiler prof(st);
    // bf16 decode layers of one token block: dispatch and gather inside the router
    RtcFuse fz = {};
    if (dtype == MOE_BF16 && L.decode && (size_t)N * k <= DISPATCH_SMALL_IDS) {
        fz.dp = dispatch_params(L, ws, topk_idx, topk_w, N, k, E);
        fz.x = static_cast<const uint8_t *>(x);
        fz.x_perm = ws + L.x_perm;
        fz.row_bytes = D * 2;
        fz.on = 1;
    }
    bool fused = false;
    rc = router_impl(x, dtype, W_g, wg_dtype, b, N, D, E, n_group, topk_group, k, norm_topk_prob,
                     alpha, topk_idx, topk_w, stream, &fz, &fused, wg_parts_ws);
    if (rc != MOE_OK) return rc;
    prof.mark();
    return forward_impl(x, gate_up, down, sh_gate, sh_up, sh_down, topk_idx, topk_w, N, D, E, d_moe,
                        d_sh, k, dtype, INFINITY, INFINITY, y, workspace, ws_bytes, stream, &prof,
                        fused);
}

int moe_device_status(void *stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    DevStatus s;
    if (cudaMemcpyFromSymbol(&s, g_status, sizeof(s)) != cudaSuccess) return MOE_ERR_CUDA;
    const DevStatus zero = {0, 0, 0, 0};
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return MOE_ERR_CUDA;
    if (s.error == DEV_TIMEOUT) return MOE_ERR_DEVICE_TIMEOUT;
    if (s.error == DEV_BAD_INDEX) return MOE_ERR_BAD_INDEX;
    return MOE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Expert parallelism (peer memory): workspace, launch sequence, IPC mapping.
// ---------------------------------------------------------------------------
namespace moe {
namespace {

struct EpWs {
    size_t chunk_hist, counts, dense_off, dmeta, pos_of, perm_tok, w_perm;
    size_t dest_base, rcounts, rtile_off, rmeta, pair_pos;
    size_t h_perm, h_sh, osh, total;
    int nchunks;
};

bool plan_ep(int P, int N_cap, int D, int E, int d, int d_sh, int k, EpSym &S, EpWs &W) {
    if (!ep_sym_layout(P, N_cap, D, E, k, S)) return false;
    if (d <= 0 || d_sh <= 0) return false;
    const size_t nk = (size_t)N_cap * k;
    if (nk > (size_t)INT32_MAX / 4) return false;
    W.nchunks = (int)((nk + DISPATCH_CHUNK - 1) / DISPATCH_CHUNK);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = round_up(off + bytes, 256);
        return at;
    };
    const int E_loc = E / P;
    W.chunk_hist = take((size_t)std::max(W.nchunks, 1) * E * 4);
    W.counts = take((size_t)E * 4);
    W.dense_off = take((size_t)(E + 1) * 4);
    W.dmeta = take(16 * 4);
    W.pos_of = take(std::max<size_t>(nk, 1) * 4);
    W.perm_tok = take(std::max<size_t>(nk, 1) * 4);
    W.w_perm = take(std::max<size_t>(nk, 1) * 4);
    W.dest_base = take((size_t)E * 4);
    W.rcounts = take((size_t)E_loc * 4);
    W.rtile_off = take((size_t)(E_loc + 1) * 4);
    W.rmeta = take(16 * 4);
    W.pair_pos = take(std::max<size_t>(nk, 1) * 4);
    W.h_perm = take((size_t)S.rows_cap * d * 2);
    W.h_sh = take(std::max<size_t>((size_t)N_cap * d_sh * 2, 16));
    W.osh = take(std::max<size_t>((size_t)N_cap * D * 4, 16));
    W.total = off;
    return true;
}

int ep_forward_impl(int phases, int P, int rank, uint32_t epoch, void *const *peer_sym, int N_cap,
                    const void *x, const void *gate_up_loc, const void *down_loc,
                    const void *sh_gate, const void *sh_up, const void *sh_down,
                    const int32_t *topk_idx, const float *topk_w, int N, int D, int E, int d_moe,
                    int d_sh, int k, void *y, void *workspace, size_t ws_bytes, void *stream) {
    if (phases <= 0 || phases > MOE_EP_ALL) return MOE_ERR_ARG;
    if (P < 1 || P > EP_MAX_RANKS || rank < 0 || rank >= P || epoch == 0) return MOE_ERR_ARG;
    if (E <= 0 || E > DISPATCH_MAXE || E % P || k <= 0 || k > 32 || k > E) return MOE_ERR_SHAPE;
    if (N < 0 || N > N_cap || D <= 0 || d_moe <= 0 || d_sh <= 0) return MOE_ERR_SHAPE;
    if (D % 8 || d_moe % 8 || d_sh % 8) return MOE_ERR_SHAPE;
    EpSym S;
    EpWs W;
    if (!plan_ep(P, N_cap, D, E, d_moe, d_sh, k, S, W)) return MOE_ERR_SHAPE;
    if (!peer_sym) return MOE_ERR_ARG;
    for (int q = 0; q < P; ++q)
        if (!peer_sym[q] || (reinterpret_cast<uintptr_t>(peer_sym[q]) & 255u)) return MOE_ERR_ARG;
    const void *ptrs[] = {gate_up_loc, down_loc, sh_gate, sh_up, sh_down};
    for (const void *q : ptrs)
        if (!q || !aligned16(q)) return MOE_ERR_ARG;
    if (N > 0) {
        const void *io[] = {x, topk_idx, topk_w, y};
        for (const void *q : io)
            if (!q || !aligned16(q)) return MOE_ERR_ARG;
    }
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return MOE_ERR_WORKSPACE;
    if (ws_bytes < W.total) return MOE_ERR_WORKSPACE;
    int rc;
    DeviceInfo *dev = nullptr;
    if ((rc = current_device_info(&dev)) != MOE_OK) return rc;
    if (dev->major != 10) return MOE_ERR_NO_DEVICE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    Profiler prof(st);
    const int E_loc = E / P;
    const int par = epoch & 1;

    EpParams ep = {};
    ep.P = P;
    ep.rank = rank;
    ep.E = E;
    ep.E_loc = E_loc;
    ep.k = k;
    ep.N = N;
    ep.D = D;
    ep.epoch = epoch;
    for (int q = 0; q < P; ++q) ep.sym[q] = static_cast<uint8_t *>(peer_sym[q]);
    ep.S = S;
    ep.x = static_cast<const uint8_t *>(x);
    ep.topk_idx = topk_idx;
    ep.topk_w = topk_w;
    ep.counts = reinterpret_cast<int32_t *>(ws + W.counts);
    ep.dense_off = reinterpret_cast<int32_t *>(ws + W.dense_off);
    ep.pos_of = reinterpret_cast<int32_t *>(ws + W.pos_of);
    ep.dest_base = reinterpret_cast<int32_t *>(ws + W.dest_base);
    ep.rcounts = reinterpret_cast<int32_t *>(ws + W.rcounts);
    ep.rtile_off = reinterpret_cast<int32_t *>(ws + W.rtile_off);
    ep.rmeta = reinterpret_cast<int32_t *>(ws + W.rmeta);
    ep.pair_pos = reinterpret_cast<int32_t *>(ws + W.pair_pos);
    ep.down_nb = (D + GEMM_BN - 1) / GEMM_BN;
    ep.wait_limit_ns = g_wait_limit_ns;

    if (phases & MOE_EP_COUNT) {
        // dense dispatch of this rank's pairs (one-row tiles: positions are
        // expert-sorted with no padding)
        DispatchParams dp;
        dp.topk_idx = topk_idx;
        dp.topk_w = topk_w;
        dp.N = N;
        dp.k = k;
        dp.E = E;
        dp.nchunks = W.nchunks;
        dp.tile_rows = 1;
        dp.chunk_hist = reinterpret_cast<int32_t *>(ws + W.chunk_hist);
        dp.counts = reinterpret_cast<int32_t *>(ws + W.counts);
        dp.tile_off = reinterpret_cast<int32_t *>(ws + W.dense_off);
        dp.meta = reinterpret_cast<int32_t *>(ws + W.dmeta);
        dp.pos_of = reinterpret_cast<int32_t *>(ws + W.pos_of);
        dp.perm_tok = reinterpret_cast<int32_t *>(ws + W.perm_tok);
        dp.w_perm = reinterpret_cast<float *>(ws + W.w_perm);
        if ((size_t)N * k <= DISPATCH_SMALL_IDS) {
            dispatch_small_kernel<<<1, DISPATCH_SMALL_THREADS, 0, st>>>(dp);
            if ((rc = launched(prof)) != MOE_OK) return rc;
        } else {
            dp.nchunks = (int)(((size_t)N * k + DISPATCH_CHUNK - 1) / DISPATCH_CHUNK);
            dispatch_count_kernel<<<dp.nchunks, DISPATCH_THREADS, 0, st>>>(dp);
            if ((rc = launched(prof)) != MOE_OK) return rc;
            dispatch_scan_kernel<<<1, DISPATCH_MAXE, 0, st>>>(dp);
            if ((rc = launched(prof)) != MOE_OK) return rc;
            dispatch_scatter_kernel<<<dp.nchunks, DISPATCH_THREADS, 0, st>>>(dp);
            if ((rc = launched(prof)) != MOE_OK) return rc;
        }
        ep_publish_kernel<<<1, 512, 0, st>>>(ep);
        if ((rc = launched(prof)) != MOE_OK) return rc;
    }
    if (phases & MOE_EP_SEND) {
        ep_layout_kernel<<<1, 512, 0, st>>>(ep);
        if ((rc = launched(prof)) != MOE_OK) return rc;
        if (N > 0) {
            const int items = N * ((D * 2 / 16 + EP_PIECE_VEC - 1) / EP_PIECE_VEC);
            const int grid = std::min((items + 7) / 8, dev->sms * 16);
            ep_send_kernel<<<grid, 256, 0, st>>>(ep);
            if ((rc = launched(prof)) != MOE_OK) return rc;
        }
    }
    uint8_t *own = ep.sym[rank];
    if (phases & MOE_EP_EXPERTS) {
        if ((rc = ensure_gemm_attrs(dev)) != MOE_OK) return rc;
        const void *recv_x = own + S.recv_x;
        __nv_bfloat16 *h_perm = reinterpret_cast<__nv_bfloat16 *>(ws + W.h_perm);
        __nv_bfloat16 *h_sh = reinterpret_cast<__nv_bfloat16 *>(ws + W.h_sh);
        const uint64_t nrows = std::max(N, 1); // maps need a row; no tile reads past N
        CUtensorMap mx_perm, mgu, mx, msg, msu, mh_perm, mdn, mh_sh, msd;
        const bool ok = make_map(&mx_perm, recv_x, D, S.rows_cap, D, 128) &&
                        make_map(&mgu, gate_up_loc, D, (uint64_t)E_loc * 2 * d_moe, D, 128) &&
                        make_map(&mx, N > 0 ? x : recv_x, D, nrows, D, 128) &&
                        make_map(&msg, sh_gate, D, d_sh, D, 128) &&
                        make_map(&msu, sh_up, D, d_sh, D, 128) &&
                        make_map(&mh_perm, h_perm, d_moe, S.rows_cap, d_moe, 128) &&
                        make_map(&mdn, down_loc, d_moe, (uint64_t)E_loc * D, d_moe, GEMM_BN) &&
                        make_map(&mh_sh, h_sh, d_sh, nrows, d_sh, 128) &&
                        make_map(&msd, sh_down, d_sh, D, d_sh, GEMM_BN);
        if (!ok) return MOE_ERR_CUDA;
        const int mt_s = (N + GEMM_BM - 1) / GEMM_BM;
        const int mt_r_max = S.rows_cap / GEMM_BM;
        GemmArgs g = {};
        g.tile_off = ep.rtile_off;
        g.meta = ep.rmeta;
        g.E = E_loc;
        g.N = N;
        g.k = k;
        g.mt_s = mt_s;
        g.wait_limit_ns = g_wait_limit_ns;
        g.gate_max = INFINITY;
        g.up_max = INFINITY;
        g.nb_r = (d_moe + 127) / 128;
        g.nb_s = (d_sh + 127) / 128;
        g.kb_r = g.kb_s = (D + GEMM_BK - 1) / GEMM_BK;
        g.b_rows_per_e = 2 * d_moe;
        g.up_off = d_moe;
        g.out_r = h_perm;
        g.ld_r = g.ncols_r = d_moe;
        g.out_s = h_sh;
        g.ld_s = g.ncols_s = d_sh;
        g.ep_wait_ctr = reinterpret_cast<const uint32_t *>(own + S.ctr) + par;
        g.ep_wait_target = ep.rmeta + 3;
        int max_tiles = mt_r_max * g.nb_r + mt_s * g.nb_s;
        rc = launch_gemm<GEMM_GATE_UP>(mx_perm, mgu, mx, msg, msu, mx, g,
                                       std::min(dev->sms, max_tiles), false, st);
        prof.mark();
        if (rc != MOE_OK) return rc;
        g.ep_wait_ctr = nullptr;
        g.ep_wait_target = nullptr;
        g.nb_r = g.nb_s = (D + GEMM_BN - 1) / GEMM_BN;
        g.kb_r = (d_moe + GEMM_BK - 1) / GEMM_BK;
        g.kb_s = (d_sh + GEMM_BK - 1) / GEMM_BK;
        g.b_rows_per_e = D;
        g.up_off = 0;
        g.out_r = nullptr;
        g.ld_r = g.ncols_r = D;
        g.out_s = static_cast<__nv_bfloat16 *>(y);
        g.ld_s = g.ncols_s = D;
        g.osh = reinterpret_cast<float *>(ws + W.osh);
        g.ep_P = P;
        g.ep_meta = reinterpret_cast<const int4 *>(own + S.recv_meta);
        for (int q = 0; q < P; ++q) {
            g.ep_out[q] = reinterpret_cast<__nv_bfloat16 *>(ep.sym[q] + S.slot);
            g.ep_ret[q] = reinterpret_cast<uint32_t *>(ep.sym[q] + S.ctr) + 2 + par;
        }
        max_tiles = mt_r_max * g.nb_r + mt_s * g.nb_s;
        rc = launch_gemm<GEMM_DOWN>(mh_perm, mdn, mh_sh, msd, msd, msd, g,
                                    std::min(dev->sms, max_tiles), true, st);
        prof.mark();
        if (rc != MOE_OK) return rc;
    }
    if ((phases & MOE_EP_COMBINE) && N > 0) {
        GemmArgs g = {};
        g.N = N;
        g.k = k;
        g.ncols_s = g.ld_s = D;
        g.ld_r = D;
        g.out_s = static_cast<__nv_bfloat16 *>(y);
        g.osh = reinterpret_cast<float *>(ws + W.osh);
        g.pos_of = ep.pair_pos;
        g.slot = reinterpret_cast<const __nv_bfloat16 *>(own + S.slot);
        const int grid = std::min((N + 7) / 8, dev->sms * 4);
        ep_combine_kernel<<<grid, 256, 0, st>>>(ep, g);
        if ((rc = launched(prof)) != MOE_OK) return rc;
    }
    return MOE_OK;
}

// Host mirror of the layout the send phase derives on the device (see
// ep_layout_kernel), for checks of the exchange logic without a GPU.
int ep_plan_host(int P, int rank, int E, const int32_t *counts, int32_t *dest_base,
                 int32_t *rcounts, int32_t *rtile_off, int32_t *rows_in, int32_t *pairs_out) {
    if (P < 1 || P > EP_MAX_RANKS || rank < 0 || rank >= P || E <= 0 || E % P) return MOE_ERR_SHAPE;
    if (!counts || !dest_base || !rcounts || !rtile_off || !rows_in || !pairs_out) return MOE_ERR_ARG;
    const int E_loc = E / P;
    int dense = 0, rin = 0, pout = 0;
    for (int e = 0; e < E; ++e) {
        const int q = e / E_loc, first = q * E_loc;
        int tprefix = 0;
        for (int e2 = first; e2 < e; ++e2) {
            int R2 = 0;
            for (int r = 0; r < P; ++r) R2 += counts[(size_t)r * E + e2];
            tprefix += (R2 + EP_TILE - 1) / EP_TILE;
        }
        int R = 0, pre = 0;
        for (int r = 0; r < P; ++r) {
            R += counts[(size_t)r * E + e];
            if (r < rank) pre += counts[(size_t)r * E + e];
        }
        dest_base[e] = tprefix * EP_TILE + pre - dense;
        dense += counts[(size_t)rank * E + e];
        pout += counts[(size_t)rank * E + e];
        if (q == rank) {
            rcounts[e - first] = R;
            rtile_off[e - first] = tprefix;
            rin += R;
            if (e - first == E_loc - 1) rtile_off[E_loc] = tprefix + (R + EP_TILE - 1) / EP_TILE;
        }
    }
    *rows_in = rin;
    *pairs_out = pout;
    return MOE_OK;
}

using PFN_getAddressRange = CUresult (*)(CUdeviceptr *, size_t *, CUdeviceptr);

PFN_getAddressRange address_range_fn() {
    static PFN_getAddressRange fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_getAddressRange>(p);
    });
    return fn;
}

}  // namespace
}  // namespace moe

extern "C" {

size_t moe_ep_symmetric_bytes(int P, int N_cap, int D, int E, int k) {
    moe::EpSym S;
    return moe::ep_sym_layout(P, N_cap, D, E, k, S) ? S.total : 0;
}

size_t moe_ep_workspace_bytes(int P, int N_cap, int D, int E, int d_moe, int d_sh, int k) {
    moe::EpSym S;
    moe::EpWs W;
    return moe::plan_ep(P, N_cap, D, E, d_moe, d_sh, k, S, W) ? W.total : 0;
}

int moe_ep_forward(int phases, int P, int rank, unsigned epoch, void *const *peer_sym, int N_cap,
                   const void *x, const void *gate_up_loc, const void *down_loc,
                   const void *sh_gate, const void *sh_up, const void *sh_down,
                   const int32_t *topk_idx, const float *topk_w, int N, int D, int E, int d_moe,
                   int d_sh, int k, void *y, void *workspace, size_t ws_bytes, void *stream) {
    return moe::ep_forward_impl(phases, P, rank, epoch, peer_sym, N_cap, x, gate_up_loc, down_loc,
                                sh_gate, sh_up, sh_down, topk_idx, topk_w, N, D, E, d_moe, d_sh, k,
                                y, workspace, ws_bytes, stream);
}

int moe_ep_plan_host(int P, int rank, int E, const int32_t *counts, int32_t *dest_base,
                     int32_t *rcounts, int32_t *rtile_off, int32_t *rows_in, int32_t *pairs_out) {
    return moe::ep_plan_host(P, rank, E, counts, dest_base, rcounts, rtile_off, rows_in, pairs_out);
}

int moe_ep_ipc_export(const void *dev_ptr, void *handle) {
    if (!dev_ptr || !handle) return MOE_ERR_ARG;
    auto range = moe::address_range_fn();
    if (!range) return MOE_ERR_CUDA;
    CUdeviceptr base = 0;
    size_t size = 0;
    if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS) return MOE_ERR_CUDA;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base)) != cudaSuccess) return MOE_ERR_CUDA;
    const uint64_t offset = reinterpret_cast<CUdeviceptr>(dev_ptr) - base;
    std::memcpy(handle, &h, sizeof(h));
    std::memcpy(static_cast<uint8_t *>(handle) + sizeof(h), &offset, sizeof(offset));
    return MOE_OK;
}

int moe_ep_ipc_open(const void *handle, void **dev_ptr) {
    if (!handle || !dev_ptr) return MOE_ERR_ARG;
    cudaIpcMemHandle_t h;
    uint64_t offset = 0;
    std::memcpy(&h, handle, sizeof(h));
    std::memcpy(&offset, static_cast<const uint8_t *>(handle) + sizeof(h), sizeof(offset));
    void *base = nullptr;
    if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess)
        return MOE_ERR_CUDA;
    *dev_ptr = static_cast<uint8_t *>(base) + offset;
    return MOE_OK;
}

int moe_ep_ipc_close(void *dev_ptr) {
    if (!dev_ptr) return MOE_ERR_ARG;
    auto range = moe::address_range_fn();
    if (!range) return MOE_ERR_CUDA;
    CUdeviceptr base = 0;
    size_t size = 0;
    if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS) return MOE_ERR_CUDA;
    return cudaIpcCloseMemHandle(reinterpret_cast<void *>(base)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
