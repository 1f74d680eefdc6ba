/*
 * moe.h — C ABI of the B200 (sm_100a) sparse mixture-of-experts FFN forward
 * (GLM-4.5 / GLM-5 style): a sigmoid router with a loss-free correction bias and
 * group-restricted top-k, token dispatch, routed SwiGLU experts, a
 * routing-weighted combine and an always-on shared expert:
 *
 *     y_n = sum_{i in T(n)} w_{n,i} E_i(x_n) + E_sh(x_n)
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers to caller-owned, contiguous,
 *     row-major memory.  The library never allocates, frees or retains them.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls only enqueue work and return; results are ready when the stream is.
 *   - Argument and shape errors are reported synchronously, before any launch;
 *     nothing is written then.  Launch failures return MOE_ERR_CUDA.  Errors
 *     found by the kernels themselves (an out-of-range expert id, a bounded wait
 *     that ran out) are recorded in a device status word that
 *     moe_device_status() reads.
 *   - Pointers must be 16-byte aligned.  For bf16 tensors the row lengths D,
 *     d_moe and d_sh must be multiples of 8 (16-byte rows for TMA).
 *   - Calls on one device may overlap only if they are on one stream: the
 *     kernels share nothing across calls except the status word, but two
 *     moe_forward calls must not share a workspace while both are in flight.
 *   - Stream order is kept.  Some kernels use programmatic dependent launch
 *     (the tensor-core router, the decode gate_up kernel).  They may be resident
 *     before the previous work on the stream ends, but they touch no memory until
 *     it has completed.  Kernels of this library also release their own
 *     successors early (griddepcontrol.launch_dependents).  So a caller's kernel
 *     launched right after with programmatic stream serialization must wait for
 *     its predecessor (griddepcontrol.wait / cudaGridDependencySynchronize)
 *     before it reads the outputs, as that launch mode requires anyway.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element types of the tensors handed across the boundary. */
typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_ARG = -1,            /* null pointer, misaligned pointer, bad flag */
    MOE_ERR_SHAPE = -2,          /* inconsistent or unsupported sizes */
    MOE_ERR_DTYPE = -3,          /* unsupported dtype combination */
    MOE_ERR_WORKSPACE = -4,      /* workspace missing or smaller than required */
    MOE_ERR_CUDA = -5,           /* a CUDA runtime call or launch failed */
    MOE_ERR_DEVICE_TIMEOUT = -6, /* a bounded device-side wait ran out */
    MOE_ERR_BAD_INDEX = -7,      /* topk_idx held an id outside [0, E]; skipped */
    MOE_ERR_NO_DEVICE = -8       /* no sm_100 device is current */
} moe_status;

/*
 * moe_router — group-restricted sigmoid router.
 * Defined by "GLM-4.5 Group Router", How it works: r = x W_g^T in float32,
 * s = sigmoid(r), s' = s + b (the correction bias is used for selection only),
 * the E experts form n_group contiguous groups of E/n_group, a group scores the
 * sum of its two largest s', the topk_group best groups are kept, T = the k
 * largest s' inside them, and w_i = alpha * s_i / (sum_{j in T} s_j + 1e-20)
 * when norm_topk_prob (else alpha * s_i).  n_group = topk_group = 1 is plain
 * top-k.  alpha is applied here and nowhere else ("GLM-4.5 MoE Forward",
 * note on applying routed_scaling_factor once).
 *
 *   x        [N, D]   x_dtype (MOE_F32 or MOE_BF16)
 *   W_g      [E, D]   wg_dtype (MOE_F32 or MOE_BF16)
 *   b        [E]      fp32 correction bias
 *   topk_idx [N, k]   int32 out: expert ids, ordered by descending s', ties to
 *                     the lower id; never the sentinel E
 *   topk_w   [N, k]   fp32 out: mixture weights matching topk_idx, alpha included
 * Sizes: 1 <= E <= 512, E % n_group == 0, E / n_group >= 2 when n_group > 1,
 * 1 <= topk_group <= n_group, 1 <= k <= min(32, topk_group * E / n_group),
 * n_group <= 64, D >= 1.  N = 0 is a no-op.
 * Logits accumulate in fp32 (bf16 x bf16 and bf16 x fp32 products are exact in
 * fp32), so ids agree with an exact evaluation except where two candidates'
 * s' lie within fp32 rounding of each other.
 */
int moe_router(const void *x, int x_dtype, const void *W_g, int wg_dtype, const float *b,
               int N, int D, int E, int n_group, int topk_group, int k, int norm_topk_prob,
               float alpha, int32_t *topk_idx, float *topk_w, void *stream);

/*
 * moe_forward_workspace — bytes of device workspace moe_forward needs for these
 * sizes (0 for invalid sizes).  The workspace holds the dispatch tables, the
 * expert-sorted copy of x, the SwiGLU intermediates and the per-slot partial
 * outputs; its size grows as N*k*(D + d_moe) + N*d_sh + E*(D + d_moe).
 */
size_t moe_forward_workspace(int N, int D, int E, int d_moe, int d_sh, int k, int dtype);

/*
 * moe_layer_forward_workspace — bytes of workspace for moe_layer_forward's
 * fastest path: moe_forward_workspace() plus, when wg_dtype is MOE_F32, room for
 * the router matrix split into three bf16 parts (3 * E * D * 2 bytes).  0 for
 * invalid sizes or dtypes.
 */
size_t moe_layer_forward_workspace(int N, int D, int E, int d_moe, int d_sh, int k, int dtype,
                                   int wg_dtype);

/*
 * moe_forward — routed experts, weighted combine and shared expert.
 * Defined by "GLM-4.5 MoE Forward", How it works: each routed expert is the
 * bias-free SwiGLU E_i(x) = W_down,i (SiLU(W_gate,i x) (.) W_up,i x) and
 * y_n = sum_{i in T(n)} w_{n,i} E_i(x_n) + E_sh(x_n), the shared expert (width
 * d_sh) on the same input at scale 1.  Weight layouts as in the GLM-5 "Mixture
 * of experts" code excerpt: gate_up_proj[i] is (2 d_moe, D) with the gate rows
 * first, down_proj[i] is (D, d_moe); an id equal to E is a sentinel that
 * contributes nothing.  topk_w already holds alpha; nothing is renormalised.
 *
 *   x        [N, D]            dtype
 *   gate_up  [E, 2*d_moe, D]   dtype
 *   down     [E, D, d_moe]     dtype
 *   sh_gate  [d_sh, D]         dtype
 *   sh_up    [d_sh, D]         dtype
 *   sh_down  [D, d_sh]         dtype
 *   topk_idx [N, k]            int32, each in [0, E]
 *   topk_w   [N, k]            fp32
 *   y        [N, D]            dtype out, fully overwritten
 *   workspace, ws_bytes        device scratch of at least moe_forward_workspace()
 * dtype MOE_BF16 runs the tensor-core path (bf16 operands, fp32 accumulation,
 * bf16 SwiGLU intermediate and per-slot partials, fp32 sum, one rounding of y);
 * MOE_F32 runs an fp32 CUDA-core path.  N = 0 is a no-op.
 * Ids outside [0, E] are skipped and reported by moe_device_status().
 */
int moe_forward(const void *x, const void *gate_up, const void *down, const void *sh_gate,
                const void *sh_up, const void *sh_down, const int32_t *topk_idx,
                const float *topk_w, int N, int D, int E, int d_moe, int d_sh, int k,
                int dtype, void *y, void *workspace, size_t ws_bytes, void *stream);

/*
 * moe_forward_clamped — moe_forward with the clamped SwiGLU of the
 * "GLM-5.3-Flash Module 02" page, section 3: every expert, routed or shared,
 * computes a = min(W_gate x, gate_max) (the gate is clamped from above only),
 * u = clip(W_up x, -up_max, up_max) and E(x) = W_down (SiLU(a) (.) u).  That
 * page's model uses gate_max = up_max = 10.  Same arguments, layouts,
 * workspace and errors as moe_forward; gate_max = up_max = +infinity gives
 * moe_forward exactly.  MOE_ERR_ARG for a NaN limit or up_max < 0.
 */
int moe_forward_clamped(const void *x, const void *gate_up, const void *down,
                        const void *sh_gate, const void *sh_up, const void *sh_down,
                        const int32_t *topk_idx, const float *topk_w, int N, int D, int E,
                        int d_moe, int d_sh, int k, int dtype, float gate_max, float up_max,
                        void *y, void *workspace, size_t ws_bytes, void *stream);

/*
 * moe_layer_forward — the whole layer in one call: moe_router then moe_forward
 * ("GLM-4.5 Group Router" and "GLM-4.5 MoE Forward", How it works), with x's
 * dtype `dtype` for the tokens and the experts and wg_dtype for W_g.  Writes
 * topk_idx / topk_w (as moe_router) and y (as moe_forward).  The workspace
 * needs at least moe_forward_workspace() bytes; with
 * moe_layer_forward_workspace() bytes (larger only for an fp32 W_g) a batch of
 * several 128-token blocks splits W_g into bf16 parts once per call instead of
 * once per token block (the same routing bit for bit, less router time).  For a bf16 layer of at most 128
 * tokens with at most 256 experts whose router runs on the tensor cores, the
 * forward's dispatch and token gather run inside the router kernel (one cluster
 * holds the whole routing), which saves two launches; the results are those of
 * the two separate calls.  All arguments are checked before anything is
 * launched; errors as moe_router and moe_forward.
 */
int moe_layer_forward(const void *x, const void *W_g, int wg_dtype, const float *b, int N, int D,
                      int E, int n_group, int topk_group, int k, int norm_topk_prob, float alpha,
                      const void *gate_up, const void *down, const void *sh_gate, const void *sh_up,
                      const void *sh_down, int d_moe, int d_sh, int dtype, int32_t *topk_idx,
                      float *topk_w, void *y, void *workspace, size_t ws_bytes, void *stream);

/*
 * moe_bias_update — one training step of the loss-free balancer on the router's
 * correction bias ("GLM-4.5 Group Router", How it works: b is updated from expert
 * load during training, at rate 0.001 for the first 15T tokens, then 0).  The page
 * gives the rate, not the rule; this implements the plainest reading of the
 * loss-free balancing it cites: with load_e the number of (token, slot) pairs of
 * topk_idx [N, k] routed to expert e (the sentinel id E counts for nobody; other
 * ids outside [0, E) are skipped and reported as MOE_ERR_BAD_INDEX by
 * moe_device_status), every b_e (fp32, device, [E], updated in place) moves by
 * `rate` towards the mean load: b_e += rate * sign(mean - load_e), decided exactly
 * in integers.  loads_out (optional, [E] int32) receives the loads.  E <= 512.
 * Errors: MOE_ERR_SHAPE, MOE_ERR_ARG (null b, NaN rate).
 */
int moe_bias_update(const int32_t *topk_idx, int N, int k, int E, float rate, float *b,
                    int32_t *loads_out, void *stream);

/* Bytes of device scratch built into the library for moe_forward_noalloc. */
#define MOE_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * moe_forward_noalloc — moe_forward for callers that cannot allocate device
 * memory.  The pages have no counterpart; this is a deployment aid.
 *
 * Some callers have no way to call cudaMalloc on the hot path.  A plugin inside
 * a serving runtime that owns every device allocation is one.  A
 * latency-critical loop that must not call cudaMalloc, because cudaMalloc can
 * synchronise the device, is another.  This entry point takes the same
 * arguments as moe_forward minus the workspace.  It uses a scratch array of
 * MOE_NOALLOC_SCRATCH_BYTES (64 MiB) that the library holds in device memory on
 * every GPU that loads it, until the process exits.  It calls no allocator.
 *   - Sizes whose moe_forward_workspace() exceeds MOE_NOALLOC_SCRATCH_BYTES are
 *     refused with MOE_ERR_WORKSPACE before any launch (small layers, e.g.
 *     N*k + 127*E up to a few thousand rows at D of a few hundred, fit).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current.  Make it before any
 *     stream capture.  The address is cached per device and never looked up
 *     again: after a cudaDeviceReset in the same process it is stale, so do
 *     not use this entry point on a device reset after its first call.
 *   - Arguments (sizes, dtype, pointers, an sm_100 device) are checked before
 *     that look-up; errors as moe_forward.
 *   - All calls on a device share the array, which keeps the last call's
 *     contents.  Each call rewrites everything it reads before reading it.
 *     Calls whose kernels overlap on the GPU race; serialise them (one stream).
 * Results equal moe_forward's for the same inputs.
 */
int moe_forward_noalloc(const void *x, const void *gate_up, const void *down,
                        const void *sh_gate, const void *sh_up, const void *sh_down,
                        const int32_t *topk_idx, const float *topk_w, int N, int D, int E,
                        int d_moe, int d_sh, int k, int dtype, void *y, void *stream);

/*
 * moe_device_status — synchronises `stream`, then returns and clears the device
 * status word: MOE_OK, MOE_ERR_DEVICE_TIMEOUT (a bounded wait ran out; the
 * output of that call is not valid) or MOE_ERR_BAD_INDEX.  Returns
 * MOE_ERR_CUDA if the synchronisation itself failed.
 */
int moe_device_status(void *stream);

/* Static, human-readable text for a status code. */
const char *moe_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int moe_version(void);

/*
 * Test hooks for the bounded device-side waits (no GPU fault is involved).
 *   moe_debug_set_wait_limit_ns: limit for every spin-wait in the kernels
 *     (default 2e9 ns); ns = 0 restores the default.
 *   moe_debug_never_signal: when on, the combine of the next moe_forward calls
 *     (the decode down kernel's shared tiles, or the prefill combine kernel)
 *     waits for one more expert tile than exists, so the wait runs out, the
 *     status word reports MOE_ERR_DEVICE_TIMEOUT and the kernel returns normally.
 */
int moe_debug_set_wait_limit_ns(uint64_t ns);
int moe_debug_never_signal(int on);

/*
 * Tuning and test hook for the prefill expert GEMMs (more than 256 bf16
 * tokens).  Mode 1 runs them on CTA pairs (two SMs share one M = 256
 * tensor-core tile) with the odd last m-tile of each expert on the one-SM
 * kernels; mode 2 runs every m-tile on CTA pairs, an odd last m-tile pairing
 * with an empty half; mode 3 runs the experts with an even number of m-tiles
 * on CTA pairs and the others on the one-SM kernels; mode 4 does that for the
 * down GEMM only; mode 0 runs every tile on the one-SM kernels; -1 restores
 * the library's default (mode 4).  Results are identical bit for bit in every
 * mode.  MOE_ERR_ARG for other values.
 */
int moe_debug_set_pair_mode(int mode);

/*
 * Test hook for the router's precision ("GLM-4.5 Group Router", How it works:
 * the gate runs in float32).  While buf is non-null, every router launch
 * (moe_router, moe_layer_forward) also writes each token's selection scores
 * s' = sigmoid(r) + b as fp32 into buf [N, E] (device memory, 16-byte aligned,
 * caller-owned, n_floats >= N * E, else the router call returns MOE_ERR_ARG
 * before any launch).  The scores are those the selection compares, before
 * any group masking.  buf = NULL turns the capture off (the default).
 */
int moe_debug_capture_scores(float *buf, size_t n_floats);

/*
 * Profiling hooks (used by the benchmark; no effect on results).
 *   moe_profile_set_events: while n > 0, every moe_forward call records
 *     events[0] on its stream before its first kernel and events[i] right after
 *     its i-th kernel launch (i = 1 .. n-1).  The events are caller-owned
 *     cudaEvent_t handles passed as void*; n = 0 turns recording off.  At most
 *     16 events; MOE_ERR_ARG otherwise.  Under stream capture the records are
 *     external (cudaEventRecordExternal), so they become event nodes of the
 *     graph and record on every replay.
 *   moe_launch_count: kernels launched by this library in this process so far.
 */
int moe_profile_set_events(void *const *events, int n);
unsigned long long moe_launch_count(void);

/* ------------------------------------------------------------------------- *
 * Expert parallelism over peer memory.
 *
 * "GLM-5.3-Flash Module 02" (expert placement and popularity) treats the
 * placement of experts across devices as a serving variable: each token's
 * hidden state is sent to the devices that hold its top-k experts and the
 * expert outputs come back.  Here P ranks (one process per GPU, P <= 8) each
 * hold E/P experts, rank q the experts [q*E/P, (q+1)*E/P), and their own batch
 * of tokens.  The exchange is done by the kernels themselves: stores and
 * atomics into the other ranks' memory over NVLink / NVSwitch, with bounded
 * waits on counters, no collective-library call.
 *
 * Every rank owns a symmetric buffer of moe_ep_symmetric_bytes() bytes (the
 * same P, N_cap, D, E, k on every rank), zero-filled once before the first
 * call, and maps every other rank's buffer into its own address space
 * (moe_ep_ipc_export / moe_ep_ipc_open).  peer_sym[q] is rank q's buffer as
 * seen from the calling rank (peer_sym[rank] = its own); 256-byte aligned.
 *
 * moe_ep_forward computes, for the calling rank's N <= N_cap tokens, the same
 * y as moe_forward would with all E experts on one device (bf16 only; the
 * per-row arithmetic is that of moe_forward's 128-row-tile kernels, so y equals
 * moe_forward's bit for bit whenever moe_forward takes those kernels, N > 256).
 *   gate_up_loc [E/P, 2*d_moe, D] and down_loc [E/P, D, d_moe]: this rank's
 *   experts; sh_*: the shared expert (replicated); topk_idx/topk_w [N, k] with
 *   global expert ids (id E is the sentinel, skipped).
 *   epoch: 1, 2, 3, ... the number of this call, equal on all ranks.
 *   phases: a mask of MOE_EP_COUNT (publish this rank's expert histogram to all
 *   ranks), MOE_EP_SEND (wait for all histograms, store token rows into the
 *   owners' buffers), MOE_EP_EXPERTS (wait for this rank's rows, run its
 *   experts and the shared expert, store weighted rows back into the sources'
 *   buffers) and MOE_EP_COMBINE (wait for this rank's rows to come back, write
 *   y).  A multi-GPU job passes MOE_EP_ALL on every rank.  Running the phases
 *   one at a time over all ranks lets P ranks run on one device, since every
 *   wait is then already satisfied.
 *   workspace: moe_ep_workspace_bytes() bytes, 256-byte aligned, private to the
 *   rank and kept between the phases of one epoch.
 * Errors: MOE_ERR_ARG (phases, P, rank, epoch, pointers), MOE_ERR_SHAPE
 * (E % P, E > 512, k, N > N_cap, D / d_moe / d_sh not multiples of 8),
 * MOE_ERR_WORKSPACE; a wait that runs out (a rank that never arrives) is
 * reported by moe_device_status as MOE_ERR_DEVICE_TIMEOUT.
 */
#define MOE_EP_COUNT 1
#define MOE_EP_SEND 2
#define MOE_EP_EXPERTS 4
#define MOE_EP_COMBINE 8
#define MOE_EP_ALL 15
#define MOE_EP_MAX_RANKS 8
#define MOE_EP_IPC_HANDLE_BYTES 72 /* CUDA IPC handle (64) + offset in its allocation (8) */

size_t moe_ep_symmetric_bytes(int P, int N_cap, int D, int E, int k);
size_t moe_ep_workspace_bytes(int P, int N_cap, int D, int E, int d_moe, int d_sh, int k);
int moe_ep_forward(int phases, int P, int rank, unsigned epoch, void *const *peer_sym, int N_cap,
                   const void *x, const void *gate_up_loc, const void *down_loc,
                   const void *sh_gate, const void *sh_up, const void *sh_down,
                   const int32_t *topk_idx, const float *topk_w, int N, int D, int E, int d_moe,
                   int d_sh, int k, void *y, void *workspace, size_t ws_bytes, void *stream);

/*
 * moe_ep_plan_host — the layout the send phase derives, computed on the host
 * (no device needed): from the P x E histogram counts[r][e] (pairs of rank r
 * routed to expert e), for sender `rank`: dest_base[e] = the row, in expert
 * e's owner's receive buffer, of this rank's first pair routed to e, minus
 * that pair's position in this rank's expert-sorted order; for `rank` as a
 * receiver: rcounts[E/P] rows per local expert, rtile_off[E/P + 1] the prefix
 * of 128-row tiles, *rows_in rows received, *pairs_out pairs sent.
 */
int moe_ep_plan_host(int P, int rank, int E, const int32_t *counts, int32_t *dest_base,
                     int32_t *rcounts, int32_t *rtile_off, int32_t *rows_in, int32_t *pairs_out);

/*
 * Mapping another rank's symmetric buffer (CUDA IPC).  moe_ep_ipc_export writes
 * MOE_EP_IPC_HANDLE_BYTES bytes naming dev_ptr (any address inside a device
 * allocation of this process); another process's moe_ep_ipc_open maps it and
 * returns the same address in its own space; moe_ep_ipc_close unmaps a pointer
 * returned by moe_ep_ipc_open.  MOE_ERR_CUDA if the driver refuses (e.g. the
 * same process, or no peer access).
 */
int moe_ep_ipc_export(const void *dev_ptr, void *handle);
int moe_ep_ipc_open(const void *handle, void **dev_ptr);
int moe_ep_ipc_close(void *dev_ptr);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
