"""B200 (sm_100a) sparse MoE FFN forward, GLM-4.5 / GLM-5 style.

Thin ctypes binding over libmoe.so (C ABI in include/moe.h).  The functions
here only marshal torch CUDA tensors into pointers, sizes and the current
stream; every step of the layer runs in the library's CUDA kernels.  There is
no fallback: if libmoe.so is missing or no sm_100 GPU is current, calls raise.

    idx, w = moe_router(x, W_g, b, n_group, topk_group, k, norm_topk_prob, alpha)
    y = moe_forward(x, gate_up, down, sh_gate, sh_up, sh_down, idx, w)
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = ["MoEError", "moe_router", "moe_forward", "moe_forward_workspace", "moe_layer",
           "moe_layer_forward_workspace",
           "moe_device_status", "moe_status_string", "moe_debug_set_wait_limit_ns",
           "moe_debug_never_signal", "moe_debug_capture_scores", "moe_debug_set_pair_mode",
           "moe_profile_set_events",
           "moe_launch_count", "moe_forward_noalloc", "library_path", "load_library", "MOE_F32", "MOE_BF16",
           "EXPORTED_SYMBOLS", "moe_ep_symmetric_bytes", "moe_ep_workspace_bytes",
           "moe_ep_forward", "moe_ep_plan_host", "moe_ep_ipc_export", "moe_ep_ipc_open",
           "moe_ep_ipc_close", "ExpertParallelGroup", "MOE_EP_COUNT", "MOE_EP_SEND",
           "MOE_EP_EXPERTS", "MOE_EP_COMBINE", "MOE_EP_ALL", "moe_bias_update"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmoe.so")
_lock = threading.Lock()
_lib = None

MOE_F32, MOE_BF16 = 0, 1
MOE_OK = 0
MOE_EP_COUNT, MOE_EP_SEND, MOE_EP_EXPERTS, MOE_EP_COMBINE = 1, 2, 4, 8
MOE_EP_ALL = 15
MOE_EP_PHASES = (MOE_EP_COUNT, MOE_EP_SEND, MOE_EP_EXPERTS, MOE_EP_COMBINE)
MOE_EP_IPC_HANDLE_BYTES = 72

EXPORTED_SYMBOLS = ("moe_router", "moe_forward_workspace", "moe_layer_forward_workspace",
                    "moe_forward", "moe_device_status",
                    "moe_status_string", "moe_version", "moe_debug_set_wait_limit_ns",
                    "moe_debug_never_signal", "moe_profile_set_events", "moe_launch_count",
                    "moe_debug_capture_scores", "moe_debug_set_pair_mode", "moe_forward_noalloc", "moe_forward_clamped", "moe_layer_forward",
                    "moe_bias_update",
                    "moe_ep_symmetric_bytes",
                    "moe_ep_workspace_bytes", "moe_ep_forward", "moe_ep_plan_host",
                    "moe_ep_ipc_export", "moe_ep_ipc_open", "moe_ep_ipc_close")


class MoEError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__("%s failed: %s (status %d)" % (what, moe_status_string(code), code))


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libmoe.so (built in-tree by sparse_moe_layer_02_b200.build); raise if absent."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError("libmoe.so not found at %s; build it with "
                               "`python -m sparse_moe_layer_02_b200.build`" % _LIB_PATH)
        lib = ctypes.CDLL(_LIB_PATH)
        P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        lib.moe_router.argtypes = [P, I, P, I, P, I, I, I, I, I, I, I, F, P, P, P]
        lib.moe_router.restype = I
        lib.moe_forward_workspace.argtypes = [I, I, I, I, I, I, I]
        lib.moe_forward_workspace.restype = ctypes.c_size_t
        lib.moe_layer_forward_workspace.argtypes = [I, I, I, I, I, I, I, I]
        lib.moe_layer_forward_workspace.restype = ctypes.c_size_t
        lib.moe_forward.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P,
                                    ctypes.c_size_t, P]
        lib.moe_forward.restype = I
        lib.moe_device_status.argtypes = [P]
        lib.moe_device_status.restype = I
        lib.moe_status_string.argtypes = [I]
        lib.moe_status_string.restype = ctypes.c_char_p
        lib.moe_version.argtypes = []
        lib.moe_version.restype = I
        lib.moe_debug_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        lib.moe_debug_set_wait_limit_ns.restype = I
        lib.moe_debug_never_signal.argtypes = [I]
        lib.moe_debug_never_signal.restype = I
        lib.moe_debug_set_pair_mode.argtypes = [I]
        lib.moe_debug_set_pair_mode.restype = I
        lib.moe_debug_capture_scores.argtypes = [P, ctypes.c_size_t]
        lib.moe_debug_capture_scores.restype = I
        lib.moe_profile_set_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), I]
        lib.moe_profile_set_events.restype = I
        lib.moe_launch_count.argtypes = []
        lib.moe_launch_count.restype = ctypes.c_ulonglong
        lib.moe_forward_noalloc.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P]
        lib.moe_forward_noalloc.restype = I
        lib.moe_forward_clamped.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, F, P,
                                            P, ctypes.c_size_t, P]
        lib.moe_forward_clamped.restype = I
        S = ctypes.c_size_t
        lib.moe_layer_forward.argtypes = [P, P, I, P, I, I, I, I, I, I, I, F, P, P, P, P, P, I, I, I,
                                          P, P, P, P, S, P]
        lib.moe_layer_forward.restype = I
        lib.moe_bias_update.argtypes = [P, I, I, I, F, P, P, P]
        lib.moe_bias_update.restype = I
        lib.moe_ep_symmetric_bytes.argtypes = [I, I, I, I, I]
        lib.moe_ep_symmetric_bytes.restype = S
        lib.moe_ep_workspace_bytes.argtypes = [I, I, I, I, I, I, I]
        lib.moe_ep_workspace_bytes.restype = S
        lib.moe_ep_forward.argtypes = [I, I, I, ctypes.c_uint, ctypes.POINTER(ctypes.c_void_p), I,
                                       P, P, P, P, P, P, P, P, I, I, I, I, I, I, P, P, S, P]
        lib.moe_ep_forward.restype = I
        lib.moe_ep_plan_host.argtypes = [I, I, I, P, P, P, P, P, P]
        lib.moe_ep_plan_host.restype = I
        lib.moe_ep_ipc_export.argtypes = [P, P]
        lib.moe_ep_ipc_export.restype = I
        lib.moe_ep_ipc_open.argtypes = [P, ctypes.POINTER(ctypes.c_void_p)]
        lib.moe_ep_ipc_open.restype = I
        lib.moe_ep_ipc_close.argtypes = [P]
        lib.moe_ep_ipc_close.restype = I
        _lib = lib
        return lib


def moe_status_string(code: int) -> str:
    return load_library().moe_status_string(int(code)).decode()


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MOE_F32
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    raise TypeError("unsupported dtype %s (float32 or bfloat16)" % t.dtype)


def _dev(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(rc: int, what: str):
    if rc != MOE_OK:
        raise MoEError(rc, what)


def moe_router(x, W_g, b, n_group: int, topk_group: int, k: int, norm_topk_prob: bool,
               alpha: float, topk_idx=None, topk_w=None, stream=None):
    """Router: returns (topk_idx [N,k] int32, topk_w [N,k] fp32) on x's device."""
    lib = load_library()
    N, D = x.shape
    E = W_g.shape[0]
    if tuple(W_g.shape) != (E, D) or tuple(b.shape) != (E,) or b.dtype != torch.float32:
        raise ValueError("W_g must be [E, D] and b [E] float32")
    if topk_idx is None:
        topk_idx = torch.empty((N, k), dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty((N, k), dtype=torch.float32, device=x.device)
    if topk_idx.dtype != torch.int32 or topk_w.dtype != torch.float32:
        raise ValueError("topk_idx must be int32 and topk_w float32")
    if tuple(topk_idx.shape) != (N, k) or tuple(topk_w.shape) != (N, k):
        raise ValueError("topk_idx / topk_w must be [N, k]")
    rc = lib.moe_router(_dev(x, "x"), _dt(x), _dev(W_g, "W_g"), _dt(W_g), _dev(b, "b"), N, D, E,
                        int(n_group), int(topk_group), int(k), int(bool(norm_topk_prob)),
                        float(alpha), _dev(topk_idx, "topk_idx"), _dev(topk_w, "topk_w"),
                        _stream(stream))
    _check(rc, "moe_router")
    return topk_idx, topk_w


def moe_forward_workspace(N: int, D: int, E: int, d_moe: int, d_sh: int, k: int,
                          dtype: torch.dtype) -> int:
    return int(load_library().moe_forward_workspace(N, D, E, d_moe, d_sh, k,
                                                     MOE_BF16 if dtype == torch.bfloat16 else MOE_F32))


def moe_layer_forward_workspace(N: int, D: int, E: int, d_moe: int, d_sh: int, k: int,
                                dtype: torch.dtype, wg_dtype: torch.dtype) -> int:
    """Workspace bytes for moe_layer: moe_forward's plus, for an fp32 router matrix,
    room to split it into bf16 parts once per call."""
    f = lambda t: MOE_BF16 if t == torch.bfloat16 else MOE_F32
    return int(load_library().moe_layer_forward_workspace(N, D, E, d_moe, d_sh, k, f(dtype),
                                                           f(wg_dtype)))


def moe_forward(x, gate_up, down, sh_gate, sh_up, sh_down, topk_idx, topk_w, y=None,
                workspace=None, stream=None, gate_max=None, up_max=None):
    """Routed experts + weighted combine + shared expert; returns y [N, D].

    gate_max / up_max (optional): the clamped SwiGLU (gate clamped from above at
    gate_max, up clipped to [-up_max, up_max]) via moe_forward_clamped."""
    lib = load_library()
    N, D = x.shape
    E, two_d, D2 = gate_up.shape
    d = two_d // 2
    d_sh = sh_gate.shape[0]
    k = topk_idx.shape[1] if topk_idx.dim() == 2 else 0
    if D2 != D or tuple(down.shape) != (E, D, d) or tuple(sh_up.shape) != (d_sh, D) \
            or tuple(sh_down.shape) != (D, d_sh) or tuple(topk_w.shape) != (N, k):
        raise ValueError("inconsistent expert or routing shapes")
    for t in (gate_up, down, sh_gate, sh_up, sh_down):
        if t.dtype != x.dtype:
            raise ValueError("expert weights must share x's dtype")
    if topk_idx.dtype != torch.int32 or topk_w.dtype != torch.float32:
        raise ValueError("topk_idx must be int32 and topk_w float32")
    if y is None:
        y = torch.empty((N, D), dtype=x.dtype, device=x.device)
    ws_bytes = int(lib.moe_forward_workspace(N, D, E, d, d_sh, k, _dt(x)))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=x.device)
    ptrs = (_dev(x, "x"), _dev(gate_up, "gate_up"), _dev(down, "down"), _dev(sh_gate, "sh_gate"),
            _dev(sh_up, "sh_up"), _dev(sh_down, "sh_down"), _dev(topk_idx, "topk_idx"),
            _dev(topk_w, "topk_w"), N, D, E, d, d_sh, k, _dt(x))
    tail = (_dev(y, "y"), _dev(workspace, "workspace"),
            workspace.numel() * workspace.element_size(), _stream(stream))
    if gate_max is None and up_max is None:
        _check(lib.moe_forward(*ptrs, *tail), "moe_forward")
    else:
        inf = float("inf")
        gm = inf if gate_max is None else float(gate_max)
        um = inf if up_max is None else float(up_max)
        _check(lib.moe_forward_clamped(*ptrs, gm, um, *tail), "moe_forward_clamped")
    return y


def moe_forward_noalloc(x, gate_up, down, sh_gate, sh_up, sh_down, topk_idx, topk_w, y,
                        stream=None):
    """moe_forward without a workspace, for callers that cannot allocate device memory:
    the library's built-in 64 MiB device scratch is used instead (small layers only;
    larger ones raise with the workspace error).  y must be preallocated."""
    lib = load_library()
    N, D = x.shape
    E, two_d, _ = gate_up.shape
    k = topk_idx.shape[1]
    rc = lib.moe_forward_noalloc(_dev(x, "x"), _dev(gate_up, "gate_up"), _dev(down, "down"),
                                 _dev(sh_gate, "sh_gate"), _dev(sh_up, "sh_up"),
                                 _dev(sh_down, "sh_down"), _dev(topk_idx, "topk_idx"),
                                 _dev(topk_w, "topk_w"), N, D, E, two_d // 2, sh_gate.shape[0], k,
                                 _dt(x), _dev(y, "y"), _stream(stream))
    _check(rc, "moe_forward_noalloc")
    return y


def moe_layer(x, W_g, b, gate_up, down, sh_gate, sh_up, sh_down, n_group, topk_group, k,
              norm_topk_prob, alpha, workspace=None, y=None, topk_idx=None, topk_w=None,
              stream=None):
    """Whole layer in one library call (router then forward; small bf16 batches run the
    dispatch inside the router kernel).  Returns (y, topk_idx, topk_w)."""
    lib = load_library()
    N, D = x.shape
    E, two_d, D2 = gate_up.shape
    d, d_sh = two_d // 2, sh_gate.shape[0]
    if D2 != D or tuple(W_g.shape) != (E, D) or tuple(b.shape) != (E,) or b.dtype != torch.float32:
        raise ValueError("inconsistent shapes")
    dev = x.device
    if topk_idx is None:
        topk_idx = torch.empty((N, k), dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty((N, k), dtype=torch.float32, device=dev)
    if y is None:
        y = torch.empty((N, D), dtype=x.dtype, device=dev)
    if workspace is None:
        workspace = torch.empty(max(moe_layer_forward_workspace(N, D, E, d, d_sh, k, x.dtype,
                                                                W_g.dtype), 256),
                                dtype=torch.uint8, device=dev)
    if N == 0:
        return y, topk_idx, topk_w
    rc = lib.moe_layer_forward(_dev(x, "x"), _dev(W_g, "W_g"), _dt(W_g), _dev(b, "b"), N, D, E,
                               n_group, topk_group, k, int(bool(norm_topk_prob)), float(alpha),
                               _dev(gate_up, "gate_up"), _dev(down, "down"),
                               _dev(sh_gate, "sh_gate"), _dev(sh_up, "sh_up"),
                               _dev(sh_down, "sh_down"), d, d_sh, _dt(x), _dev(topk_idx, "topk_idx"),
                               _dev(topk_w, "topk_w"), _dev(y, "y"), _dev(workspace, "workspace"),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "moe_layer_forward")
    return y, topk_idx, topk_w


def moe_bias_update(topk_idx, b, rate: float = 1e-3, loads=None, stream=None):
    """One loss-free balancing step on the router bias b (fp32 [E], updated in place):
    b_e += rate * sign(mean load - load_e) over the routing topk_idx [N, k].  Returns
    (b, loads) with loads [E] int32 (allocated if not given)."""
    if b.dtype != torch.float32 or b.dim() != 1:
        raise ValueError("b must be a 1-D float32 tensor")
    E = b.shape[0]
    N, k = topk_idx.shape
    if loads is None:
        loads = torch.empty(E, dtype=torch.int32, device=b.device)
    rc = load_library().moe_bias_update(_dev(topk_idx, "topk_idx") if N else 0, N, k, E,
                                        float(rate), _dev(b, "b"), _dev(loads, "loads"),
                                        _stream(stream))
    _check(rc, "moe_bias_update")
    return b, loads


def moe_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return int(load_library().moe_device_status(_stream(stream)))


def moe_debug_set_wait_limit_ns(ns: int):
    _check(load_library().moe_debug_set_wait_limit_ns(int(ns)), "moe_debug_set_wait_limit_ns")


def moe_debug_never_signal(on: bool):
    _check(load_library().moe_debug_never_signal(int(bool(on))), "moe_debug_never_signal")


def moe_debug_set_pair_mode(mode: int) -> None:
    """Prefill expert GEMMs on CTA pairs: 1 full pairs plus one-SM tails, 2 padded pairs
    only, 3 even-count experts on pairs and the rest on one SM, 4 that split for the down
    GEMM only, 0 never; -1 restores the library's default."""
    _check(load_library().moe_debug_set_pair_mode(int(mode)), "moe_debug_set_pair_mode")


def moe_debug_capture_scores(buf) -> None:
    """Test hook: while `buf` (a contiguous fp32 CUDA tensor of at least N*E
    elements) is set, router launches also write their selection scores
    s' = sigmoid(r) + b into it as [N, E]; None turns the capture off."""
    if buf is None:
        _check(load_library().moe_debug_capture_scores(None, 0), "moe_debug_capture_scores")
        return
    if buf.dtype != torch.float32:
        raise ValueError("the score buffer must be float32")
    _check(load_library().moe_debug_capture_scores(_dev(buf, "buf"), buf.numel()),
           "moe_debug_capture_scores")


def moe_profile_set_events(events) -> None:
    """Record the given torch.cuda.Event objects at the next calls' kernel boundaries
    (events[0] before the first kernel, events[i] after the i-th; None skips a
    boundary); [] turns it off."""
    handles = [int(e.cuda_event) if e is not None else 0 for e in events]
    arr = (ctypes.c_void_p * max(len(handles), 1))(*handles)
    _check(load_library().moe_profile_set_events(arr, len(handles)), "moe_profile_set_events")


def moe_launch_count() -> int:
    return int(load_library().moe_launch_count())


# ----------------------------------------------------------------------------- experts
# spread over ranks (peer memory; see include/moe.h, "Expert parallelism")

def moe_ep_symmetric_bytes(P: int, N_cap: int, D: int, E: int, k: int) -> int:
    return int(load_library().moe_ep_symmetric_bytes(P, N_cap, D, E, k))


def moe_ep_workspace_bytes(P: int, N_cap: int, D: int, E: int, d_moe: int, d_sh: int,
                           k: int) -> int:
    return int(load_library().moe_ep_workspace_bytes(P, N_cap, D, E, d_moe, d_sh, k))


def moe_ep_forward(phases: int, P: int, rank: int, epoch: int, peer_sym, N_cap: int, x, gate_up_loc,
                   down_loc, sh_gate, sh_up, sh_down, topk_idx, topk_w, E: int, y, workspace,
                   stream=None):
    """One rank's part of an expert-parallel forward.  peer_sym: the P symmetric buffers'
    device addresses as seen from this rank; gate_up_loc / down_loc: this rank's E/P
    experts; topk_idx holds global expert ids.  y [N, D] must be preallocated."""
    lib = load_library()
    N, D = x.shape
    E_loc, two_d, _ = gate_up_loc.shape
    k = topk_idx.shape[1]
    arr = (ctypes.c_void_p * P)(*[int(a) for a in peer_sym])
    dp = lambda t, name: _dev(t, name) if t.numel() else 0
    rc = lib.moe_ep_forward(phases, P, rank, epoch, arr, N_cap, dp(x, "x"),
                            _dev(gate_up_loc, "gate_up_loc"), _dev(down_loc, "down_loc"),
                            _dev(sh_gate, "sh_gate"), _dev(sh_up, "sh_up"), _dev(sh_down, "sh_down"),
                            dp(topk_idx, "topk_idx"), dp(topk_w, "topk_w"), N, D, E, two_d // 2,
                            sh_gate.shape[0], k, dp(y, "y"), _dev(workspace, "workspace"),
                            workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "moe_ep_forward")
    return y


def moe_ep_plan_host(P: int, rank: int, counts):
    """Host mirror of the send-phase layout from the P x E histogram (numpy int32)."""
    import numpy as np
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    Pc, E = counts.shape
    if Pc != P:
        raise ValueError("counts must be [P, E]")
    E_loc = E // P if P else 0
    dest = np.zeros(E, np.int32)
    rc_ = np.zeros(max(E_loc, 1), np.int32)
    rto = np.zeros(E_loc + 1, np.int32)
    rows_in = ctypes.c_int32(0)
    pairs_out = ctypes.c_int32(0)
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    rc = load_library().moe_ep_plan_host(P, rank, E, ptr(counts), ptr(dest), ptr(rc_), ptr(rto),
                                         ctypes.byref(rows_in), ctypes.byref(pairs_out))
    _check(rc, "moe_ep_plan_host")
    return {"dest_base": dest, "rcounts": rc_[:E_loc], "rtile_off": rto,
            "rows_in": int(rows_in.value), "pairs_out": int(pairs_out.value)}


def moe_ep_ipc_export(t: torch.Tensor) -> bytes:
    buf = ctypes.create_string_buffer(MOE_EP_IPC_HANDLE_BYTES)
    _check(load_library().moe_ep_ipc_export(_dev(t, "buffer"), buf), "moe_ep_ipc_export")
    return buf.raw


def moe_ep_ipc_open(handle: bytes) -> int:
    out = ctypes.c_void_p()
    buf = ctypes.create_string_buffer(bytes(handle), MOE_EP_IPC_HANDLE_BYTES)
    _check(load_library().moe_ep_ipc_open(buf, ctypes.byref(out)), "moe_ep_ipc_open")
    return int(out.value)


def moe_ep_ipc_close(ptr: int) -> None:
    _check(load_library().moe_ep_ipc_close(ctypes.c_void_p(ptr)), "moe_ep_ipc_close")


class ExpertParallelGroup:
    """Expert-parallel layer state of one rank in a torch.distributed job (one process per
    GPU): allocates this rank's symmetric buffer and workspace, exchanges CUDA IPC handles
    with the other ranks (all_gather_object over the default group) and maps their
    buffers.  forward() runs all four phases for the next epoch."""

    def __init__(self, N_cap: int, D: int, E: int, k: int, d_moe: int, d_sh: int, device=None,
                 group=None):
        import torch.distributed as dist
        self.P = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.N_cap, self.E = N_cap, E
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        sym_bytes = moe_ep_symmetric_bytes(self.P, N_cap, D, E, k)
        ws_bytes = moe_ep_workspace_bytes(self.P, N_cap, D, E, d_moe, d_sh, k)
        if not sym_bytes or not ws_bytes:
            raise ValueError("unsupported expert-parallel shape")
        self.sym = torch.zeros(sym_bytes, dtype=torch.uint8, device=dev)
        self.workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        torch.cuda.synchronize(dev)
        handles = [None] * self.P
        dist.all_gather_object(handles, moe_ep_ipc_export(self.sym), group=group)
        self._opened = []
        self.peer_sym = []
        for q, h in enumerate(handles):
            if q == self.rank:
                self.peer_sym.append(self.sym.data_ptr())
            else:
                ptr = moe_ep_ipc_open(h)
                self._opened.append(ptr)
                self.peer_sym.append(ptr)
        dist.barrier(group=group)
        self.epoch = 0

    def forward(self, x, gate_up_loc, down_loc, sh_gate, sh_up, sh_down, topk_idx, topk_w,
                y=None, stream=None):
        if y is None:
            y = torch.empty_like(x)
        self.epoch += 1
        return moe_ep_forward(MOE_EP_ALL, self.P, self.rank, self.epoch, self.peer_sym, self.N_cap,
                              x, gate_up_loc, down_loc, sh_gate, sh_up, sh_down, topk_idx, topk_w,
                              self.E, y, self.workspace, stream)

    def close(self):
        for ptr in self._opened:
            moe_ep_ipc_close(ptr)
        self._opened = []
