"""Plain fp64 CPU oracle for the GLM-4.5 / GLM-5 sparse MoE FFN forward.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the bench's
CPU-baseline / reference legs are the only callers.  Nothing here imports or
calls the CUDA package, and the CUDA package never imports this one.

The arithmetic lives in ``oracle.c`` (plain loops, fp64).  This module compiles
it with gcc if needed, loads it with ctypes and marshals torch CPU tensors.
``forward_expert_major`` is a second, independent formulation of the same sum
(a loop over hit experts with a scatter-add, as the GLM-5 "Mixture of experts"
page's code excerpt describes the experts' forward), used only to cross-check
the token-major C loops.

Pins (tests/test_oracle_*.py) tie every function here to the pages:
G = 1 equals a full sort; brute-force enumeration on tiny group-routed inputs;
sum(w) = alpha; w ratios equal s ratios (bias never in the weights);
closed-form sigmoid and SwiGLU values; shared expert unscaled; sentinel skipped;
the pages' parameter counts.

``bias_update`` (the loss-free balancer's training step): parity unpinned.  The
pages give its rate, not its rule; the function follows a stated reading, and
its pins check that reading's properties, not values the pages print.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP, strict IEEE fp64)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def configure(lib):
    """Declare the C signatures on a loaded oracle library (also used by the tests
    that load deliberately broken copies of oracle.c)."""
    P = ctypes.c_void_p
    I = ctypes.c_int
    Dd = ctypes.c_double
    lib.oracle_num_threads.restype = I
    lib.oracle_router_logits.argtypes = [P, I, P, I, I, I, I, P]
    lib.oracle_router_logits.restype = None
    lib.oracle_select.argtypes = [P, P, I, I, I, I, I, I, Dd, P, P, P, P, P, P]
    lib.oracle_select.restype = I
    lib.oracle_forward.argtypes = [P, P, P, P, P, P, I, P, P, I, I, I, I, I, I, P, I, Dd, Dd, P]
    lib.oracle_forward.restype = I
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = configure(ctypes.CDLL(_LIB))
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError("oracle inputs must be float32 or bfloat16, got %s" % t.dtype)


def _host(t: torch.Tensor) -> torch.Tensor:
    return t.detach().to("cpu").contiguous()


def _ptr(a) -> int:
    if isinstance(a, torch.Tensor):
        return a.data_ptr()
    return a.ctypes.data


def router_logits(x: torch.Tensor, W_g: torch.Tensor) -> np.ndarray:
    """r = x W_g^T in fp64 (GLM-4.5 Group Router, "How it works", gate equation)."""
    x, W_g = _host(x), _host(W_g)
    N, D = x.shape
    E = W_g.shape[0]
    assert W_g.shape[1] == D
    r = np.empty((N, E), dtype=np.float64)
    _load().oracle_router_logits(_ptr(x), _dt(x), _ptr(W_g), _dt(W_g), N, D, E, _ptr(r))
    return r


def select(r: np.ndarray, b: torch.Tensor, n_group: int, topk_group: int, k: int,
           norm_topk_prob: bool, alpha: float) -> dict:
    """Sigmoid, bias, group top-2 score, group keep, top-k, weights from logits r [N,E].

    GLM-4.5 Group Router, "How it works" (s, s', g_g, T, s-bar, w equations).
    Returns idx [N,k] int32, w [N,k] fp64, s [N,E] fp64, margin_exp [N],
    margin_grp [N], zero_fill_differs [N].
    """
    r = np.ascontiguousarray(r, dtype=np.float64)
    b = _host(b).to(torch.float32)
    N, E = r.shape
    idx = np.empty((N, k), dtype=np.int32)
    w = np.empty((N, k), dtype=np.float64)
    s = np.empty((N, E), dtype=np.float64)
    me = np.empty(N, dtype=np.float64)
    mg = np.empty(N, dtype=np.float64)
    zf = np.empty(N, dtype=np.int32)
    rc = _load().oracle_select(_ptr(r), _ptr(b), N, E, n_group, topk_group, k,
                               int(bool(norm_topk_prob)), float(alpha), _ptr(idx), _ptr(w),
                               _ptr(s), _ptr(me), _ptr(mg), _ptr(zf))
    if rc != 0:
        raise ValueError("invalid router configuration (E=%d, G=%d, topk_group=%d, k=%d)"
                         % (E, n_group, topk_group, k))
    return {"idx": idx, "w": w, "s": s, "margin_exp": me, "margin_grp": mg,
            "zero_fill_differs": zf, "r": r}


def router(x: torch.Tensor, W_g: torch.Tensor, b: torch.Tensor, n_group: int, topk_group: int,
           k: int, norm_topk_prob: bool, alpha: float) -> dict:
    """Logits then selection (the whole router), fp64."""
    return select(router_logits(x, W_g), b, n_group, topk_group, k, norm_topk_prob, alpha)


def forward(x, gate_up, down, sh_gate, sh_up, sh_down, idx, w, tokens=None,
            gate_max: float = float("inf"), up_max: float = float("inf")) -> np.ndarray:
    """y rows for `tokens` (default all), token-major fp64 (GLM-4.5 MoE Forward, y_n).

    x [N,D]; gate_up [E,2d,D]; down [E,D,d]; sh_gate, sh_up [d_sh,D]; sh_down [D,d_sh];
    idx [N,k] (value E = sentinel, skipped); w [N,k] (alpha already included).
    gate_max / up_max: clamped SwiGLU (GLM-5.3-Flash Module 02, section 3):
    a = min(gate, gate_max), u = clip(up, -up_max, up_max); infinity = plain SwiGLU.
    """
    x, gate_up, down = _host(x), _host(gate_up), _host(down)
    sh_gate, sh_up, sh_down = _host(sh_gate), _host(sh_up), _host(sh_down)
    dt = _dt(x)
    for t in (gate_up, down, sh_gate, sh_up, sh_down):
        if _dt(t) != dt:
            raise TypeError("all expert tensors must share x's dtype")
    N, D = x.shape
    E, two_d, D2 = gate_up.shape
    d = two_d // 2
    d_sh = sh_gate.shape[0]
    assert D2 == D and tuple(down.shape) == (E, D, d)
    assert tuple(sh_up.shape) == (d_sh, D) and tuple(sh_down.shape) == (D, d_sh)
    idx = np.ascontiguousarray(np.asarray(idx), dtype=np.int32)
    w = np.ascontiguousarray(np.asarray(w), dtype=np.float64)
    k = idx.shape[1]
    assert idx.shape == (N, k) and w.shape == (N, k)
    if tokens is None:
        tokens = np.arange(N, dtype=np.int32)
    tokens = np.ascontiguousarray(np.asarray(tokens), dtype=np.int32)
    y = np.empty((len(tokens), D), dtype=np.float64)
    rc = _load().oracle_forward(_ptr(x), _ptr(gate_up), _ptr(down), _ptr(sh_gate), _ptr(sh_up),
                                _ptr(sh_down), dt, _ptr(idx), _ptr(w), N, D, E, d, d_sh, k,
                                _ptr(tokens), len(tokens), float(gate_max), float(up_max),
                                _ptr(y))
    if rc != 0:
        raise ValueError("oracle_forward rejected its arguments (token or expert id out of range)")
    return y


def _silu_np(a: np.ndarray) -> np.ndarray:
    return a / (1.0 + np.exp(-a))


def forward_expert_major(x, gate_up, down, sh_gate, sh_up, sh_down, idx, w) -> np.ndarray:
    """Second formulation of the same y, expert-major with a scatter-add, fp64 numpy.

    Follows the order the GLM-5 "Mixture of experts" page describes for the experts'
    forward: for every hit expert, gather its tokens, apply the SwiGLU expert, scale
    by the routing weight of that (token, slot) and add into the output; then add
    the shared expert on the same input.  Used only to cross-check `forward`.
    """
    f = lambda t: _host(t).to(torch.float64).numpy()
    X, GU, DN = f(x), f(gate_up), f(down)
    SG, SU, SD = f(sh_gate), f(sh_up), f(sh_down)
    idx = np.asarray(idx)
    w = np.asarray(w, dtype=np.float64)
    N, D = X.shape
    E = GU.shape[0]
    d = GU.shape[1] // 2
    out = np.zeros((N, D), dtype=np.float64)
    for e in np.unique(idx):
        if e == E:
            continue
        tok, slot = np.nonzero(idx == e)
        xs = X[tok]
        a = xs @ GU[e, :d, :].T
        u = xs @ GU[e, d:, :].T
        o = (_silu_np(a) * u) @ DN[e].T
        np.add.at(out, tok, o * w[tok, slot][:, None])
    out += (_silu_np(X @ SG.T) * (X @ SU.T)) @ SD.T
    return out


def param_counts(D: int, E: int, d: int, n_shared: int = 1, router_bias: bool = True) -> dict:
    """Parameter accounting of one MoE block (GLM-5 "Mixture of experts", Parameters table).

    A SwiGLU expert holds gate, up (d x D each) and down (D x d): 3 D d.  The router
    holds W_g (E x D) plus, as a buffer, the E correction-bias values.
    """
    expert = 3 * D * d
    shared = 3 * D * d * n_shared
    router_p = E * D + (E if router_bias else 0)
    return {"expert": expert, "routed": E * expert, "shared": shared, "router": router_p,
            "block": E * expert + shared + router_p}


def bias_update(idx, E: int, rate: float, b) -> tuple:
    """One step of the loss-free balancer ("GLM-4.5 Group Router", How it works: the
    bias b is updated from expert load during training, at rate 0.001 for the first
    15T tokens, then 0).  The pages give the rate, not the rule; this follows the
    plainest reading of the loss-free balancing they cite: every expert's bias moves
    by `rate` towards the mean load, b_e += rate * sign(mean_load - load_e), with the
    load counted over the routed (token, slot) pairs (the sentinel id E and any id
    outside [0, E) count for nobody) and the comparison made exactly in integers
    (sign(total - E * load_e)).  b is the fp32 buffer; the sum is taken in fp64 and
    rounded once to fp32, as an fp32 add of rate would be.  Returns (b_new, loads).
    parity unpinned: the rule is a reading, its pins check the reading's properties.
    """
    ids = np.asarray(idx).reshape(-1)
    ids = ids[(ids >= 0) & (ids < E)]
    loads = np.bincount(ids, minlength=E).astype(np.int64)
    total = int(loads.sum())
    sign = np.sign(total - E * loads).astype(np.float64)
    b64 = np.asarray(torch.as_tensor(b).detach().cpu().float().numpy(), dtype=np.float64)
    rate32 = float(np.float32(rate))
    b_new = (b64 + rate32 * sign).astype(np.float32)
    return b_new, loads
