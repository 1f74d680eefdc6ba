"""Expert parallelism on one GPU: P ranks emulated phase by phase.

Each rank holds E/P experts and its own tokens; the ranks exchange token rows and
expert outputs through each other's symmetric buffers (here all on one device).
Running every rank's count phase, then every rank's send phase, and so on, means
each bounded wait in the kernels is already satisfied when it starts, so no kernel
ever waits for another one that is still running.

The expert rows go through the same prefill kernels, with the same operand rows,
weights and k-block order as on one device, so each rank's y must equal
moe_forward's on that rank's tokens bit for bit (token counts above 256, where
moe_forward takes those kernels); smaller batches are compared within the bf16
bound, and one rank against the oracle.
"""

import numpy as np
import pytest
import torch

import oracle
import sparse_moe_layer_02_b200 as moe
from workloads import CONFIGS, make_inputs

from _parity import Y_TOL, rel_err

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _reset_hooks():
    moe.moe_debug_set_wait_limit_ns(0)
    yield
    moe.moe_debug_set_wait_limit_ns(0)


class _Ranks:
    def __init__(self, P, N_cap, D, E, k, d, d_sh):
        self.P, self.N_cap, self.E = P, N_cap, E
        self.syms = [torch.zeros(moe.moe_ep_symmetric_bytes(P, N_cap, D, E, k), dtype=torch.uint8,
                                 device=DEV) for _ in range(P)]
        self.wss = [torch.empty(moe.moe_ep_workspace_bytes(P, N_cap, D, E, d, d_sh, k),
                                dtype=torch.uint8, device=DEV) for _ in range(P)]
        self.peers = [s.data_ptr() for s in self.syms]

    def run(self, epoch, inp, xs, ids, wts, phases=moe.MOE_EP_PHASES, ranks=None):
        E_loc = self.E // self.P
        ys = [torch.empty_like(x) for x in xs]
        for ph in phases:
            for r in (range(self.P) if ranks is None else ranks):
                moe.moe_ep_forward(ph, self.P, r, epoch, self.peers, self.N_cap, xs[r],
                                   inp.gate_up[r * E_loc:(r + 1) * E_loc],
                                   inp.down[r * E_loc:(r + 1) * E_loc], inp.sh_gate, inp.sh_up,
                                   inp.sh_down, ids[r], wts[r], self.E, ys[r], self.wss[r])
        return ys


def _batch(inp, Ns, k, seed, sentinel_frac=0.03):
    D = inp.x.shape[1]
    E = inp.gate_up.shape[0]
    g = torch.Generator(device=DEV).manual_seed(seed)
    z = torch.randn(sum(Ns), D, generator=g, device=DEV)
    x_all = (z / z.pow(2).mean(1, keepdim=True).add(1e-6).sqrt()).to(torch.bfloat16)
    idx, w = moe.moe_router(x_all, inp.W_g, inp.b, 1, 1, k, True, 2.5)
    drop = torch.rand(idx.shape, generator=g, device=DEV) < sentinel_frac
    idx = torch.where(drop, torch.full_like(idx, E), idx).contiguous()
    offs = np.cumsum([0] + list(Ns))
    cut = lambda t: [t[offs[r]:offs[r + 1]].contiguous() for r in range(len(Ns))]
    return cut(x_all), cut(idx), cut(w)


@pytest.mark.parametrize("P,Ns", [(2, [300, 520]), (4, [257, 300, 0, 400]),
                                  (8, [260, 270, 280, 290, 300, 310, 320, 330])])
def test_ep_emulated_equals_single_device(P, Ns):
    E = 16 if P <= 4 else 32
    k, D, d, d_sh = 4, 256, 128, 192
    cfg = CONFIGS["glm5_prefill"].with_(N=8, D=D, E=E, k=k, d_moe=d, d_sh=d_sh)
    inp = make_inputs(cfg, seed=3, device=DEV)
    ranks = _Ranks(P, max(Ns), D, E, k, d, d_sh)
    for epoch in (1, 2, 3):  # both counter parities, and a reset
        xs, ids, wts = _batch(inp, Ns, k, seed=epoch)
        ys = ranks.run(epoch, inp, xs, ids, wts)
        assert moe.moe_device_status() == 0
        for r in range(P):
            if Ns[r] == 0:
                continue
            y_ref = moe.moe_forward(xs[r], inp.gate_up, inp.down, inp.sh_gate, inp.sh_up,
                                    inp.sh_down, ids[r], wts[r])
            assert torch.equal(ys[r], y_ref), (epoch, r)
    # rank 0 of the last epoch against the oracle
    host = lambda t: t.cpu()
    y_orc = oracle.forward(host(xs[0]), host(inp.gate_up), host(inp.down), host(inp.sh_gate),
                           host(inp.sh_up), host(inp.sh_down), host(ids[0]).numpy(),
                           host(wts[0]).double().numpy())
    e = rel_err(ys[0].float().cpu().numpy(), y_orc)
    assert e["max_rel"] <= Y_TOL[torch.bfloat16] and e["max_row_l2_rel"] <= Y_TOL[torch.bfloat16]


def test_ep_emulated_small_batches():
    P, Ns, E, k, D, d, d_sh = 2, [5, 64], 16, 8, 256, 128, 128
    cfg = CONFIGS["glm5_decode"].with_(N=8, D=D, E=E, k=k, d_moe=d, d_sh=d_sh)
    inp = make_inputs(cfg, seed=4, device=DEV)
    ranks = _Ranks(P, 64, D, E, k, d, d_sh)
    xs, ids, wts = _batch(inp, Ns, k, seed=9)
    ys = ranks.run(1, inp, xs, ids, wts)
    assert moe.moe_device_status() == 0
    for r in range(P):
        y_ref = moe.moe_forward(xs[r], inp.gate_up, inp.down, inp.sh_gate, inp.sh_up,
                                inp.sh_down, ids[r], wts[r])
        err = rel_err(ys[r].float().cpu().numpy(), y_ref.float().cpu().numpy())
        assert err["max_rel"] <= Y_TOL[torch.bfloat16]
        assert err["max_row_l2_rel"] <= Y_TOL[torch.bfloat16]


def test_ep_missing_rank_times_out_and_context_survives():
    # rank 1 never publishes its histogram: rank 0's send phase gives up after the
    # wait limit, reports a timeout and sends nothing; the device stays usable.
    P, Ns, E, k, D, d, d_sh = 2, [300, 300], 16, 4, 256, 128, 128
    cfg = CONFIGS["glm5_prefill"].with_(N=8, D=D, E=E, k=k, d_moe=d, d_sh=d_sh)
    inp = make_inputs(cfg, seed=5, device=DEV)
    ranks = _Ranks(P, 300, D, E, k, d, d_sh)
    xs, ids, wts = _batch(inp, Ns, k, seed=11)
    moe.moe_debug_set_wait_limit_ns(20_000_000)
    ranks.run(1, inp, xs, ids, wts, phases=(moe.MOE_EP_COUNT, moe.MOE_EP_SEND), ranks=[0])
    assert moe.moe_device_status() == -6  # MOE_ERR_DEVICE_TIMEOUT
    moe.moe_debug_set_wait_limit_ns(0)
    fresh = _Ranks(P, 300, D, E, k, d, d_sh)
    ys = fresh.run(1, inp, xs, ids, wts)
    assert moe.moe_device_status() == 0
    y_ref = moe.moe_forward(xs[1], inp.gate_up, inp.down, inp.sh_gate, inp.sh_up, inp.sh_down,
                            ids[1], wts[1])
    assert torch.equal(ys[1], y_ref)
