"""moe_forward_noalloc: the forward for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc on the hot path, for example a plugin inside
a serving runtime that owns all device memory, or a latency-critical loop where
an allocation could synchronise the device.  For them the library keeps a 64 MiB
device scratch of its own.  These tests call that entry point through the C ABI
and check it against the workspace entry point, moe_forward, on two calls in a
row (the second call finds the first call's leftovers in the shared scratch).

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""

import ctypes

import pytest
import torch

import sparse_moe_layer_02_b200 as moe
from workloads import CONFIGS, make_inputs

from _parity import Y_TOL, rel_err

CASES = {
    # more than 256 tokens: the 128-row tile kernels and the combine launch
    "bf16": CONFIGS["glm5_prefill"].with_(N=300, D=512, E=8, k=4, d_moe=256, d_sh=256),
    # at most 256 tokens: the decode kernels, whose down kernel waits on a per-call
    # tile counter in the scratch before it combines (the latency-bound callers)
    "bf16_decode": CONFIGS["air_decode"].with_(N=64, D=1024, E=32, k=8, d_moe=512, d_sh=512),
    "fp32": CONFIGS["tiny_fp32"],
}


@pytest.mark.gpu
@pytest.mark.parametrize("case", list(CASES))
def test_noalloc_matches_workspace_entry_point_twice(case):
    cfg = CASES[case]
    lib = moe.load_library()
    dev = "cuda:0"
    torch.cuda.set_device(0)
    inp = make_inputs(cfg, seed=11, device=dev)
    idx, w = moe.moe_router(inp.x, inp.W_g, inp.b, cfg.n_group, cfg.topk_group, cfg.k,
                            cfg.norm_topk_prob, cfg.alpha)
    y_ref = moe.moe_forward(inp.x, inp.gate_up, inp.down, inp.sh_gate, inp.sh_up, inp.sh_down,
                            idx, w)
    assert moe.moe_device_status() == 0
    dtype = moe.MOE_BF16 if cfg.dtype == torch.bfloat16 else moe.MOE_F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        y = torch.full_like(y_ref, float("nan"))
        rc = lib.moe_forward_noalloc(
            inp.x.data_ptr(), inp.gate_up.data_ptr(), inp.down.data_ptr(),
            inp.sh_gate.data_ptr(), inp.sh_up.data_ptr(), inp.sh_down.data_ptr(),
            idx.data_ptr(), w.data_ptr(), cfg.N, cfg.D, cfg.E, cfg.d_moe, cfg.d_sh, cfg.k, dtype,
            y.data_ptr(), stream)
        assert rc == 0, moe.moe_status_string(rc)
        assert moe.moe_device_status() == 0
        err = rel_err(y.float().cpu().numpy(), y_ref.float().cpu().numpy())
        assert err["finite"], "call %d left non-finite values" % call
        assert err["max_rel"] <= Y_TOL[cfg.dtype], (call, err)
        # the same kernels on the same inputs: the forward is deterministic, so the
        # outputs agree bit for bit
        assert torch.equal(y, y_ref), (call, err)


def test_noalloc_refuses_sizes_beyond_its_scratch():
    # The GLM-5 prefill layer needs gigabytes of workspace: refused before any launch.
    lib = moe.load_library()
    c = CONFIGS["glm5_prefill"]
    assert lib.moe_forward_workspace(c.N, c.D, c.E, c.d_moe, c.d_sh, c.k, 1) > (64 << 20)
    rc = lib.moe_forward_noalloc(*([None] * 8), c.N, c.D, c.E, c.d_moe, c.d_sh, c.k, 1, None, None)
    assert rc == -4
    assert lib.moe_forward_noalloc(*([None] * 8), 10, 64, 8, 32, 32, 2, 9, None, None) == -3
    # null pointers are refused before the scratch address is looked up on a device
    assert lib.moe_forward_noalloc(*([None] * 8), 10, 64, 8, 32, 32, 2, 1, None, None) == -1
