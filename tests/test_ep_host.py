"""Host logic of the expert-parallel path (no GPU): the receive layout every rank
derives from the exchanged expert histograms, checked by brute force, on two gloo
ranks that really exchange their histograms, and the C ABI's argument checks.

The layout ("GLM-5.3-Flash Module 02", expert placement: each token's hidden
state goes to the device that holds each of its top-k experts): rank q owns
experts [q*E/P, (q+1)*E/P); its receive buffer holds, per local expert in order,
a 128-row padded segment with the rows of rank 0's pairs, then rank 1's, ... each
in that rank's (token, slot) order.  Every sender must address exactly those rows
and no two pairs may share one.
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import sparse_moe_layer_02_b200 as moe

TILE = 128


def _check_layout(P, E, counts, plans):
    """Every pair of every sender lands on its own row, and the rows of each receiver
    are exactly its segments' first R rows, sources in rank order."""
    E_loc = E // P
    dense_off = np.concatenate([np.zeros((P, 1), np.int64), np.cumsum(counts, 1)], 1)
    for q in range(P):
        R = counts[:, q * E_loc:(q + 1) * E_loc].sum(0)
        tiles = (R + TILE - 1) // TILE
        np.testing.assert_array_equal(plans[q]["rcounts"], R)
        np.testing.assert_array_equal(plans[q]["rtile_off"], np.concatenate([[0], np.cumsum(tiles)]))
        assert plans[q]["rows_in"] == R.sum()
        for el in range(E_loc):
            e = q * E_loc + el
            got = []
            for r in range(P):
                base = plans[r]["dest_base"][e] + dense_off[r, e]
                got.extend(base + np.arange(counts[r, e]))
            seg = plans[q]["rtile_off"][el] * TILE
            np.testing.assert_array_equal(np.array(got, np.int64), seg + np.arange(R[el]))
    for r in range(P):
        assert plans[r]["pairs_out"] == counts[r].sum()


@pytest.mark.parametrize("P,E", [(1, 8), (2, 16), (4, 16), (8, 64), (4, 256)])
def test_plan_places_every_pair_once(P, E):
    rng = np.random.default_rng(P * 1000 + E)
    for trial in range(5):
        # loads from empty to several tiles, some experts with exact tile multiples
        counts = rng.integers(0, 300, size=(P, E)).astype(np.int32)
        counts[rng.random((P, E)) < 0.2] = 0
        if trial == 1:
            counts[:] = 0
        if trial == 2:
            counts[:, 0] = TILE
        plans = [moe.moe_ep_plan_host(P, r, counts) for r in range(P)]
        _check_layout(P, E, counts.astype(np.int64), plans)


def test_plan_rejects_bad_shapes():
    c = np.zeros((2, 6), np.int32)
    with pytest.raises(moe.MoEError):
        moe.moe_ep_plan_host(2, 2, c)           # rank out of range
    with pytest.raises(moe.MoEError):
        moe.moe_ep_plan_host(4, 0, np.zeros((4, 6), np.int32))  # E % P != 0


def test_buffer_sizes_and_argument_checks():
    lib = moe.load_library()
    assert moe.moe_ep_symmetric_bytes(3, 64, 256, 16, 4) == 0          # E % P
    assert moe.moe_ep_symmetric_bytes(9, 64, 256, 72, 4) == 0          # P > 8
    small = moe.moe_ep_symmetric_bytes(2, 64, 256, 16, 4)
    assert small > 2 * 64 * 4 * 256 * 2                                 # recv rows of all pairs
    assert moe.moe_ep_symmetric_bytes(2, 128, 256, 16, 4) > small
    assert moe.moe_ep_workspace_bytes(2, 64, 256, 16, 128, 128, 4) > 0
    import ctypes
    peers = (ctypes.c_void_p * 2)(256, 512)
    call = lambda **kw: lib.moe_ep_forward(
        kw.get("phases", 15), kw.get("P", 2), kw.get("rank", 0), kw.get("epoch", 1),
        kw.get("peers", peers), 64, *([16] * 8), kw.get("N", 10), 256, kw.get("E", 16), 128, 128,
        kw.get("k", 4), 16, kw.get("ws", 256), kw.get("wsb", 1 << 30), None)
    assert call(phases=0) == -1
    assert call(phases=16) == -1
    assert call(P=9) == -1
    assert call(rank=2) == -1
    assert call(epoch=0) == -1
    assert call(E=15) == -2
    assert call(N=65) == -2                                             # N > N_cap
    assert call(k=33) == -2
    assert call(peers=(ctypes.c_void_p * 2)(256, 0)) == -1
    assert call(peers=(ctypes.c_void_p * 2)(256, 100)) == -1            # not 256-byte aligned
    assert call(ws=0) == -4
    assert call(wsb=16) == -4


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        E, k = 16, 4
        N = [37, 301][rank]
        rng = np.random.default_rng(100 + rank)
        idx = np.stack([rng.permutation(E)[:k] for _ in range(N)]).astype(np.int32)
        idx[rng.random(idx.shape) < 0.05] = E          # a few sentinel ids go nowhere
        counts = np.bincount(idx[idx < E], minlength=E).astype(np.int32)
        allc = [torch.zeros(E, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(allc, torch.from_numpy(counts))
        matrix = torch.stack(allc).numpy()
        plan = moe.moe_ep_plan_host(world, rank, matrix)
        plans = [None] * world
        dist.all_gather_object(plans, plan)
        mats = [None] * world
        dist.all_gather_object(mats, matrix)
        ok = all(np.array_equal(m, mats[0]) for m in mats)
        _check_layout(world, E, matrix.astype(np.int64), plans)
        q.put((rank, ok, plan["rows_in"], plan["pairs_out"], int((idx < E).sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_exchange():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ok0, in0, out0, v0), (r1, ok1, in1, out1, v1) = out
    assert ok0 and ok1                     # both ranks hold the same histogram matrix
    assert out0 == v0 and out1 == v1       # every routed pair is sent, sentinels are not
    assert in0 + in1 == v0 + v1            # and received exactly once
