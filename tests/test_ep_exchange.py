"""Expert parallelism on the CPU: the exchange plan (moe_ep_plan, host code of the library) and
the dispatch / combine All-to-All of sparse_mixture_experts_warp_b200.ep on 2 gloo ranks.

"Top-k 路由", "通訊拓撲：All-to-All": every row goes to the rank holding its expert and its output
comes back.  What each rank must hold after the dispatch is fixed by the single-device layer:
for each of its experts, the rows that expert would get from the ranks' batches laid end to
end, i.e. the oracle's dispatch (rows of an expert in ascending (token, slot) order) of the
concatenated batch when nothing is dropped, and the concatenation over source ranks of each
source's own dispatch under a per-rank capacity limit.  The rows are checked bit for bit
(token ids and the row payloads), and the reverse exchange must hand every rank back exactly
the rows it sent.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import moe_oracle as O
from sparse_mixture_experts_warp_b200 import ep
from sparse_mixture_experts_warp_b200.workloads import WORKLOADS, make_inputs, scaled


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _local_layout(plan, recv):
    """Expert-major layout of a source-major receive buffer, from the plan's blocks."""
    out = np.zeros((max(plan.recv_total, 0),) + recv.shape[1:], dtype=recv.dtype)
    for b in range(plan.G * plan.Eg):
        n = plan.block_rows[b]
        out[plan.block_local[b]:plan.block_local[b] + n] = \
            recv[plan.block_recv[b]:plan.block_recv[b] + n]
    return out


def test_plan_blocks_tile_both_layouts():
    """moe_ep_plan on random counts (host only): the blocks tile the receive buffer in
    (source, expert) order and the local layout in (expert, source) order, and the split sizes
    add up."""
    rng = np.random.default_rng(5)
    for G, Eg in [(1, 8), (2, 4), (4, 2), (8, 1), (3, 5)]:
        send = rng.integers(0, 40, size=G * Eg)
        recv = rng.integers(0, 40, size=G * Eg)
        recv[rng.integers(G * Eg)] = 0                     # an empty block
        p = ep.ep_plan(G, Eg, send.tolist(), recv.tolist())
        assert p.send_rows == [int(send[r * Eg:(r + 1) * Eg].sum()) for r in range(G)]
        assert p.send_offsets == [int(send[:r * Eg].sum()) for r in range(G)]
        assert p.recv_rows == [int(recv[s * Eg:(s + 1) * Eg].sum()) for s in range(G)]
        # label every received row by its (source, expert) block and check both layouts
        lab_recv = np.concatenate([[b] * int(recv[b]) for b in range(G * Eg)] or [[]])
        lab_local = _local_layout(p, lab_recv.reshape(-1, 1)).reshape(-1)
        want = np.concatenate([[s * Eg + e] * int(recv[s * Eg + e])
                               for e in range(Eg) for s in range(G)] or [[]])
        np.testing.assert_array_equal(lab_local, want)
        counts_e = [int(sum(recv[s * Eg + e] for s in range(G))) for e in range(Eg)]
        assert p.local_offsets == [0] + np.cumsum(counts_e).tolist()
        assert p.max_block_rows == int(recv.max())


def test_plan_rejects_bad_counts():
    with pytest.raises(Exception):
        ep.ep_plan(2, 2, [1, -1, 0, 0], [0, 0, 0, 0])


def _rank_main(rank, world, port, wname, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = {"mixtral": scaled(WORKLOADS["mixtral"], T=37, D=64, E=8, F=64),
             "switch": scaled(WORKLOADS["switch"], T=50, D=64, E=8, F=64)}[wname]
        G, Eg, T, k = world, w.E // world, w.T, w.k
        # every rank draws the same global batch; rank r owns tokens [r T, (r+1) T)
        glob = make_inputs(scaled(w, T=G * T), seed=3, device="cpu", experts=False)
        x_all = glob.x.float().numpy().astype(np.float64)
        Wg = glob.Wg.float().numpy().astype(np.float64)
        ids_all, _, _ = O.route_token_choice(O.router_logits(x_all, Wg), k, w.score, w.gate)
        cap = O.capacity(w.capacity_factor, T, k, w.E) if w.overflow == "drop" else None
        disp = [O.dispatch_token_choice(ids_all[s * T:(s + 1) * T], w.E, cap) for s in range(G)]
        _, kept, _, row_src, _ = disp[rank]
        # the send buffer a rank's permute produces: its rows grouped by expert, and their
        # (global token, slot) labels
        tok = rank * T + row_src // k
        send_x = glob.x[torch.as_tensor(tok)].contiguous()
        send_lab = torch.as_tensor(np.stack([tok, row_src % k], 1), dtype=torch.int64)
        a2a = ep.DistAllToAll()
        rows_recv = ep.exchange_counts(a2a, [torch.as_tensor(kept, dtype=torch.int32)], Eg)[0]
        plan = ep.ep_plan(G, Eg, kept.tolist(), rows_recv.tolist())
        recv_x = ep.exchange_rows(a2a, [send_x], [plan], w.D, send_x.dtype)[0]
        recv_lab = ep.exchange_rows(a2a, [send_lab], [plan], 2, torch.int64)[0]
        loc_lab = _local_layout(plan, recv_lab[:plan.recv_total].numpy())
        loc_x = _local_layout(plan, recv_x[:plan.recv_total].view(torch.int16).numpy())
        # expected: per local expert, the sources' kept rows in source order
        want = []
        for e in range(rank * Eg, (rank + 1) * Eg):
            for s in range(G):
                _, _, off_s, rs_s, _ = disp[s]
                rows = rs_s[off_s[e]:off_s[e + 1]]
                want.extend(zip(s * T + rows // k, rows % k))
        want = np.asarray(want, dtype=np.int64).reshape(-1, 2)
        np.testing.assert_array_equal(loc_lab, want)
        np.testing.assert_array_equal(loc_x, glob.x[torch.as_tensor(want[:, 0])]
                                      .view(torch.int16).numpy())
        if cap is None:
            # dropless: exactly the single-device dispatch of the whole batch
            _, _, off_g, rs_g, _ = O.dispatch_token_choice(ids_all, w.E)
            rows_g = rs_g[off_g[rank * Eg]:off_g[(rank + 1) * Eg]]
            np.testing.assert_array_equal(loc_lab[:, 0], rows_g // k)
        # the reverse exchange returns every row to the slot it left from
        back = ep.exchange_rows(a2a, [recv_x], [plan], w.D, send_x.dtype, reverse=True)[0]
        assert torch.equal(back[:len(tok)], send_x)
        out[rank] = (int(plan.recv_total), int(plan.send_total))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("wname", ["mixtral", "switch"])
def test_two_rank_dispatch_matches_oracle(wname):
    world = 2
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), wname, out), nprocs=world,
                           join=True, start_method="spawn")
        res = dict(out)
    # every row that left a rank arrived somewhere
    assert sum(r for r, _ in res.values()) == sum(s for _, s in res.values())
