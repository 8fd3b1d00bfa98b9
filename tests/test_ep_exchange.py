"""The expert-parallel exchange on CPU ranks (gloo, world size 2 and 4).

mixture_experts_softmax_b200.ep.ep_forward composes the layer's three device steps with
its all-to-all exchanges.  Here the device steps are stood in for by the fp64 oracle on
the host (routing + stable grouping, one expert FFN per received row, the gate-weighted
sum in slot order), so the test pins the exchange itself: every rank's output equals
oracle.forward on its own tokens bit for bit, every rank receives exactly the rows of
its experts in source order (each source's rows grouped by expert, ascending token
order), and padding tokens are neither sent nor given an output.  The same ep_forward,
with the CUDA steps, is checked on one GPU in test_gpu_ep.py.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

E, D, F = 8, 256, 512


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _tokens(rank):
    """Each rank's own batch (different sizes, one of them a small one) and padding mask."""
    import moe_synth
    T = [37, 5, 64, 1][rank % 4]
    g = moe_synth.generator(100 + rank, "cpu")
    x = moe_synth.draw_tokens(T, D, g, "cpu")
    mask = (torch.rand(T, generator=g) > 0.25).to(torch.uint8)
    mask[0] = 1
    return x, mask


def _rank_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    import moe_synth
    import oracle
    from mixture_experts_softmax_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        layer = moe_synth.make_inputs("tiny", device="cpu").layers[0]   # the same model on every rank
        x, mask = _tokens(rank)
        T = x.shape[0]
        first, last = ep.expert_range(E, world, rank)
        state = {}

        def dispatch():
            r = oracle.route(x, layer["router_w"])
            idx = np.where(mask.numpy()[:, None] != 0, r["idx"], -1).astype(np.int32)
            counts, offsets, perm = oracle.dispatch(idx, E)
            n = int(offsets[-1])
            state.update(idx=idx, gate=np.where(idx >= 0, r["gate"], 0.0), perm=perm[:n])
            rows = x[torch.from_numpy(perm[:n] // 2).long()]
            return rows, torch.from_numpy(counts.astype(np.int32))

        def experts(recv_counts, recv_rows):
            rc = recv_counts.numpy()
            state["recv_counts"], state["recv_rows"] = rc, recv_rows.clone()
            # received rows: source after source, each source's rows grouped by local expert
            experts_of_rows = [first + k for s in range(world) for k in range(last - first) for _ in range(rc[s, k])]
            assert len(experts_of_rows) == recv_rows.shape[0]
            y = np.zeros((recv_rows.shape[0], D))
            xr = recv_rows.to(torch.float64).numpy()
            for i, e in enumerate(experts_of_rows):
                y[i] = oracle.expert_ffn(xr[i], layer, e, nthreads=1)
            return torch.from_numpy(y)

        def combine(y_back):
            pos = np.full(2 * T, -1)
            pos[state["perm"]] = np.arange(len(state["perm"]))
            yb = y_back.numpy()
            out = np.zeros((T, D))
            for t in range(T):
                if state["idx"][t, 0] < 0:
                    continue
                out[t] = state["gate"][t, 0] * yb[pos[2 * t]] + state["gate"][t, 1] * yb[pos[2 * t + 1]]
            return out

        out = ep.ep_forward(dispatch, experts, combine, world, E)
        ref, ridx, _ = oracle.forward(layer, x, mask=mask.numpy(), nthreads=1)
        # what this rank should have received: from each source, its real tokens' routes to
        # this rank's experts, grouped by expert, ascending token order
        want = []
        for s in range(world):
            xs, ms = _tokens(s)
            rs = oracle.route(xs, layer["router_w"])
            for e in range(first, last):
                for t in range(xs.shape[0]):
                    if ms[t] and e in rs["idx"][t]:
                        want.append(xs[t])
        want = torch.stack(want) if want else torch.empty((0, D), dtype=torch.bfloat16)
        q.put((rank, bool(np.array_equal(out, ref)), bool(torch.equal(state["recv_rows"], want)),
               bool((ridx[mask.numpy() == 0] == -1).all()), int(state["recv_rows"].shape[0])))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ep_exchange_matches_oracle(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, exact, rows_ok, pad_ok, nrecv in res:
        assert exact, f"rank {rank}: output differs from oracle.forward"
        assert rows_ok, f"rank {rank}: received rows not in the documented order"
        assert pad_ok
    assert sum(r[4] for r in res) > 0


def test_plan_exchange():
    from mixture_experts_softmax_b200 import ep
    send = [3, 0, 2, 5, 1, 1, 0, 4]
    recv = [[3, 0], [7, 1], [0, 0], [2, 2]]
    assert ep.plan_exchange(send, recv, 4) == ([3, 7, 2, 4], [3, 8, 0, 4])
    assert ep.expert_range(8, 4, 3) == (6, 8)
    with pytest.raises(ValueError):
        ep.expert_range(8, 3, 0)


def test_local_all_to_all_is_the_exchange():
    """local_all_to_all (one process holding every rank's buffers) delivers what the rank-wise
    all-to-all delivers: rank r gets, from each source in order, that source's rows for r."""
    from mixture_experts_softmax_b200 import ep
    sends = [torch.arange(5).view(5, 1), torch.arange(10, 13).view(3, 1)]
    splits = [[2, 3], [1, 2]]
    got = ep.local_all_to_all(sends, splits)
    assert got[0].view(-1).tolist() == [0, 1, 10]
    assert got[1].view(-1).tolist() == [2, 3, 4, 11, 12]
