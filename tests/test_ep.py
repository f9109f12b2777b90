"""Expert parallelism (EP): the route bookkeeping, the exchange steps of
EPGroup.forward over 2 and 4 gloo ranks on the CPU, and (on a GPU) the EP
kernels with the ranks emulated on one GPU -- each against the single-rank
oracle on the same tokens.

On the CPU the device steps are the oracle's (the oracle computes every
expert FFN in fp64), so these runs check the bookkeeping and collectives
exactly: the per-rank counts, the W x W count matrix, the send / receive
offsets, the all-to-all splits and the return order.  The structure is the
TPU kernel's on the page "tpu_inference/kernels/fused_moe/v1/kernel.py"
(all_reduce_metadata, start_a2a_scatter, start_a2a_gather, bt_acc)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from moe_inputs import make_inputs  # noqa: E402
from mixture_experts_expert_softmax_b200 import ep  # noqa: E402


# ------------------------------------------------------------------ bookkeeping
def test_routes_small_matrix():
    # counts[s][d]: rows rank s sends to rank d
    c = [[2, 0, 3],
         [1, 4, 0],
         [0, 2, 5]]
    rt = ep.routes(c)
    assert rt.send_off == [[0, 2, 2, 5], [0, 1, 5, 5], [0, 0, 2, 7]]
    assert rt.recv_off == [[0, 2, 3, 3], [0, 0, 4, 6], [0, 3, 3, 8]]
    # rank 1's rows for rank 2 start after rank 0's rows there (none from 1)
    assert rt.pack_row0[1] == [2, 0, 3] and rt.pack_row0[2] == [3, 4, 3]
    # rank 2's results for rank 0 go back to rank 0's send-order rows 2..4
    assert rt.ret_row0[2] == [2, 5, 2]


def test_routes_rejects_bad_counts():
    with pytest.raises(ValueError):
        ep.routes([[1, 2], [3]])
    with pytest.raises(ValueError):
        ep.routes([[1, -1], [0, 0]])


def test_routes_every_row_lands_once():
    rng = np.random.default_rng(0)
    for w in (1, 2, 3, 5, 8):
        c = rng.integers(0, 7, (w, w)).tolist()
        rt = ep.routes(c)
        for d in range(w):
            slots = []
            for s in range(w):
                a = rt.pack_row0[s][d]
                slots += list(range(a, a + c[s][d]))
            assert sorted(slots) == list(range(rt.recv_off[d][w]))  # a permutation
        for s in range(w):  # the return fills the sender's send order exactly
            back = []
            for d in range(w):
                a = rt.ret_row0[d][s]
                back += list(range(a, a + c[s][d]))
            assert sorted(back) == list(range(rt.send_off[s][w]))


def test_owner_of_blocks():
    assert [ep.owner_of(e, 8, 4) for e in range(8)] == [0, 0, 1, 1, 2, 2, 3, 3]


# ------------------------------------------------------------------ CPU steps
class OracleOps:
    """EP device steps restated on the host with the oracle: the stable
    grouping by owner rank, row copies, the fp64 expert FFN and the combine
    in slot order."""

    def dispatch_plan(self, ids, E, world):
        ids_np = ids.numpy()
        per = E // world
        owner = np.where((ids_np >= 0) & (ids_np < E), ids_np // per, -1).astype(np.int32)
        rows, offs = oracle.permute(owner, world)
        n = ids_np.size
        inv = np.full(n, -1, np.int32)
        nv = int(offs[-1])
        inv[rows[:nv]] = np.arange(nv)
        return torch.as_tensor(rows.astype(np.int32)), [int(x) for x in offs], torch.as_tensor(inv)

    def pack(self, hidden, ids, E, world, send_rows, send_off, dst_x, dst_eid, dst_row0):
        k = ids.shape[1]
        per = E // world
        flat_ids = ids.reshape(-1)
        for d in range(world):
            for r in range(send_off[d], send_off[d + 1]):
                q = dst_row0[d] + r - send_off[d]
                f = int(send_rows[r])
                dst_x[d][q] = hidden[f // k]
                dst_eid[d][q] = int(flat_ids[f]) - d * per

    def expert_ffn(self, x, w1, w2, eid):
        n = x.shape[0]
        if n == 0:
            return torch.empty(0, x.shape[1], dtype=torch.float64)
        y = oracle.moe_token_loop(x, w1, w2, np.ones((n, 1)), eid.numpy().reshape(n, 1))
        return torch.as_tensor(y)

    def ret(self, y, world, recv_off, dst_y, dst_row0):
        for s in range(world):
            for q in range(recv_off[s], recv_off[s + 1]):
                dst_y[s][dst_row0[s] + q - recv_off[s]] = y[q]

    def combine(self, y_back, inv, weights, H):
        T, k = weights.shape
        out = torch.zeros(T, H, dtype=torch.float64)
        for t in range(T):
            for j in range(k):
                r = int(inv[t * k + j])
                if r >= 0:
                    out[t] += float(weights[t, j]) * y_back[r].double()
        return out


def _rank_inputs(rank, T, H, I, E, k, seed):
    """Every rank draws the same full expert weights and its own tokens."""
    _, w1, w2, _ = make_inputs(1, H, I, E, seed=seed)
    hidden, _, _, logits = make_inputs(T, H, I, E, seed=seed + 100 + rank)
    ids, w = oracle.route(logits.numpy(), k, True)
    return hidden, w1, w2, torch.as_tensor(ids), torch.as_tensor(w)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ep_worker(rank, world, port, shape, q):
    try:
        sys.path.insert(0, ROOT)
        from datetime import timedelta
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=timedelta(seconds=60))
        T, H, I, E, k = shape
        hidden, w1, w2, ids, w = _rank_inputs(rank, T + 3 * rank, H, I, E, k, seed=9)
        if rank == 1:
            ids[0, 0] = -1  # an invalid id: skipped on every rank's side
        per = E // world
        # the oracle steps keep the expert outputs in fp64 through the
        # exchange, so every rank must reproduce the single-rank oracle
        group = ep.EPGroup(E, ops=OracleOps())
        out = group.forward(hidden, w1[rank * per:(rank + 1) * per],
                            w2[rank * per:(rank + 1) * per], w, ids)
        ref = oracle.moe_token_loop(hidden, w1, w2, w.numpy(), ids.numpy())
        err = float(np.max(np.abs(out.numpy() - ref) / (1e-6 + np.abs(ref))))
        dist.destroy_process_group()
        q.put((rank, err, None))
    except Exception as e:  # report instead of hanging the parent
        import traceback
        q.put((rank, None, traceback.format_exc()))


@pytest.mark.parametrize("world,shape", [(2, (13, 128, 128, 8, 2)), (4, (9, 256, 128, 16, 4)),
                                         (4, (5, 128, 256, 8, 8)), (8, (6, 128, 128, 16, 3))])
def test_ep_gloo_ranks_match_single_rank_oracle(world, shape):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, shape, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, err, tb = q.get(timeout=180)
        res[rank] = (err, tb)
    for p in procs:
        p.join(timeout=60)
    for rank, (err, tb) in sorted(res.items()):
        assert tb is None, f"rank {rank}:\n{tb}"
        assert err < 1e-9, f"rank {rank}: relative error {err}"


# ------------------------------------------------------------------ GPU
@pytest.mark.gpu
@pytest.mark.parametrize("world,shape", [(1, (64, 256, 128, 8, 2)), (2, (300, 512, 256, 8, 2)),
                                         (4, (200, 384, 256, 16, 4)), (4, (100, 256, 128, 128, 8))])
def test_ep_virtual_ranks_on_one_gpu(world, shape):
    """The CUDA dispatch plan, pack (rows stored into the receiving rank's
    buffer), expert FFNs (moe_forward, top-k 1), return and combine, with
    `world` ranks emulated on one GPU, against the oracle on each rank's
    tokens with all E experts."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from moe_testutil import assert_output_close
    import mixture_experts_expert_softmax_b200 as moe
    T, H, I, E, k = shape
    per = E // world
    dev = torch.device("cuda")
    ins = [_rank_inputs(r, T + 17 * r, H, I, E, k, seed=5) for r in range(world)]
    hid = [i[0].to(dev) for i in ins]
    w1 = [ins[0][1][r * per:(r + 1) * per].contiguous().to(dev) for r in range(world)]
    w2 = [ins[0][2][r * per:(r + 1) * per].contiguous().to(dev) for r in range(world)]
    ids = [i[3].to(dev) for i in ins]
    wts = [i[4].float().to(dev) for i in ins]
    outs = ep.forward_local(hid, w1, w2, wts, ids, E)
    torch.cuda.synchronize()
    assert moe.get_device_status() == 0
    for r in range(world):
        ref = oracle.moe_token_loop(ins[r][0], ins[0][1], ins[0][2], ins[r][4].numpy(),
                                    ins[r][3].numpy())
        assert_output_close(outs[r].cpu().numpy(), ref, f"rank {r} of {world}")


@pytest.mark.gpu
def test_ep_group_over_nccl_one_rank():
    """EPGroup.forward with the CUDA steps over a one-rank NCCL group: the
    count all-gather and the three all_to_all_single exchanges run through
    NCCL (trivially, with one rank)."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from datetime import timedelta
    from moe_testutil import assert_output_close
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60))
    try:
        T, H, I, E, k = 150, 256, 128, 8, 2
        hidden, w1, w2, ids, w = _rank_inputs(0, T, H, I, E, k, seed=6)
        dev = torch.device("cuda")
        group = ep.EPGroup(E)
        out = group.forward(hidden.to(dev), w1.to(dev), w2.to(dev), w.float().to(dev),
                            ids.to(dev))
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref = oracle.moe_token_loop(hidden, w1, w2, w.numpy(), ids.numpy())
    assert_output_close(out.cpu().numpy(), ref, "EPGroup, one NCCL rank")
