"""Expert-parallel (EP) MoE forward over `world` ranks, one per GPU.

Rank r owns the experts [r * E / world, (r + 1) * E / world) and routes its
own tokens; a forward sends every (token, slot) row to the owner of its
expert, runs the expert FFNs of the rows each rank received and sends the
results back for the fixed-order weighted sum.  This is the structure of
the TPU kernel on the page "tpu_inference/kernels/fused_moe/v1/kernel.py":
the per-device expert counts are exchanged first (all_reduce_metadata; here
an all-gather of every rank's per-destination row counts, the W x W count
matrix), then the scatter of token rows to the owners (start_a2a_scatter),
the expert FFNs, the gather back to the token owner (start_a2a_gather) and
the sum over the k results in slot order (bt_acc).

Two drivers share the route bookkeeping (`routes`):

* `EPGroup.forward`: one process per rank over torch.distributed (NCCL on
  GPUs, gloo on CPU).  Rows are packed into a local send buffer in send
  order and exchanged with all_to_all_single, then the results likewise.
* `forward_local`: `world` ranks emulated in one process on one GPU; the
  pack and return kernels store every row straight into the receiving
  rank's buffer, as they would into peer-mapped memory of other GPUs.

The device steps (`Ops`) are the library's CUDA kernels by default; tests
on a CPU-only host pass their own (oracle-based) steps to exercise the
bookkeeping and the collectives.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


# ------------------------------------------------------------------ bookkeeping
@dataclass
class Routes:
    """Where every row goes, from the W x W count matrix counts[s][d] (rows
    rank s sends to rank d)."""
    send_off: list[list[int]]   # [s][0..W]: segment offsets of s's send order
    recv_off: list[list[int]]   # [d][0..W]: segment offsets of d's receive order (by source)
    pack_row0: list[list[int]]  # [s][d]: first row of s's rows in d's receive buffer
    ret_row0: list[list[int]]   # [d][s]: first row of d's results in s's send-order buffer


def _prefix(xs):
    out = [0]
    for x in xs:
        out.append(out[-1] + int(x))
    return out


def routes(counts: list[list[int]]) -> Routes:
    w = len(counts)
    if any(len(row) != w for row in counts) or any(c < 0 for row in counts for c in row):
        raise ValueError("counts must be a square matrix of non-negative row counts")
    send_off = [_prefix(counts[s]) for s in range(w)]
    recv_off = [_prefix(counts[s][d] for s in range(w)) for d in range(w)]
    pack_row0 = [[recv_off[d][s] for d in range(w)] for s in range(w)]
    ret_row0 = [[send_off[s][d] for s in range(w)] for d in range(w)]
    return Routes(send_off, recv_off, pack_row0, ret_row0)


def owner_of(expert: int, E: int, world: int) -> int:
    """The rank that owns a (global) expert id."""
    return expert // (E // world)


# ------------------------------------------------------------------ device steps
class Ops:
    """The device steps of an EP forward on one rank (the library's CUDA
    kernels through its C ABI)."""

    def __init__(self):
        import mixture_experts_expert_softmax_b200 as moe
        self.moe = moe

    def dispatch_plan(self, ids: torch.Tensor, E: int, world: int):
        """-> send_rows [T*k] int32, send_off (host list of world+1), inv [T*k] int32."""
        moe = self.moe
        T, k = ids.shape
        rows = torch.empty(T * k, dtype=torch.int32, device=ids.device)
        offs = torch.empty(world + 1, dtype=torch.int32, device=ids.device)
        inv = torch.empty(T * k, dtype=torch.int32, device=ids.device)
        moe._check(moe._lib.moe_ep_dispatch_plan(ids.data_ptr(), T, k, E, world, rows.data_ptr(),
                                                 offs.data_ptr(), inv.data_ptr(),
                                                 moe._stream(None)), "moe_ep_dispatch_plan")
        return rows, [int(x) for x in offs.cpu().tolist()], inv

    def pack(self, hidden, ids, E, world, send_rows, send_off, dst_x, dst_eid, dst_row0):
        moe = self.moe
        import ctypes
        T, k = ids.shape
        c_i64 = (ctypes.c_int64 * (world + 1))(*send_off)
        c_row0 = (ctypes.c_int64 * world)(*dst_row0)
        c_x = (ctypes.c_void_p * world)(*[None if t is None else t.data_ptr() for t in dst_x])
        c_e = (ctypes.c_void_p * world)(*[None if t is None else t.data_ptr() for t in dst_eid])
        moe._check(moe._lib.moe_ep_pack(hidden.data_ptr(), hidden.shape[1], ids.data_ptr(), T, k,
                                        E, world, send_rows.data_ptr(), c_i64, c_x, c_e, c_row0,
                                        moe._stream(None)), "moe_ep_pack")

    def expert_ffn(self, x, w1, w2, eid):
        """y[r] = FFN_{eid[r]}(x[r]) (top-k 1, weight 1): [rows, H] fp32."""
        n = x.shape[0]
        if n == 0:
            return torch.empty(0, x.shape[1], dtype=torch.float32, device=x.device)
        ones = torch.ones(n, 1, dtype=torch.float32, device=x.device)
        return self.moe.moe_forward(x, w1, w2, ones, eid.view(n, 1))

    def ret(self, y, world, recv_off, dst_y, dst_row0):
        moe = self.moe
        import ctypes
        c_off = (ctypes.c_int64 * (world + 1))(*recv_off)
        c_row0 = (ctypes.c_int64 * world)(*dst_row0)
        c_y = (ctypes.c_void_p * world)(*[None if t is None else t.data_ptr() for t in dst_y])
        moe._check(moe._lib.moe_ep_return(y.data_ptr() if y.numel() else None, y.shape[1], world,
                                          c_off, c_y, c_row0, moe._stream(None)), "moe_ep_return")

    def combine(self, y_back, inv, weights, H):
        moe = self.moe
        T, k = weights.shape
        out = torch.empty(T, H, dtype=torch.float32, device=weights.device)
        moe._check(moe._lib.moe_ep_combine(y_back.data_ptr(), inv.data_ptr(), weights.data_ptr(),
                                           out.data_ptr(), T, H, k, moe._stream(None)),
                   "moe_ep_combine")
        return out


# ------------------------------------------------------------------ drivers
class EPGroup:
    """One rank of an EP group over torch.distributed (the default process
    group unless `group` is given).  w1 / w2 hold this rank's E / world
    experts: [E/world, 2I, H] and [E/world, H, I] bf16."""

    def __init__(self, E: int, ops: Ops | None = None, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if E % self.world:
            raise ValueError(f"E={E} must be a multiple of the world size {self.world}")
        self.E = E
        self.ops = ops if ops is not None else Ops()

    def exchange_counts(self, send_counts: list[int], device) -> list[list[int]]:
        """All-gather of every rank's per-destination row counts: the W x W
        matrix counts[s][d]."""
        mine = torch.tensor(send_counts, dtype=torch.int64, device=device)
        parts = [torch.empty_like(mine) for _ in range(self.world)]
        self.dist.all_gather(parts, mine, group=self.group)
        return [[int(x) for x in p.cpu().tolist()] for p in parts]

    def forward(self, hidden, w1, w2, weights, ids):
        """This rank's tokens: hidden [T, H] bf16, weights / ids [T, k] ->
        out [T, H] fp32 (every rank calls it, in the same order)."""
        W, r, ops, dist = self.world, self.rank, self.ops, self.dist
        T, H = hidden.shape
        dev = hidden.device
        send_rows, send_off, inv = ops.dispatch_plan(ids, self.E, W)
        counts = self.exchange_counts([send_off[d + 1] - send_off[d] for d in range(W)], dev)
        rt = routes(counts)
        n_send, n_recv = send_off[W], rt.recv_off[r][W]
        # pack in send order into a local buffer, then the all-to-all
        send_x = torch.empty(max(n_send, 1), H, dtype=hidden.dtype, device=dev)
        send_e = torch.empty(max(n_send, 1), dtype=torch.int32, device=dev)
        ops.pack(hidden, ids, self.E, W, send_rows, send_off, [send_x] * W, [send_e] * W,
                 send_off[:W])
        s_split = [counts[r][d] for d in range(W)]
        r_split = [counts[s][r] for s in range(W)]
        recv_x = torch.empty(n_recv, H, dtype=hidden.dtype, device=dev)
        recv_e = torch.empty(n_recv, dtype=torch.int32, device=dev)
        dist.all_to_all_single(recv_x, send_x[:n_send], r_split, s_split, group=self.group)
        dist.all_to_all_single(recv_e, send_e[:n_send], r_split, s_split, group=self.group)
        y = ops.expert_ffn(recv_x, w1, w2, recv_e)
        y_back = torch.empty(max(n_send, 1), H, dtype=y.dtype, device=dev)
        dist.all_to_all_single(y_back[:n_send], y.contiguous(), s_split, r_split, group=self.group)
        return ops.combine(y_back, inv, weights, H)


def forward_local(hidden: list, w1: list, w2: list, weights: list, ids: list, E: int,
                  ops: Ops | None = None) -> list:
    """`world = len(hidden)` ranks emulated in one process: rank r's tokens
    hidden[r], weights[r], ids[r] and its experts w1[r], w2[r].  The pack
    and return kernels store every row straight into the receiving rank's
    buffer (peer stores on a real multi-GPU node).  Returns every rank's
    out [T_r, H] fp32."""
    ops = ops if ops is not None else Ops()
    W = len(hidden)
    H = hidden[0].shape[1]
    dev = hidden[0].device
    plans = [ops.dispatch_plan(ids[r], E, W) for r in range(W)]
    counts = [[plans[s][1][d + 1] - plans[s][1][d] for d in range(W)] for s in range(W)]
    rt = routes(counts)
    recv_x = [torch.empty(max(rt.recv_off[d][W], 1), H, dtype=hidden[d].dtype, device=dev)
              for d in range(W)]
    recv_e = [torch.empty(max(rt.recv_off[d][W], 1), dtype=torch.int32, device=dev)
              for d in range(W)]
    for s in range(W):
        rows, off, _ = plans[s]
        ops.pack(hidden[s], ids[s], E, W, rows, off, recv_x, recv_e, rt.pack_row0[s])
    y_back = [torch.empty(max(plans[s][1][W], 1), H, dtype=torch.float32, device=dev)
              for s in range(W)]
    for d in range(W):
        n = rt.recv_off[d][W]
        y = ops.expert_ffn(recv_x[d][:n], w1[d], w2[d], recv_e[d][:n])
        ops.ret(y, W, rt.recv_off[d], y_back, rt.ret_row0[d])
    return [ops.combine(y_back[s], plans[s][2], weights[s], H) for s in range(W)]


__all__ = ["Routes", "routes", "owner_of", "Ops", "EPGroup", "forward_local"]
