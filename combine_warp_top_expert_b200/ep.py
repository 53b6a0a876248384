"""Expert parallelism across GPUs: the MoE layer with every GPU owning E/R experts.

Page "Expert Parallelism" §1 (experts on GPUs in contiguous blocks) and §4 "The
All-to-All": DISPATCH counts the tokens per GPU, exchanges the counts and then the
token rows, so that every GPU holds a contiguous run of rows per expert it owns;
COMPUTE runs each GPU's experts as one grouped GEMM; COMBINE returns every result
to the GPU its token came from and sums it with its gate.

The exchanges are done by the library's kernels over peer memory (include/moe.h,
"Expert parallelism across GPUs"). This module only allocates the peer-mapped
buffers, builds the device tables of their addresses, and issues the C ABI calls
of one layer call in order. It holds none of the method's arithmetic.

Two ways to get the peer buffers:
  EPPeers.symmetric(group, ...)  one process per GPU; the buffers are PyTorch
                                 symmetric memory, mapped into every rank over NVLink;
  EPPeers.emulated(R, ...)       R ranks' buffers on one GPU (tests): the calls of
                                 the R ranks are then issued phase by phase
                                 (run_emulated), so every wait finds what it waits
                                 for already signalled and no kernel waits on
                                 another one still to run.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import combine_warp_top_expert_b200 as moe


@dataclass
class EPPeers:
    """Peer-mapped buffers of R ranks (this process's views) and the device tables of
    their addresses, as moe_ep_peers_t wants them."""
    R: int
    E: int
    d: int
    rows_cap: int
    counts: list          # R views of int32 [R, E] count tables (only [rank] is local memory across GPUs)
    recv: list            # R views of bf16 [rows_cap, d] receive buffers
    y: list               # R views of bf16 [rows_cap, d] expert-output buffers
    flags: list           # R views of uint64 [4, R] flags
    tables: dict          # name -> int64 device tensor [R] of addresses
    keep_alive: Optional[list] = None

    def c(self) -> "moe.moe_ep_peers_t":
        t = self.tables
        return moe.moe_ep_peers_t(t["counts"].data_ptr(), t["recv"].data_ptr(), t["y"].data_ptr(),
                                  t["flags"].data_ptr(), self.rows_cap)

    @staticmethod
    def _tables(ptrs: dict, device) -> dict:
        import torch
        return {k: torch.tensor(v, dtype=torch.int64, device=device) for k, v in ptrs.items()}

    @classmethod
    def emulated(cls, R: int, E: int, d: int, rows_cap: int, device="cuda") -> "EPPeers":
        """R ranks' buffers on one GPU."""
        import torch
        counts = [torch.zeros((R, E), dtype=torch.int32, device=device) for _ in range(R)]
        recv = [torch.zeros((rows_cap, d), dtype=torch.bfloat16, device=device) for _ in range(R)]
        y = [torch.zeros((rows_cap, d), dtype=torch.bfloat16, device=device) for _ in range(R)]
        flags = [torch.zeros((4, R), dtype=torch.int64, device=device) for _ in range(R)]
        ptrs = dict(counts=[t.data_ptr() for t in counts], recv=[t.data_ptr() for t in recv],
                    y=[t.data_ptr() for t in y], flags=[t.data_ptr() for t in flags])
        return cls(R, E, d, rows_cap, counts, recv, y, flags, cls._tables(ptrs, device))

    @classmethod
    def symmetric(cls, group, E: int, d: int, rows_cap: int, device) -> "EPPeers":
        """One rank's view of buffers in PyTorch symmetric memory (every rank of `group`
        calls this together). Only this rank's own buffers are returned as tensors; the
        peers' are reached by the kernels through the address tables."""
        import torch
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm_mem
        R, rank = dist.get_world_size(group), dist.get_rank(group)
        own, ptrs, handles = {}, {}, []
        for name, numel, dtype in (("counts", R * E, torch.int32), ("recv", rows_cap * d, torch.bfloat16),
                                   ("y", rows_cap * d, torch.bfloat16), ("flags", 4 * R, torch.int64)):
            t = symm_mem.empty(numel, dtype=dtype, device=device)
            t.zero_()
            h = symm_mem.rendezvous(t, group)
            handles.append(h)
            own[name] = t
            ptrs[name] = list(h.buffer_ptrs)
        torch.cuda.synchronize(device)
        dist.barrier(group)  # every rank's flags are zero before anyone signals
        views = {k: [None] * R for k in own}
        views["counts"][rank] = own["counts"].view(R, E)
        views["recv"][rank] = own["recv"].view(rows_cap, d)
        views["y"][rank] = own["y"].view(rows_cap, d)
        views["flags"][rank] = own["flags"].view(4, R)
        return cls(R, E, d, rows_cap, views["counts"], views["recv"], views["y"], views["flags"],
                   cls._tables(ptrs, device), keep_alive=handles + list(own.values()))


class EPMoELayer:
    """Rank `rank`'s part of an expert-parallel MoE layer: its own batch of shape.T tokens,
    the weights of its experts [rank*E/R, (rank+1)*E/R) (w13 [E/R, 2f, d], w2 [E/R, d, f]),
    a shared expert on its own tokens if shape.n_shared (w13s, w2s: every rank holds them)."""

    def __init__(self, shape: "moe.Shape", rank: int, w13, w2, peers: EPPeers, w13s=None, w2s=None, device="cuda"):
        import torch
        R, E = shape.R, shape.E
        if E % R or peers.R != R or peers.E != E or peers.d != shape.d:
            raise ValueError("the peers' R, E and d must match the shape, and E % R == 0")
        self.shape, self.rank, self.peers = shape, rank, peers
        self.w13, self.w2, self.w13s, self.w2s = w13, w2, w13s, w2s
        Er = E // R
        self.ws = moe.new_workspace(shape, device)
        self.shape_recv = moe.Shape(T=peers.rows_cap, d=shape.d, E=Er, k=1, f=shape.f, R=1)
        self.ws_recv = moe.new_workspace(self.shape_recv, device)
        i32, f32, bf = torch.int32, torch.float32, torch.bfloat16
        T, k, d = shape.T, shape.k, shape.d
        self.topk_idx = torch.empty((T, k), dtype=i32, device=device)
        self.topk_gate = torch.empty((T, k), dtype=f32, device=device)
        self.expert_counts = torch.empty((E,), dtype=i32, device=device)
        self.send_row = torch.empty((T * k,), dtype=i32, device=device)
        self.recv_offsets = torch.empty((Er + 1,), dtype=i32, device=device)
        self.out = torch.empty((T, d), dtype=bf, device=device)
        self.y_shared = None
        if shape.n_shared:
            self.shape_sh = moe.Shape(T=T, d=d, E=1, k=1, f=shape.f, R=1)
            self.ws_sh = moe.new_workspace(self.shape_sh, device)
            self.offs_sh = torch.tensor([0, T], dtype=i32, device=device)
            self.y_shared = torch.empty((T, d), dtype=bf, device=device)
        self.epoch = 0
        self._x = None

    # one layer call, in phases (run_emulated issues each phase for every rank in turn)
    def route_and_count(self, logits):
        self.epoch += 1
        moe.moe_route(self.shape, logits, self.topk_idx, self.topk_gate, self.ws)
        moe.moe_ep_exchange_counts(self.shape, self.rank, self.epoch, self.topk_idx, self.expert_counts, self.peers,
                                   self.ws)

    def send(self, x):
        self._x = x
        moe.moe_ep_dispatch(self.shape, self.rank, self.epoch, x, self.topk_idx, self.send_row, self.recv_offsets,
                            self.peers, self.ws)

    def compute(self):
        R, p = self.shape.R, self.peers
        moe.moe_ep_wait(R, self.rank, moe.EP_SLOT_ROWS, self.epoch, p, self.ws)
        moe.moe_expert_ffn(self.shape_recv, p.recv[self.rank], self.recv_offsets, self.w13, self.w2, None, None, None,
                           p.y[self.rank], None, self.ws_recv)
        if self.shape.n_shared:
            moe.moe_expert_ffn(self.shape_sh, self._x, self.offs_sh, self.w13s.unsqueeze(0), self.w2s.unsqueeze(0),
                               None, None, None, self.y_shared, None, self.ws_sh)
        moe.moe_ep_signal(R, self.rank, moe.EP_SLOT_OUTPUTS, self.epoch, p)

    def combine(self):
        moe.moe_ep_combine(self.shape, self.rank, self.epoch, self.send_row, self.topk_idx, self.topk_gate,
                           self.y_shared, self.out, self.peers, self.ws)

    def end(self):
        moe.moe_ep_wait(self.shape.R, self.rank, moe.EP_SLOT_DONE, self.epoch, self.peers, self.ws)

    def __call__(self, logits, x):
        """The whole layer call on this rank (one process per GPU)."""
        self.route_and_count(logits)
        self.send(x)
        self.compute()
        self.combine()
        self.end()
        return self.out

    def status(self) -> int:
        return moe.get_status(self.ws) | moe.get_status(self.ws_recv) | (
            moe.get_status(self.ws_sh) if self.shape.n_shared else 0)


def run_emulated(layers: List[EPMoELayer], logits: list, xs: list):
    """One layer call of R ranks emulated on one GPU: each phase for every rank, in order."""
    for r, lay in enumerate(layers):
        lay.route_and_count(logits[r])
    for r, lay in enumerate(layers):
        lay.send(xs[r])
    for lay in layers:
        lay.compute()
    for lay in layers:
        lay.combine()
    for lay in layers:
        lay.end()
    return [lay.out for lay in layers]
