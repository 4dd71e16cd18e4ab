"""Expert-parallel FFN pool over several GPUs: the exchange around the layer call.

FastAFD, "Methodology / System Design": attention GPUs publish FP8 tokens and routing
metadata into pre-allocated receive buffers on the FFN GPUs (item 2); the FFN GPUs run the
expert layer and push the results back (M2N, item 3). With the experts sharded over F FFN
GPUs, each holding a disjoint range [e0, e0 + E_l), every FFN GPU needs each token whose
top-K touches its range. Here every token goes to every FFN GPU (the FP8 slabs are small
next to the expert weights), each FFN GPU skips the ids it does not hold and writes a
partial sum per token, and the return path adds the F partials of every token.

One process per GPU; rank r plays attention rank r (it owns M_local slabs) and FFN rank r.
Transport, on one torch.distributed process group (NCCL on GPUs, gloo in the CPU tests):
  dispatch  all_gather_into_tensor of every slab field from each rank's send buffers into
            the receive buffers, laid out as F x M_local slabs (slab s came from rank
            s // M_local);
  combine   reduce_scatter_tensor, summing in fp32, of the F ranks' partial outputs, so
            that rank r receives the sum over FFN ranks for its own slabs, then one
            rounding to bf16 into its slabs' output rows.
The layer itself is passed in as a callable (an FfnLayer on a GPU).

PeerEpExchange is the same exchange over mapped peer memory instead of collectives: each
rank exposes its receive buffers and its accumulators to the other ranks (CUDA IPC on
GPUs, so that reads and writes cross NVLink; shared memory on the CPU), the attention side
copies its slabs straight into every FFN rank's receive buffers (item 2), every FFN
rank's down projection adds its partial rows straight into the owning rank's fp32
accumulators (item 3; afd_ffn_set_combine_targets), and after a barrier the owner rounds
each sum once to bf16 (afd_combine_finalize).
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Dict, List, Optional

import torch
import torch.distributed as dist


@dataclasses.dataclass
class SlabView:
    x: torch.Tensor             # uint8 [cap, H]
    x_scale: torch.Tensor       # float32 [cap, H/128]
    topk_ids: torch.Tensor      # int32 [cap, K]
    topk_weights: torch.Tensor  # float32 [cap, K]
    y: torch.Tensor             # bf16 [cap, H]


class EpExchange:
    """Send and receive buffers of one EP-sharded FFN layer on this rank.

    The attention side writes its M_local slabs into `send` (views of contiguous
    [M_local, cap, ...] buffers) and its row counts into `send_counts`; `step(layer_fn)`
    then dispatches, runs `layer_fn(recv_slabs, recv_counts)` (which must write each
    received slab's partial output into its `y`) and returns the summed outputs in `out`
    ([M_local, cap, H] bf16; rows >= n_m are zero).
    """

    def __init__(self, num_local_slabs: int, capacity: int, hidden: int, top_k: int,
                 device, group=None):
        self.group = group
        self.F = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        M, cap, H, K = num_local_slabs, capacity, hidden, top_k
        self.M, self.cap, self.H, self.K = M, cap, H, K
        kw = dict(device=device)
        MF = M * self.F
        self._send = {
            "x": torch.zeros((M, cap, H), dtype=torch.uint8, **kw),
            "x_scale": torch.zeros((M, cap, H // 128), dtype=torch.float32, **kw),
            "topk_ids": torch.full((M, cap, K), -1, dtype=torch.int32, **kw),
            "topk_weights": torch.zeros((M, cap, K), dtype=torch.float32, **kw),
        }
        self.send_counts = torch.zeros(M, dtype=torch.int32, **kw)
        self._recv = {k: torch.empty((MF,) + tuple(v.shape[1:]), dtype=v.dtype, **kw)
                      for k, v in self._send.items()}
        self.recv_counts = torch.zeros(MF, dtype=torch.int32, **kw)
        self._recv_y = torch.zeros((MF, cap, H), dtype=torch.bfloat16, **kw)
        self._partial = torch.empty((MF, cap, H), dtype=torch.float32, **kw)
        self._sum = torch.empty((M, cap, H), dtype=torch.float32, **kw)
        self.out = torch.zeros((M, cap, H), dtype=torch.bfloat16, **kw)
        self.send = [SlabView(self._send["x"][m], self._send["x_scale"][m], self._send["topk_ids"][m],
                              self._send["topk_weights"][m], self.out[m]) for m in range(M)]
        self.recv = [SlabView(self._recv["x"][s], self._recv["x_scale"][s], self._recv["topk_ids"][s],
                              self._recv["topk_weights"][s], self._recv_y[s]) for s in range(MF)]

    def dispatch(self) -> None:
        """Every rank's slabs into every rank's receive buffers (slab s from rank s // M)."""
        for k, buf in self._send.items():
            dist.all_gather_into_tensor(self._recv[k], buf, group=self.group)
        dist.all_gather_into_tensor(self.recv_counts, self.send_counts, group=self.group)

    def combine(self) -> None:
        """Sum the F partial outputs of this rank's slabs (fp32) into `out` (bf16)."""
        self._partial.copy_(self._recv_y)
        dist.reduce_scatter_tensor(self._sum, self._partial, op=dist.ReduceOp.SUM, group=self.group)
        self.out.copy_(self._sum)

    def step(self, layer_fn: Callable[[List[SlabView], torch.Tensor], None]) -> torch.Tensor:
        self.dispatch()
        self._recv_y.zero_()
        layer_fn(self.recv, self.recv_counts)
        self.combine()
        return self.out


def share_views(tensors: Dict[str, torch.Tensor], group=None) -> List[Dict[str, torch.Tensor]]:
    """Every rank's `tensors` as tensors of this process: this rank's own, the others' as
    mappings of their memory (CUDA IPC handles for CUDA tensors, whose pages are then read
    and written over NVLink; shared-memory files for CPU tensors, with the file_system
    sharing strategy). The handles travel with one all_gather_object; the owners must keep
    their tensors alive while the views are used."""
    import pickle
    from multiprocessing.reduction import ForkingPickler
    import torch.multiprocessing  # noqa: F401  (registers the tensor reductions used below)
    F = dist.get_world_size(group)
    me = dist.get_rank(group)
    if F == 1:
        return [tensors]
    # torch's inter-process tensor reductions: the pickled form names the memory (an IPC
    # handle, a shared-memory file) instead of copying it
    mine = {k: bytes(ForkingPickler.dumps(t)) for k, t in tensors.items()}
    every: List[Optional[dict]] = [None] * F
    dist.all_gather_object(every, mine, group=group)
    out = []
    for r, handles in enumerate(every):
        out.append(tensors if r == me else {k: pickle.loads(b) for k, b in handles.items()})
    return out


class PeerEpExchange:
    """The EP exchange over mapped peer memory (one process per GPU, rank r = attention rank
    r = FFN rank r, M_local slabs per attention rank).

    Buffers of this rank, mapped by every other rank:
      recv     [F*M_local, cap, ...] slab fields and counts: slab s holds attention rank
               s // M_local's slab s % M_local (the FFN side's receive buffers);
      acc      [M_local, cap, H] fp32: the sums of this rank's own tokens, added into by
               every FFN rank's down projection, zero between steps.
    The attention side writes its slabs into `send` and `send_counts` (local); `step`
    copies them into every rank's receive buffers, runs `layer_fn(recv_slabs, recv_counts,
    targets)` (the FFN layer over every received slab, adding received slab s's rows into
    targets[s], i.e. into the owner's accumulator), waits for every rank, and runs
    `finalize_fn(out_slabs, send_counts, accs)` (bf16 of the sums into `out`, accumulators
    cleared; ffn.combine_finalize on a GPU).
    """

    def __init__(self, num_local_slabs: int, capacity: int, hidden: int, top_k: int, device,
                 group=None):
        self.group = group
        self.F = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        M, cap, H, K = num_local_slabs, capacity, hidden, top_k
        self.M, self.cap, self.H, self.K = M, cap, H, K
        kw = dict(device=device)
        MF = M * self.F
        self._send = {
            "x": torch.zeros((M, cap, H), dtype=torch.uint8, **kw),
            "x_scale": torch.zeros((M, cap, H // 128), dtype=torch.float32, **kw),
            "topk_ids": torch.full((M, cap, K), -1, dtype=torch.int32, **kw),
            "topk_weights": torch.zeros((M, cap, K), dtype=torch.float32, **kw),
        }
        self.send_counts = torch.zeros(M, dtype=torch.int32, **kw)
        own = {k: torch.zeros((MF,) + tuple(v.shape[1:]), dtype=v.dtype, **kw) for k, v in self._send.items()}
        own["counts"] = torch.zeros(MF, dtype=torch.int32, **kw)
        own["acc"] = torch.zeros((M, cap, H), dtype=torch.float32, **kw)
        self._own = own
        self._peers = share_views(own, group)
        self.out = torch.zeros((M, cap, H), dtype=torch.bfloat16, **kw)
        # the FFN side's slabs need an output row buffer; with combine targets set nothing
        # is written to it, so every received slab shares one
        self._recv_y = torch.zeros((cap, H), dtype=torch.bfloat16, **kw)
        self.send = [SlabView(self._send["x"][m], self._send["x_scale"][m], self._send["topk_ids"][m],
                              self._send["topk_weights"][m], self.out[m]) for m in range(M)]
        self.recv = [SlabView(own["x"][s], own["x_scale"][s], own["topk_ids"][s], own["topk_weights"][s],
                              self._recv_y) for s in range(MF)]
        self.recv_counts = own["counts"]
        # received slab s adds into the accumulator of its owner's slab
        self.targets = [self._peers[s // M]["acc"][s % M] for s in range(MF)]
        self.accs = [own["acc"][m] for m in range(M)]

    def dispatch(self) -> None:
        """This rank's slabs into every rank's receive buffers (peer copies), then a barrier:
        every rank's receive buffers are complete when it returns."""
        lo, hi = self.rank * self.M, (self.rank + 1) * self.M
        for peer in self._peers:
            for k, buf in self._send.items():
                peer[k][lo:hi].copy_(buf, non_blocking=True)
            peer["counts"][lo:hi].copy_(self.send_counts, non_blocking=True)
        dist.barrier(group=self.group)

    def step(self, layer_fn: Callable, finalize_fn: Callable) -> torch.Tensor:
        self.dispatch()
        layer_fn(self.recv, self.recv_counts, self.targets)
        dist.barrier(group=self.group)      # every FFN rank's additions have landed
        finalize_fn(self.send, self.send_counts, self.accs)
        return self.out
