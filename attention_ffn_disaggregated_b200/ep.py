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
"""
from __future__ import annotations

import dataclasses
from typing import Callable, List

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
