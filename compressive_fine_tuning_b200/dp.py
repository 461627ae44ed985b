"""Multi-GPU plumbing of the sketched linear layer (one process per GPU).

Two ways the layer shards, and the one exchange that either needs:

* Fine-tuning shards the token batch.  Every rank runs the forward and both
  backward products on its own tokens with its own copy of the frozen index
  map and the LUTs.  The LUT gradient is a sum over tokens (the corrected Eq. 6
  of the "Sketch to Adapt" OpenReview discussion, reply Q1: the gradient of the
  loss w.r.t. the LUT is dL/dy times (M X) transposed, summed over the batch),
  so summing the per-rank fp32 LUT gradients gives the gradient of the whole
  batch.  That sum is the only exchange: one all-reduce per layer, n * gpr * k
  * 4 bytes, issued on a side stream right after the layer's LUT-gradient
  launch so that it overlaps the backward of the next layer.  It is a few
  microseconds of NVLink traffic against milliseconds of tensor-core work, so
  it stays a library collective (NCCL) rather than a fused kernel.
* Serving may shard the weight rows: each rank keeps the index rows and every
  task's LUT rows of its slice and computes its slice of Y with no exchange.
  Only a consumer that wants the whole Y gathers the slices.

* The sketching stage shards its calibration tokens and then its rows.  The
  Gram matrix is a sum over tokens, so each rank computes it over its own
  calibration shard and one all-reduce (d * d * 4 bytes) gives everyone the
  whole matrix; every rank then factors it (the same launches on the same
  data) and runs Lloyd and the mapping for its own slice of weight rows,
  which need nothing from the other rows.  Only a consumer that wants the
  whole index map or all the LUTs gathers the row blocks.

Everything here is host logic over ``torch.distributed``; the arithmetic runs
in the library's kernels.  The functions accept CPU tensors too (``gloo``), so
the exchange logic can be exercised without a GPU.
"""
from __future__ import annotations

from typing import List, Optional

import torch
import torch.distributed as dist


def token_shard(T: int, rank: int, world: int) -> slice:
    """Contiguous near-equal split of T tokens: the first T % world ranks get
    one token more.  Ranks may receive zero tokens when T < world."""
    if world < 1 or not 0 <= rank < world or T < 0:
        raise ValueError(f"bad shard request T={T} rank={rank} world={world}")
    base, extra = divmod(T, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


def row_shard(n: int, rank: int, world: int, align: int = 8) -> slice:
    """Contiguous split of n weight rows in blocks of `align` rows (the layer
    wants n % 8 == 0 on every rank).  n must be a multiple of `align`."""
    if n % align:
        raise ValueError(f"n={n} is not a multiple of {align}")
    s = token_shard(n // align, rank, world)
    return slice(s.start * align, s.stop * align)


class LutGradReducer:
    """Sums LUT gradients over the ranks of `group`, overlapped with compute.

    ``submit(dlut)`` is called right after the launch that wrote `dlut`, on the
    stream that launched it: the all-reduce is queued on a side stream that
    first waits for that launch.  ``wait()`` makes the current stream wait for
    every submitted reduction (call it before the optimizer reads the
    gradients).  ``average=True`` divides by the world size afterwards (the
    gradient of a loss averaged over the ranks' batches); the default is the
    plain sum.  CPU tensors (gloo) are reduced synchronously.
    """

    def __init__(self, group: Optional[dist.ProcessGroup] = None, average: bool = False):
        self.group = group
        self.average = average
        self.world = dist.get_world_size(group)
        self._stream: Optional[torch.cuda.Stream] = None
        self._pending: List[torch.Tensor] = []

    def _side_stream(self, device: torch.device) -> torch.cuda.Stream:
        if self._stream is None:
            self._stream = torch.cuda.Stream(device)
        return self._stream

    def submit(self, dlut: torch.Tensor) -> None:
        if dlut.dtype != torch.float32:
            raise TypeError("LUT gradients are fp32")
        if self.world == 1:
            return
        if dlut.device.type != "cuda":
            dist.all_reduce(dlut, op=dist.ReduceOp.SUM, group=self.group)
            if self.average:
                dlut.div_(self.world)
            return
        producer = torch.cuda.current_stream(dlut.device)
        side = self._side_stream(dlut.device)
        side.wait_stream(producer)
        with torch.cuda.stream(side):
            dist.all_reduce(dlut, op=dist.ReduceOp.SUM, group=self.group)
            if self.average:
                dlut.div_(self.world)
        dlut.record_stream(side)
        self._pending.append(dlut)

    def wait(self) -> None:
        if self._stream is not None and self._pending:
            torch.cuda.current_stream(self._pending[0].device).wait_stream(self._stream)
        self._pending.clear()


def gather_rows(y_local: torch.Tensor, n: int, group: Optional[dist.ProcessGroup] = None,
                align: int = 8) -> torch.Tensor:
    """Assemble the [T][n] output from every rank's [T][rows of its shard]
    slice (the rows of `row_shard`).  Only for a consumer that needs all of Y."""
    world = dist.get_world_size(group)
    if world == 1:
        return y_local
    T = y_local.shape[0]
    widths = [row_shard(n, r, world, align) for r in range(world)]
    width_max = max(s.stop - s.start for s in widths)
    buf = y_local.new_zeros((T, width_max))
    buf[:, : y_local.shape[1]] = y_local
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf.contiguous(), group=group)
    return torch.cat([p[:, : s.stop - s.start] for p, s in zip(parts, widths)], dim=1)


def reduce_gram(H: torch.Tensor, group: Optional[dist.ProcessGroup] = None) -> torch.Tensor:
    """Sum, in place, the Gram matrices that the ranks computed over their
    shards of the calibration tokens (sk.gram of the local rows of X).  The
    summation order of the all-reduce is the library's, so the sum can differ
    from a single-device Gram matrix in the last bits."""
    if dist.get_world_size(group) > 1:
        dist.all_reduce(H, op=dist.ReduceOp.SUM, group=group)
    return H


def gather_row_blocks(x_local: torch.Tensor, n: int, group: Optional[dist.ProcessGroup] = None,
                      align: int = 8) -> torch.Tensor:
    """Concatenate every rank's block of rows [rows of its shard][...] (the
    rows of `row_shard`) into [n][...], e.g. the index map or the LUTs that
    the ranks sketched for their own rows."""
    world = dist.get_world_size(group)
    if world == 1:
        return x_local
    shards = [row_shard(n, r, world, align) for r in range(world)]
    rows_max = max(sh.stop - sh.start for sh in shards)
    buf = x_local.new_zeros((rows_max,) + tuple(x_local.shape[1:]))
    buf[: x_local.shape[0]] = x_local
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf.contiguous(), group=group)
    return torch.cat([p[: sh.stop - sh.start] for p, sh in zip(parts, shards)], dim=0)
