"""Data-parallel streaming LM-head loss: token rows sharded across ranks.

Each rank streams its own token rows through the forward and backward.  The loss is a sum
of independent per-token terms normalised by the number of valid tokens of the whole
batch, and the LM-head gradient is a sum over every token ("Training speculative decoders:
removing the logits and attention bottlenecks", "Streaming Cross Entropy": chunking is
over tokens and the mean divides by the total valid count, never by a chunk count; the
technique is orthogonal to data parallelism).  So the ranks exchange exactly three things:

  1. the valid-token count, summed across ranks BEFORE the backward, so each rank's
     upstream gradient is 1 / n_valid(global);
  2. dW, summed across ranks after the backward;
  3. the loss sum, summed across ranks, for the global mean.

dH stays local: each rank owns the gradient of its own hidden states.

dW can also be left sharded by vocabulary rows, as a fully sharded (FSDP-style) optimiser
keeps it: with ``dW_full`` the sum over ranks is a reduce-scatter, and rank r receives rows
[r * Vs, (r + 1) * Vs) of the summed dW, Vs = ceil(V / world).  The backward writes the
first V rows of ``dW_full`` (world * Vs rows, the rest zero), so that every shard has the
same size.

The per-rank compute is passed in as two callables, so the same exchange runs over NCCL
with the CUDA kernels (``cuda_step``) or over any other process group.

Overlap: dW is final when the last token chunk's dW GEMM is done, but the backward still
has that chunk's dH GEMM to run.  ``cuda_step(overlap=True)`` asks the library to run the
last dW GEMM first and record an event there (``slm_loss_bwd_overlap``), and sums dW
across ranks on a side stream that waits on that event, so the reduction runs while the
last dH GEMM does.  That GEMM leaves ``reserve_sms`` SMs idle for the reduction's kernels.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Any, Callable

import torch
import torch.distributed as dist


@dataclass
class DPResult:
    loss_mean: torch.Tensor   # float64 [1], global mean over valid tokens (0 if none)
    loss_sum: torch.Tensor    # float64 [1], global sum
    n_valid: torch.Tensor     # int64 [1], global count
    dH: torch.Tensor          # this rank's rows
    dW: torch.Tensor          # summed over ranks: all V rows, or this rank's shard
    dW_rows: tuple | None = None  # (first, end) vocabulary rows of the shard, end <= V


def shard_rows(V: int, world: int) -> int:
    """Vocabulary rows per rank when dW is reduce-scattered: ceil(V / world)."""
    return -(-int(V) // int(world))


def dw_full_buffer(V: int, d: int, world: int, device) -> torch.Tensor:
    """A zeroed fp32 [world * shard_rows(V, world), d] buffer; the backward writes its first
    V rows (pass ``buf[:V]`` as dW), the padding rows stay zero."""
    return torch.zeros(world * shard_rows(V, world), d, dtype=torch.float32, device=device)


def _sum_dW(dW, dW_full, group):
    """All-reduce dW in place, or reduce-scatter dW_full by vocabulary rows.  Returns the
    result and its row range (None for the whole of dW)."""
    if dW_full is None:
        dist.all_reduce(dW, group=group)
        return dW, None
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if dW_full.shape[0] % world != 0 or dW.data_ptr() != dW_full.data_ptr():
        raise ValueError("dW must be the first rows of dW_full, whose row count is a "
                         "multiple of the world size")
    rows = dW_full.shape[0] // world
    shard = torch.empty(rows, dW_full.shape[1], dtype=dW_full.dtype, device=dW_full.device)
    dist.reduce_scatter_tensor(shard, dW_full, group=group)
    V = dW.shape[0]
    return shard, (min(rank * rows, V), min((rank + 1) * rows, V))


def fwd_bwd(fwd: Callable[[], Any], bwd: Callable[[Any, torch.Tensor], tuple],
            group=None, comm_stream=None, dW_full=None) -> DPResult:
    """Run one data-parallel forward + backward.

    ``fwd()`` returns an object with ``loss_sum`` (float64 [1]) and ``n_valid`` (int64 [1])
    tensors for this rank's rows.  ``bwd(res, n_valid_global)`` returns (dH, dW) for this
    rank's rows with the upstream gradient 1 / n_valid_global on valid rows, or
    (dH, dW, ready): a ``torch.cuda.Event`` recorded once dW is final.  With a ready event
    and a ``comm_stream``, dW is summed on that stream after the event, overlapping
    whatever the backward still runs on the current stream; the current stream waits for
    the sum before this function returns.
    With ``dW_full`` (see ``dw_full_buffer``; the backward's dW is its first V rows), dW is
    reduce-scattered by vocabulary rows instead of all-reduced, and the result holds this
    rank's shard and its row range.
    Every rank makes the same collective calls in the same order.
    """
    res = fwd()
    n_valid = res.n_valid.clone()
    dist.all_reduce(n_valid, group=group)
    out = bwd(res, n_valid)
    dH, dW = out[0], out[1]
    ready = out[2] if len(out) > 2 else None
    if ready is not None and comm_stream is not None:
        main = torch.cuda.current_stream()
        comm_stream.wait_event(ready)
        with torch.cuda.stream(comm_stream):
            dW_sum, dW_rows = _sum_dW(dW, dW_full, group)
        if dW_sum is not dW:
            # The shard was allocated on the side stream and is used on this one next.
            dW_sum.record_stream(main)
    else:
        comm_stream = None
        dW_sum, dW_rows = _sum_dW(dW, dW_full, group)
    loss_sum = res.loss_sum.clone()
    dist.all_reduce(loss_sum, group=group)
    if comm_stream is not None:
        torch.cuda.current_stream().wait_stream(comm_stream)
    den = n_valid.clamp_min(1).to(loss_sum.dtype)
    loss_mean = torch.where(n_valid > 0, loss_sum / den, torch.zeros_like(loss_sum))
    return DPResult(loss_mean, loss_sum, n_valid, dH, dW_sum, dW_rows)


def fused_fwd_bwd(count: Callable[[], torch.Tensor],
                  fused: Callable[[torch.Tensor], tuple], group=None,
                  dW_full=None) -> DPResult:
    """One data-parallel step through a single-call forward + backward.

    The single call (``slm_loss_fwd_bwd``) forms the gradient of this rank's mean loss, i.e.
    it divides by the rank's own valid count, scaled by ``grad_scale``.  So the counts are
    summed first: ``count()`` returns this rank's valid-row count (int64 [1]), and
    ``fused(scale)`` is called with scale = n_local / n_global (float32 [1]), which turns the
    local mean's gradient into the global mean's.  It returns (res, dH, dW) with
    ``res.loss_sum``.  dW and the loss sum are then summed across ranks, as in ``fwd_bwd``
    (``dW_full``: reduce-scattered by vocabulary rows).
    """
    n_local = count().reshape(1).to(torch.int64)
    n_valid = n_local.clone()
    dist.all_reduce(n_valid, group=group)
    scale = (n_local.to(torch.float64) / n_valid.clamp_min(1).to(torch.float64)).to(torch.float32)
    res, dH, dW = fused(scale)
    dW_sum, dW_rows = _sum_dW(dW, dW_full, group)
    loss_sum = res.loss_sum.clone()
    dist.all_reduce(loss_sum, group=group)
    den = n_valid.clamp_min(1).to(loss_sum.dtype)
    loss_mean = torch.where(n_valid > 0, loss_sum / den, torch.zeros_like(loss_sum))
    return DPResult(loss_mean, loss_sum, n_valid, dH, dW_sum, dW_rows)


_COMM_STREAMS = {}


def comm_stream_for(device) -> torch.cuda.Stream:
    """The side stream this module sums dW on, one per device."""
    idx = torch.device(device).index
    if idx is None:
        idx = torch.cuda.current_device()
    if idx not in _COMM_STREAMS:
        _COMM_STREAMS[idx] = torch.cuda.Stream(device=idx)
    return _COMM_STREAMS[idx]


def cuda_step(kind, hidden, weight, labels=None, target_hidden=None, ignore_index=-100,
              group=None, chunk_tokens=0, workspace=None, out=None, dH=None, dW=None,
              overlap=True, reserve_sms=8, shard_dW=False):
    """Data-parallel step over the CUDA kernels (one rank per GPU, NCCL process group).

    With ``overlap`` the sum of dW over ranks runs on a side stream while the last token
    chunk's dH GEMM runs (on ``reserve_sms`` fewer SMs); the results are the same.
    With ``shard_dW`` dW is reduce-scattered by vocabulary rows (``dW``, if given, must then
    be a ``dw_full_buffer``) and the result holds this rank's shard."""
    from .loss import lm_head_loss_bwd, lm_head_loss_fwd

    dW_full = None
    if shard_dW:
        world = dist.get_world_size(group)
        V, d = weight.shape
        dW_full = dW if dW is not None else dw_full_buffer(V, d, world, hidden.device)
        dW = dW_full[:V]

    def _fwd():
        return lm_head_loss_fwd(kind, hidden, weight, labels, target_hidden, ignore_index,
                                workspace=workspace, chunk_tokens=chunk_tokens, out=out)

    def _bwd(res, n_valid_global):
        # The backward divides by the count it is handed: the global one.
        res.n_valid.copy_(n_valid_global)
        if not overlap:
            return lm_head_loss_bwd(res, hidden, weight, labels, target_hidden, ignore_index,
                                    dH=dH, dW=dW, chunk_tokens=chunk_tokens)
        ready = torch.cuda.Event()
        gh, gw = lm_head_loss_bwd(res, hidden, weight, labels, target_hidden, ignore_index,
                                  dH=dH, dW=dW, chunk_tokens=chunk_tokens, dw_ready=ready,
                                  reserve_sms=reserve_sms)
        return gh, gw, ready

    return fwd_bwd(_fwd, _bwd, group, comm_stream_for(hidden.device) if overlap else None,
                   dW_full)


def cuda_step_fused(kind, hidden, weight, labels=None, target_hidden=None, ignore_index=-100,
                    group=None, chunk_tokens=0, workspace=None, out=None, dH=None, dW=None,
                    shard_dW=False):
    """Data-parallel step over the fused single call (each chunk's logits kept).

    The rank's valid count comes from the library (``slm_count_valid``) before the call, so
    it leaves out exactly the rows the kernels mask: ignore_index, and for CE a label
    outside [0, V) (which the library also flags in its status word).  ``shard_dW`` as for
    ``cuda_step``."""
    from .loss import count_valid, lm_head_loss_fwd_bwd

    N = hidden.shape[0]
    V, d = weight.shape
    dW_full = None
    if shard_dW:
        world = dist.get_world_size(group)
        dW_full = dW if dW is not None else dw_full_buffer(V, d, world, hidden.device)
        dW = dW_full[:V]

    def _count():
        return count_valid(kind, labels, N, V, ignore_index)

    def _fused(scale):
        return lm_head_loss_fwd_bwd(kind, hidden, weight, labels, target_hidden, ignore_index,
                                    grad_scale=scale, chunk_tokens=chunk_tokens,
                                    workspace=workspace, out=out, dH=dH, dW=dW)

    return fused_fwd_bwd(_count, _fused, group, dW_full)
