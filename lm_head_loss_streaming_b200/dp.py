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
    dW: torch.Tensor          # summed over ranks


def fwd_bwd(fwd: Callable[[], Any], bwd: Callable[[Any, torch.Tensor], tuple],
            group=None, comm_stream=None) -> DPResult:
    """Run one data-parallel forward + backward.

    ``fwd()`` returns an object with ``loss_sum`` (float64 [1]) and ``n_valid`` (int64 [1])
    tensors for this rank's rows.  ``bwd(res, n_valid_global)`` returns (dH, dW) for this
    rank's rows with the upstream gradient 1 / n_valid_global on valid rows, or
    (dH, dW, ready): a ``torch.cuda.Event`` recorded once dW is final.  With a ready event
    and a ``comm_stream``, dW is summed on that stream after the event, overlapping
    whatever the backward still runs on the current stream; the current stream waits for
    the sum before this function returns.
    Every rank makes the same collective calls in the same order.
    """
    res = fwd()
    n_valid = res.n_valid.clone()
    dist.all_reduce(n_valid, group=group)
    out = bwd(res, n_valid)
    dH, dW = out[0], out[1]
    ready = out[2] if len(out) > 2 else None
    if ready is not None and comm_stream is not None:
        comm_stream.wait_event(ready)
        with torch.cuda.stream(comm_stream):
            dist.all_reduce(dW, group=group)
    else:
        comm_stream = None
        dist.all_reduce(dW, group=group)
    loss_sum = res.loss_sum.clone()
    dist.all_reduce(loss_sum, group=group)
    if comm_stream is not None:
        torch.cuda.current_stream().wait_stream(comm_stream)
    den = n_valid.clamp_min(1).to(loss_sum.dtype)
    loss_mean = torch.where(n_valid > 0, loss_sum / den, torch.zeros_like(loss_sum))
    return DPResult(loss_mean, loss_sum, n_valid, dH, dW)


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
              overlap=True, reserve_sms=8):
    """Data-parallel step over the CUDA kernels (one rank per GPU, NCCL process group).

    With ``overlap`` the sum of dW over ranks runs on a side stream while the last token
    chunk's dH GEMM runs (on ``reserve_sms`` fewer SMs); the results are the same."""
    from .loss import lm_head_loss_bwd, lm_head_loss_fwd

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

    return fwd_bwd(_fwd, _bwd, group, comm_stream_for(hidden.device) if overlap else None)
