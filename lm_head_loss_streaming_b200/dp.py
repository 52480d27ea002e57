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


def fused_fwd_bwd(count: Callable[[], torch.Tensor],
                  fused: Callable[[torch.Tensor], tuple], group=None) -> DPResult:
    """One data-parallel step through a single-call forward + backward.

    The single call (``slm_loss_fwd_bwd``) forms the gradient of this rank's mean loss, i.e.
    it divides by the rank's own valid count, scaled by ``grad_scale``.  So the counts are
    summed first: ``count()`` returns this rank's valid-row count (int64 [1]), and
    ``fused(scale)`` is called with scale = n_local / n_global (float32 [1]), which turns the
    local mean's gradient into the global mean's.  It returns (res, dH, dW) with
    ``res.loss_sum``.  dW and the loss sum are then summed across ranks, as in ``fwd_bwd``.
    """
    n_local = count().reshape(1).to(torch.int64)
    n_valid = n_local.clone()
    dist.all_reduce(n_valid, group=group)
    scale = (n_local.to(torch.float64) / n_valid.clamp_min(1).to(torch.float64)).to(torch.float32)
    res, dH, dW = fused(scale)
    dist.all_reduce(dW, group=group)
    loss_sum = res.loss_sum.clone()
    dist.all_reduce(loss_sum, group=group)
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


def cuda_step_fused(kind, hidden, weight, labels=None, target_hidden=None, ignore_index=-100,
                    group=None, chunk_tokens=0, workspace=None, out=None, dH=None, dW=None):
    """Data-parallel step over the fused single call (each chunk's logits kept).

    The rank's valid count is taken from its labels (rows whose label is not ignore_index;
    every row without labels) before the call.  A CE label outside [0, V) is masked by the
    library and flagged in its status word, but counted here: such a batch is invalid."""
    from .loss import lm_head_loss_fwd_bwd

    def _count():
        if labels is None:
            return torch.full((1,), hidden.shape[0], dtype=torch.int64, device=hidden.device)
        return (labels != ignore_index).sum().reshape(1)

    def _fused(scale):
        return lm_head_loss_fwd_bwd(kind, hidden, weight, labels, target_hidden, ignore_index,
                                    grad_scale=scale, chunk_tokens=chunk_tokens,
                                    workspace=workspace, out=out, dH=dH, dW=dW)

    return fused_fwd_bwd(_count, _fused, group)
