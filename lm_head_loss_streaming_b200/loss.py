"""PyTorch-facing API of the streaming LM-head loss.

PyTorch supplies device memory and the current stream; the loss, its statistics and its
gradients are computed by the kernels of ``libslm.so`` through the C ABI.  The interface
is the one of a regular loss function with a custom backward rule ("Training speculative
decoders: removing the logits and attention bottlenecks", "Backward pass").
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _lib
from .synthetic import IGNORE_INDEX


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _kind_id(kind):
    if isinstance(kind, int):
        return kind
    try:
        return _lib.KIND[kind]
    except KeyError:
        raise ValueError(f"unknown loss kind {kind!r}; expected one of {list(_lib.KIND)}")


def _check_inputs(kind, hidden, weight, labels, target_hidden, grad_tok=None):
    """The kernels see raw pointers and the sizes taken from ``hidden`` and ``weight``: every
    tensor must be on the current CUDA device with the layout and extent those sizes imply,
    or the kernels would read past it.  Raises ValueError before anything is launched."""
    for name, t in (("hidden", hidden), ("weight", weight), ("target_hidden", target_hidden)):
        if t is None:
            continue
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 2:
            raise ValueError(f"{name} must be a contiguous 2-D bf16 CUDA tensor")
    N, d = hidden.shape
    if weight.shape[1] != d:
        raise ValueError(f"weight is {tuple(weight.shape)}; expected [V, {d}]")
    if target_hidden is not None and target_hidden.shape != hidden.shape:
        raise ValueError(f"target_hidden is {tuple(target_hidden.shape)}; expected {(N, d)}")
    if labels is not None:
        if (not labels.is_cuda or labels.dtype != torch.int32 or not labels.is_contiguous()
                or labels.shape != (N,)):
            raise ValueError(f"labels must be a contiguous int32 CUDA tensor of shape ({N},)")
    if grad_tok is not None:
        if (not grad_tok.is_cuda or grad_tok.dtype != torch.float32
                or not grad_tok.is_contiguous() or grad_tok.shape != (N,)):
            raise ValueError(f"grad_tok must be a contiguous float32 CUDA tensor of shape ({N},)")
    dev = torch.cuda.current_device()
    for name, t in (("hidden", hidden), ("weight", weight), ("target_hidden", target_hidden),
                    ("labels", labels), ("grad_tok", grad_tok)):
        if t is not None and t.device.index != dev:
            raise ValueError(f"{name} is on {t.device}, not on the current device cuda:{dev}")
    if kind is None:       # weighted combinations: the library checks what each term needs
        return
    if kind != _lib.SLM_CE and target_hidden is None:
        raise ValueError("distribution losses need target_hidden (H_p)")
    if kind == _lib.SLM_CE and labels is None:
        raise ValueError("ce needs labels")


def _check_out(name, t, shape, dtype):
    """A caller-provided output buffer must have exactly the extent the kernels write."""
    if t is None:
        return
    if (not t.is_cuda or t.dtype != dtype or not t.is_contiguous() or tuple(t.shape) != shape
            or t.device.index != torch.cuda.current_device()):
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {shape} on the "
                         f"current CUDA device")


def _check_fwd_out(out, k, N):
    """Caller-provided forward results must match the sizes the kernels write."""
    _check_out("out.loss_mean", out.loss_mean, (1,), torch.float32)
    _check_out("out.loss_sum", out.loss_sum, (1,), torch.float64)
    _check_out("out.n_valid", out.n_valid, (1,), torch.int64)
    _check_out("out.loss_tok", out.loss_tok, (N,), torch.float32)
    _check_out("out.alpha_tok", out.alpha_tok, (N,), torch.float32)
    _check_out("out.stats", out.stats, (_lib.slm_stats_floats(k), N), torch.float32)


def _check_grads(dH, dW, N, d, V):
    _check_out("dH", dH, (N, d), torch.bfloat16)
    _check_out("dW", dW, (V, d), torch.float32)


def _check_scale(grad_scale):
    if grad_scale is not None:
        _check_out("grad_scale", grad_scale, (1,), torch.float32)


@dataclass
class FwdResult:
    kind: int
    loss_mean: torch.Tensor   # float32 [1]
    loss_sum: torch.Tensor    # float64 [1]
    n_valid: torch.Tensor     # int64 [1]
    loss_tok: torch.Tensor    # float32 [N]
    alpha_tok: torch.Tensor | None
    stats: torch.Tensor       # float32 [k, N]
    workspace: torch.Tensor   # uint8


def workspace_bytes(kind, N, d, V, chunk_tokens=0):
    return _lib.slm_workspace_bytes(_kind_id(kind), N, d, V, chunk_tokens)


def count_valid(kind, labels, N, V, ignore_index=IGNORE_INDEX, out=None):
    """Valid-row count through ``slm_count_valid``: rows whose label is not
    ``ignore_index`` and, for CE, lies in [0, V) -- the rows the kernels do not mask.
    ``labels`` may be None for the distribution kinds (every row counts).  Returns an int64
    [1] CUDA tensor (``out`` if given), filled asynchronously on the current stream."""
    k = _kind_id(kind)
    if labels is not None:
        if (not labels.is_cuda or labels.dtype != torch.int32 or not labels.is_contiguous()
                or labels.shape != (N,) or labels.device.index != torch.cuda.current_device()):
            raise ValueError(f"labels must be a contiguous int32 tensor of shape ({N},) on the "
                             f"current CUDA device")
    if out is None:
        out = torch.empty(1, dtype=torch.int64, device=torch.cuda.current_device())
    else:
        _check_out("out", out, (1,), torch.int64)
    _lib.check(_lib.slm_count_valid(k, _ptr(labels), ignore_index, N, V, _ptr(out), _stream()),
               "slm_count_valid")
    return out


def lm_head_loss_fwd(kind, hidden, weight, labels=None, target_hidden=None,
                     ignore_index=IGNORE_INDEX, workspace=None, chunk_tokens=0,
                     out=None) -> FwdResult:
    """Forward through ``slm_loss_fwd``; returns the per-token loss, the sums and the
    statistics the backward needs.  ``out`` may hold preallocated result buffers."""
    k = _kind_id(kind)
    _check_inputs(k, hidden, weight, labels, target_hidden)
    N, d = hidden.shape
    V = weight.shape[0]
    dev = hidden.device
    ws_need = _lib.slm_workspace_bytes(k, N, d, V, chunk_tokens)
    if workspace is None or workspace.numel() < ws_need:
        workspace = torch.empty(max(ws_need, 256), dtype=torch.uint8, device=dev)
    if out is None:
        nk = _lib.slm_stats_floats(k)
        out = FwdResult(
            k,
            torch.empty(1, dtype=torch.float32, device=dev),
            torch.empty(1, dtype=torch.float64, device=dev),
            torch.empty(1, dtype=torch.int64, device=dev),
            torch.empty(N, dtype=torch.float32, device=dev),
            torch.empty(N, dtype=torch.float32, device=dev) if k in _lib.ALPHA_KINDS else None,
            torch.empty(nk, N, dtype=torch.float32, device=dev),
            workspace)
    else:
        _check_fwd_out(out, k, N)
        out.workspace = workspace
    st = _lib.slm_loss_fwd(k, _ptr(hidden), _ptr(target_hidden), _ptr(weight), _ptr(labels),
                           ignore_index, N, d, V, _ptr(out.loss_tok), _ptr(out.alpha_tok),
                           _ptr(out.loss_sum), _ptr(out.n_valid), _ptr(out.loss_mean),
                           _ptr(out.stats), _ptr(workspace), workspace.numel(), _stream())
    _lib.check(st, "slm_loss_fwd")
    return out


def lm_head_loss_bwd(fwd: FwdResult, hidden, weight, labels=None, target_hidden=None,
                     ignore_index=IGNORE_INDEX, grad_tok=None, grad_scale=None,
                     normalize=True, dH=None, dW=None, accumulate_dW=False, chunk_tokens=0,
                     dw_ready=None, reserve_sms=0):
    """Backward through ``slm_loss_bwd``.  With ``normalize`` the upstream gradient is
    divided by the forward's valid-row count (gradient of the mean loss).

    ``dw_ready`` (a ``torch.cuda.Event``) or ``reserve_sms`` > 0 selects
    ``slm_loss_bwd_overlap``: the event is recorded on the current stream as soon as dW is
    final, before the last chunk's dH GEMM, which then leaves ``reserve_sms`` SMs idle, so
    that a reduction of dW on another stream can overlap it.  The results are the same.
    Returns (dH bf16 [N, d], dW fp32 [V, d])."""
    k = fwd.kind
    _check_inputs(k, hidden, weight, labels, target_hidden, grad_tok)
    N, d = hidden.shape
    V = weight.shape[0]
    dev = hidden.device
    if tuple(fwd.stats.shape) != (_lib.slm_stats_floats(k), N):
        raise ValueError("fwd does not come from a forward over these hidden states")
    _check_grads(dH, dW, N, d, V)
    _check_scale(grad_scale)
    if dH is None:
        dH = torch.empty(N, d, dtype=torch.bfloat16, device=dev)
    if dW is None:
        dW = torch.empty(V, d, dtype=torch.float32, device=dev)
    ws_need = _lib.slm_workspace_bytes(k, N, d, V, chunk_tokens)
    ws = fwd.workspace
    if ws.numel() < ws_need:
        ws = torch.empty(ws_need, dtype=torch.uint8, device=dev)
    args = (k, _ptr(hidden), _ptr(target_hidden), _ptr(weight), _ptr(labels), ignore_index,
            N, d, V, _ptr(grad_tok), _ptr(grad_scale),
            _ptr(fwd.n_valid) if normalize else None, _ptr(fwd.stats), _ptr(dH), _ptr(dW),
            1 if accumulate_dW else 0, chunk_tokens, _ptr(ws), ws.numel(), _stream())
    if dw_ready is None and not reserve_sms:
        _lib.check(_lib.slm_loss_bwd(*args), "slm_loss_bwd")
        return dH, dW
    handle = None
    if dw_ready is not None:
        # torch creates the CUDA event on its first record; the library records it again
        # at the point where dW is final.
        dw_ready.record(torch.cuda.current_stream())
        handle = dw_ready.cuda_event
    _lib.check(_lib.slm_loss_bwd_overlap(*args, handle, reserve_sms), "slm_loss_bwd_overlap")
    return dH, dW


@dataclass
class ComboResult:
    weights: dict
    loss_mean: torch.Tensor      # float32 [1], the weighted combination's mean
    loss_sum: torch.Tensor       # float64 [1]
    n_valid: torch.Tensor        # int64 [1]
    loss_tok: torch.Tensor       # float32 [N], sum_k w_k loss_k
    term_loss_tok: torch.Tensor  # float32 [SLM_NUM_KINDS, N], before weighting
    term_loss_sum: torch.Tensor  # float64 [SLM_NUM_KINDS]
    stats: torch.Tensor          # float32 [SLM_COMBO_STATS, N]
    workspace: torch.Tensor

    def term_means(self):
        """{kind: mean loss of that term, before weighting} (the per-term log values)."""
        nv = max(int(self.n_valid.item()), 1)
        sums = self.term_loss_sum.cpu()
        return {k: float(sums[_lib.KIND[k]]) / nv for k in self.weights}


def lm_head_loss_combo_fwd(weights, hidden, weight, labels=None, target_hidden=None,
                           ignore_index=IGNORE_INDEX, chunk_tokens=0) -> ComboResult:
    """Forward of a weighted combination {kind: weight} through ``slm_combo_fwd``."""
    for k in weights:
        _kind_id(k)
    _check_inputs(None, hidden, weight, labels, target_hidden)
    N, d = hidden.shape
    V = weight.shape[0]
    dev = hidden.device
    ws = torch.empty(max(_lib.slm_combo_workspace_bytes(N, d, V, chunk_tokens), 256),
                     dtype=torch.uint8, device=dev)
    r = ComboResult(dict(weights), torch.empty(1, device=dev),
                    torch.empty(1, dtype=torch.float64, device=dev),
                    torch.empty(1, dtype=torch.int64, device=dev), torch.empty(N, device=dev),
                    torch.empty(_lib.SLM_NUM_KINDS, N, device=dev),
                    torch.empty(_lib.SLM_NUM_KINDS, dtype=torch.float64, device=dev),
                    torch.empty(_lib.SLM_COMBO_STATS, N, device=dev), ws)
    st = _lib.slm_combo_fwd(weights, _ptr(hidden), _ptr(target_hidden), _ptr(weight),
                            _ptr(labels), ignore_index, N, d, V, _ptr(r.loss_tok),
                            _ptr(r.term_loss_tok), _ptr(r.loss_sum), _ptr(r.term_loss_sum),
                            _ptr(r.n_valid), _ptr(r.loss_mean), _ptr(r.stats), _ptr(ws),
                            ws.numel(), _stream())
    _lib.check(st, "slm_combo_fwd")
    return r


def lm_head_loss_combo_bwd(fwd: ComboResult, hidden, weight, labels=None, target_hidden=None,
                           ignore_index=IGNORE_INDEX, grad_tok=None, grad_scale=None,
                           normalize=True, dH=None, dW=None, accumulate_dW=False,
                           chunk_tokens=0):
    """Backward of a weighted combination through ``slm_combo_bwd``."""
    _check_inputs(None, hidden, weight, labels, target_hidden, grad_tok)
    N, d = hidden.shape
    V = weight.shape[0]
    dev = hidden.device
    if tuple(fwd.stats.shape) != (_lib.SLM_COMBO_STATS, N):
        raise ValueError("fwd does not come from a forward over these hidden states")
    _check_grads(dH, dW, N, d, V)
    _check_scale(grad_scale)
    if dH is None:
        dH = torch.empty(N, d, dtype=torch.bfloat16, device=dev)
    if dW is None:
        dW = torch.empty(V, d, dtype=torch.float32, device=dev)
    ws = fwd.workspace
    need = _lib.slm_combo_workspace_bytes(N, d, V, chunk_tokens)
    if ws.numel() < need:
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    st = _lib.slm_combo_bwd(fwd.weights, _ptr(hidden), _ptr(target_hidden), _ptr(weight),
                            _ptr(labels), ignore_index, N, d, V, _ptr(grad_tok),
                            _ptr(grad_scale), _ptr(fwd.n_valid) if normalize else None,
                            _ptr(fwd.stats), _ptr(dH), _ptr(dW), 1 if accumulate_dW else 0,
                            chunk_tokens, _ptr(ws), ws.numel(), _stream())
    _lib.check(st, "slm_combo_bwd")
    return dH, dW


def lm_head_loss_fwd_bwd(kind, hidden, weight, labels=None, target_hidden=None,
                        ignore_index=IGNORE_INDEX, grad_tok=None, grad_scale=None,
                        chunk_tokens=0, workspace=None, out=None, dH=None, dW=None,
                        accumulate_dW=False):
    """Forward and backward in one call through ``slm_loss_fwd_bwd`` (the chunk's logits are
    kept instead of recomputed).  Returns (FwdResult, dH, dW); the gradient is that of the
    mean loss, scaled by grad_tok / grad_scale when given."""
    k = _kind_id(kind)
    _check_inputs(k, hidden, weight, labels, target_hidden, grad_tok)
    N, d = hidden.shape
    V = weight.shape[0]
    dev = hidden.device
    _check_grads(dH, dW, N, d, V)
    _check_scale(grad_scale)
    need = max(_lib.slm_fused_workspace_bytes(k, N, d, V, chunk_tokens), 256)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if out is None:
        out = FwdResult(
            k, torch.empty(1, dtype=torch.float32, device=dev),
            torch.empty(1, dtype=torch.float64, device=dev),
            torch.empty(1, dtype=torch.int64, device=dev),
            torch.empty(N, dtype=torch.float32, device=dev),
            torch.empty(N, dtype=torch.float32, device=dev) if k in _lib.ALPHA_KINDS else None,
            torch.empty(_lib.slm_stats_floats(k), N, dtype=torch.float32, device=dev),
            workspace)
    else:
        _check_fwd_out(out, k, N)
        out.workspace = workspace
    if dH is None:
        dH = torch.empty(N, d, dtype=torch.bfloat16, device=dev)
    if dW is None:
        dW = torch.empty(V, d, dtype=torch.float32, device=dev)
    st = _lib.slm_loss_fwd_bwd(k, _ptr(hidden), _ptr(target_hidden), _ptr(weight),
                               _ptr(labels), ignore_index, N, d, V, _ptr(grad_tok),
                               _ptr(grad_scale), _ptr(out.loss_tok), _ptr(out.alpha_tok),
                               _ptr(out.loss_sum), _ptr(out.n_valid), _ptr(out.loss_mean),
                               _ptr(out.stats), _ptr(dH), _ptr(dW), 1 if accumulate_dW else 0,
                               chunk_tokens, _ptr(workspace), workspace.numel(), _stream())
    _lib.check(st, "slm_loss_fwd_bwd")
    return out, dH, dW


def chunk_for_budget(kind, N, d, V, budget_bytes, fused=False):
    """The largest token chunk whose workspace fits in ``budget_bytes`` (0 if none): set the
    budget to the next memory peak of the training step so the loss path stays below it."""
    return int(_lib.slm_chunk_for_budget(_kind_id(kind), N, d, V, budget_bytes, fused))


def align_labels(tokens, shift, loss_mask=None, seq_ids=None, ignore_index=IGNORE_INDEX):
    """Labels of a draft head that predicts ``shift`` tokens ahead, aligned before chunking
    (through ``slm_align_labels``).  tokens int32 [B, S] (CUDA); loss_mask bool/uint8 [B, S]
    or None; seq_ids int32 [B, S] or None.  Returns int32 [B * S]."""
    if tokens.dtype != torch.int32 or not tokens.is_cuda or tokens.dim() != 2:
        raise ValueError("tokens must be a 2-D int32 CUDA tensor")
    B, S = tokens.shape
    for name, t in (("loss_mask", loss_mask), ("seq_ids", seq_ids)):
        if t is not None and (not t.is_cuda or t.device != tokens.device
                              or tuple(t.shape) != (B, S)):
            raise ValueError(f"{name} must be a CUDA tensor of shape {(B, S)} on {tokens.device}")
    if tokens.device.index != torch.cuda.current_device():
        raise ValueError(f"tokens is on {tokens.device}, not on the current CUDA device")
    tokens = tokens.contiguous()
    mask = None if loss_mask is None else loss_mask.to(torch.uint8).contiguous()
    seq = None if seq_ids is None else seq_ids.to(torch.int32).contiguous()
    out = torch.empty(B * S, dtype=torch.int32, device=tokens.device)
    st = _lib.slm_align_labels(_ptr(tokens), _ptr(mask), _ptr(seq), B, S, shift, ignore_index,
                               _ptr(out), _stream())
    _lib.check(st, "slm_align_labels")
    return out


def target_flatness(target_hidden, weight):
    """Per-token flatness cos(p, uniform) of p = softmax(target_hidden weight^T) through
    ``slm_target_flatness``.  Returns float32 [N]."""
    _check_inputs(_lib.SLM_KL, target_hidden, weight, None, target_hidden)
    N, d = target_hidden.shape
    V = weight.shape[0]
    dev = target_hidden.device
    ws = torch.empty(max(_lib.slm_flatness_workspace_bytes(N, d, V), 256), dtype=torch.uint8,
                     device=dev)
    out = torch.empty(N, dtype=torch.float32, device=dev)
    st = _lib.slm_target_flatness(_ptr(target_hidden), _ptr(weight), N, d, V, _ptr(out),
                                  _ptr(ws), ws.numel(), _stream())
    _lib.check(st, "slm_target_flatness")
    return out


def device_status(fwd: FwdResult):
    """Synchronise and return the device status of the last call on this workspace."""
    return _lib.slm_device_status(_ptr(fwd.workspace), _stream())


class StreamingLMHeadLoss(torch.autograd.Function):
    """Mean streaming LM-head loss with a custom backward: gradients for the draft hidden
    states and the LM-head weight; the target hidden states are detached."""

    @staticmethod
    def forward(ctx, hidden, weight, labels, target_hidden, kind, ignore_index, chunk_tokens):
        fwd = lm_head_loss_fwd(kind, hidden, weight, labels, target_hidden, ignore_index,
                               chunk_tokens=chunk_tokens)
        ctx.save_for_backward(hidden, weight, labels, target_hidden)
        ctx.fwd = fwd
        ctx.ignore_index = ignore_index
        ctx.chunk_tokens = chunk_tokens
        return fwd.loss_mean.reshape(())

    @staticmethod
    def backward(ctx, grad_out):
        hidden, weight, labels, target_hidden = ctx.saved_tensors
        g = grad_out.reshape(1).to(torch.float32).contiguous()
        dH, dW = lm_head_loss_bwd(ctx.fwd, hidden, weight, labels, target_hidden,
                                  ctx.ignore_index, grad_scale=g,
                                  chunk_tokens=ctx.chunk_tokens)
        return dH, dW.to(weight.dtype), None, None, None, None, None


class StreamingLMHeadLossFused(torch.autograd.Function):
    """The same loss through the fused single call (``slm_loss_fwd_bwd``): the gradients
    of the mean are computed in the forward, with each chunk's logits kept instead of
    recomputed, and the backward only scales them by the upstream gradient."""

    @staticmethod
    def forward(ctx, hidden, weight, labels, target_hidden, kind, ignore_index, chunk_tokens):
        fwd, dH, dW = lm_head_loss_fwd_bwd(kind, hidden, weight, labels, target_hidden,
                                           ignore_index, chunk_tokens=chunk_tokens)
        ctx.dH, ctx.dW, ctx.wdtype = dH, dW, weight.dtype
        return fwd.loss_mean.reshape(())

    @staticmethod
    def backward(ctx, grad_out):
        dH, dW = ctx.dH, ctx.dW
        ctx.dH = ctx.dW = None
        g = grad_out.to(torch.float32)
        return ((dH.float() * g).to(dH.dtype), (dW * g).to(ctx.wdtype),
                None, None, None, None, None)


def streaming_lm_head_loss(hidden, weight, labels=None, target_hidden=None, kind="ce",
                           ignore_index=IGNORE_INDEX, chunk_tokens=0, fused=False):
    """Mean loss over valid rows; differentiable w.r.t. ``hidden`` and ``weight``.

    ``fused=False`` recomputes each chunk's logits in the backward (memory bounded by one
    bf16 chunk of logit gradients).  ``fused=True`` computes the gradients in the forward
    with the fused single call (each chunk's fp32 logits kept, 1.2-1.7x faster, a larger
    workspace) and holds them until the backward."""
    fn = StreamingLMHeadLossFused if fused else StreamingLMHeadLoss
    return fn.apply(hidden, weight, labels, target_hidden, _kind_id(kind), ignore_index,
                    chunk_tokens)
