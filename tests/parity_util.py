"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and the
float64 oracle on the same seeded inputs, and compare within the stated tolerances.

Tolerances (bf16 inputs, fp32 accumulation; the oracle is float64):
  * loss:      |L_gpu - L_ref| <= 2e-3 |L_ref| on the mean loss, and per token
               max_n |l_gpu - l_ref| <= 2e-3 * max(max_n |l_ref|, 1e-2)
  * gradients: max |dX_gpu - dX_ref| / max |dX_ref| <= 1e-2 for X in {H_q, W}
"""

from __future__ import annotations

import numpy as np
import torch

import oracle

LOSS_RTOL = 2e-3
GRAD_RTOL = 1e-2

# Headroom record: every comparison below appends (test, what, error / tolerance) so that a
# run can report how much of each tolerance was used (tests/conftest.py prints the worst per
# test, and writes them all to $SLM_MARGINS_OUT when set).  Near-tie comparisons also record
# how many entries fell inside the band and the largest slack they used, as a fraction of
# the tolerance.
MARGINS = []
CURRENT_TEST = [""]


def _record(what, frac, **extra):
    MARGINS.append(dict(test=CURRENT_TEST[0], what=what, frac_of_tol=float(frac), **extra))


def _np64(t):
    return t.detach().to("cpu").double().numpy()


def gpu_fwd_bwd(inp, kind=None, chunk_tokens=0, grad_tok=None, normalize=True,
                accumulate_dW=None, fused=False):
    """Forward and backward through the C ABI on cuda:0 (two calls, or the fused single
    call).  Returns numpy results plus the device status after each call."""
    from lm_head_loss_streaming_b200 import _lib
    from lm_head_loss_streaming_b200.loss import (device_status, lm_head_loss_bwd,
                                                  lm_head_loss_fwd, lm_head_loss_fwd_bwd)

    kind = kind or inp.kind
    dev = torch.device("cuda", 0)
    Hq = inp.Hq.to(dev)
    W = inp.W.to(dev)
    Hp = inp.Hp.to(dev) if (kind != "ce" and inp.Hp is not None) else None
    labels = inp.labels.to(dev) if inp.labels is not None else None
    gt = None
    if grad_tok is not None:
        gt = torch.as_tensor(grad_tok, dtype=torch.float32).to(dev).contiguous()
    dW = None
    if accumulate_dW is not None:
        dW = torch.as_tensor(accumulate_dW, dtype=torch.float32).to(dev).contiguous()
    if fused:
        assert normalize, "the fused call always divides by the valid count"
        fwd, dH, dW = lm_head_loss_fwd_bwd(kind, Hq, W, labels, Hp, inp.ignore_index,
                                           grad_tok=gt, chunk_tokens=chunk_tokens, dW=dW,
                                           accumulate_dW=accumulate_dW is not None)
        st_fwd = st_bwd = device_status(fwd)
    else:
        fwd = lm_head_loss_fwd(kind, Hq, W, labels, Hp, inp.ignore_index,
                               chunk_tokens=chunk_tokens)
        st_fwd = device_status(fwd)
        dH, dW = lm_head_loss_bwd(fwd, Hq, W, labels, Hp, inp.ignore_index, grad_tok=gt,
                                  normalize=normalize, chunk_tokens=chunk_tokens, dW=dW,
                                  accumulate_dW=accumulate_dW is not None)
        st_bwd = device_status(fwd)
    torch.cuda.synchronize()
    out = dict(
        loss_tok=_np64(fwd.loss_tok), loss_mean=float(fwd.loss_mean.item()),
        loss_sum=float(fwd.loss_sum.item()), n_valid=int(fwd.n_valid.item()),
        stats=_np64(fwd.stats), stats32=fwd.stats.cpu().numpy(),
        alpha=None if fwd.alpha_tok is None else _np64(fwd.alpha_tok),
        dH=_np64(dH), dW=_np64(dW), st_fwd=st_fwd, st_bwd=st_bwd,
    )
    assert _lib.SLM_OK == 0
    return out


def oracle_fwd_bwd(inp, kind=None, rows=None, grad_tok=None, chunk_size=512):
    """The oracle on the same inputs (optionally on a subset of rows)."""
    kind = kind or inp.kind
    sl = slice(None) if rows is None else rows
    Hq = inp.Hq[sl]
    Hp = None if kind == "ce" else inp.Hp[sl]
    lab = None if inp.labels is None else inp.labels[sl]
    f = oracle.forward(kind, Hq, inp.W, lab, Hp, inp.ignore_index, chunk_size)
    dH, dW = oracle.backward(kind, Hq, inp.W, lab, Hp, grad_tok, inp.ignore_index,
                             chunk_size)
    f["dH"] = dH
    f["dW"] = dW
    return f


def assert_loss_close(gpu_tok, ref_tok, gpu_mean=None, ref_mean=None, what=""):
    gpu_tok = np.asarray(gpu_tok)
    ref_tok = np.asarray(ref_tok)
    assert np.isfinite(gpu_tok).all(), f"{what}: non-finite per-token loss"
    scale = max(float(np.abs(ref_tok).max()) if ref_tok.size else 0.0, 1e-2)
    err = float(np.abs(gpu_tok - ref_tok).max()) if ref_tok.size else 0.0
    _record(f"{what} loss_tok", err / (LOSS_RTOL * scale))
    assert err <= LOSS_RTOL * scale, f"{what}: per-token loss err {err:.3e} > {LOSS_RTOL}*{scale:.3e}"
    if ref_mean is not None:
        tol = LOSS_RTOL * max(abs(ref_mean), 1e-2)
        _record(f"{what} loss_mean", abs(gpu_mean - ref_mean) / tol)
        assert abs(gpu_mean - ref_mean) <= tol, f"{what}: mean {gpu_mean} vs {ref_mean}"


# Relative band |q_v - p_v| <= TIE_BAND * max(q_v, p_v) inside which the GPU's fp32
# decision m_v = [q_v < p_v] may legitimately differ from the oracle's float64 one: the
# GPU's q and p each carry a relative error of a few 1e-6 (fp32 logits accumulated over d
# products, ex2.approx, fp32 sums).
TIE_BAND = 1e-5


def tie_slack(inp, kind, rows=None, grad_tok=None):
    """Elementwise bound on how far dH (rows) and dW may move if every near-tie of the
    indicator m_v = [q_v < p_v] is decided the other way.  Zero for kinds without it.

    Flipping m_j of row n changes dz_nj by c_n q_nj and, through S_n, every dz_nk by
    c_n q_nk q_nj, where c_n = g_n (tv), g_n / alpha_n (nla), g_n (1 - lambda_n) (lk_hybrid).
    """
    if kind not in ("tv", "nla", "lk_hybrid"):
        return 0.0, 0.0
    sl = slice(None) if rows is None else rows
    Hq = inp.Hq[sl].double().numpy()
    Hp = inp.Hp[sl].double().numpy()
    W = inp.W.double().numpy()
    q = np.exp(oracle.log_softmax(oracle.logits(Hq, W)))
    p = np.exp(oracle.log_softmax(oracle.logits(Hp, W)))
    n = Hq.shape[0]
    valid = np.ones(n, dtype=bool)
    if inp.labels is not None:
        valid = inp.labels[sl].numpy() != inp.ignore_index
    if grad_tok is None:
        g = np.full(n, 1.0 / max(int(valid.sum()), 1))
    else:
        g = np.asarray(grad_tok, dtype=np.float64)
    g = np.where(valid, np.abs(g), 0.0)
    alpha = np.minimum(p, q).sum(axis=1)
    if kind == "tv":
        c = g
    elif kind == "nla":
        c = g / alpha
    else:
        c = g * (1.0 - np.exp(-3.0 * alpha))
    near = np.abs(q - p) <= TIE_BAND * np.maximum(q, p)
    near &= valid[:, None] & (g[:, None] != 0.0)
    tie_slack.last_count = int(near.sum())
    tie_slack.last_entries = int(near.size)
    # Rows whose gradient a flip changes to first order: token rows with a near-tie (dH) and
    # vocabulary rows with a near-tie in some token row (dW).
    tie_slack.last_rows = near.any(axis=1)
    tie_slack.last_cols = near.any(axis=0)
    qn = np.where(near, q, 0.0)
    qsum = qn.sum(axis=1)
    aW, aH = np.abs(W), np.abs(Hq)
    slack_h = c[:, None] * (qn @ aW + qsum[:, None] * (q @ aW))
    slack_w = (c[:, None] * qn).T @ aH + ((c * qsum)[:, None] * q).T @ aH
    return slack_h, slack_w


def assert_grad_close(g, r, what="", slack=0.0):
    g = np.asarray(g)
    r = np.asarray(r)
    assert np.isfinite(g).all(), f"{what}: non-finite gradient"
    den = float(np.abs(r).max()) if r.size else 0.0
    diff = np.abs(g - r)
    err = float(np.maximum(diff - slack, 0.0).max()) if r.size else 0.0
    if den == 0.0:
        _record(f"{what} (zero)", err / 1e-6)
        assert err <= 1e-6, f"{what}: expected zero gradient, max {err:.3e}"
        return
    extra = {}
    if not np.isscalar(slack) or slack != 0.0:
        # How much the near-tie allowance was actually drawn on, and how many entries of
        # the last tie_slack call fell inside the band.
        used = float(np.minimum(diff, slack).max()) if r.size else 0.0
        extra = dict(slack_used_frac=used / (GRAD_RTOL * den),
                     raw_frac=float(diff.max()) / (GRAD_RTOL * den),
                     near_ties=getattr(tie_slack, "last_count", None),
                     entries=getattr(tie_slack, "last_entries", None))
        # The raw error (no slack) on the rows no near-tie touches to first order.
        for mask in (getattr(tie_slack, "last_cols", None), getattr(tie_slack, "last_rows", None)):
            if mask is not None and g.ndim == 2 and len(mask) == g.shape[0]:
                off = ~mask
                extra["raw_frac_off_tie_rows"] = (
                    float(diff[off].max()) / (GRAD_RTOL * den) if off.any() else 0.0)
                extra["tie_rows"] = int(mask.sum())
                break
    _record(f"{what} grad", err / den / GRAD_RTOL, **extra)
    assert err / den <= GRAD_RTOL, f"{what}: grad rel err {err / den:.3e} > {GRAD_RTOL}"


# Band inside which the GPU's fp32 argmax of the target logits may pick another column
# than the float64 one: the GPU's z_p carry an absolute error of a few 1e-6 (fp32
# accumulation over d products), far below this band.
ARGMAX_BAND = 1e-4


def argmax_targets_valid(inp, y_gpu, rows=None):
    """Check every GPU target is an argmax of the oracle's float64 target logits up to
    ARGMAX_BAND (masked rows carry ignore_index).  Returns the fraction of rows where the
    GPU picked another column than the float64 argmax (a near-tie)."""
    sl = slice(None) if rows is None else rows
    zp = oracle.logits(inp.Hp[sl], inp.W)
    y_ref = oracle.argmax_target(zp)
    y = np.asarray(y_gpu, dtype=np.int64)
    valid = np.ones(len(y), dtype=bool)
    if inp.labels is not None:
        valid = inp.labels[sl].numpy() != inp.ignore_index
    assert (y[~valid] == inp.ignore_index).all()
    yv = y[valid]
    assert ((yv >= 0) & (yv < inp.V)).all()
    top = zp[valid].max(axis=1)
    picked = zp[valid][np.arange(valid.sum()), yv]
    assert (top - picked <= ARGMAX_BAND * np.maximum(1.0, np.abs(top))).all()
    return float((yv != y_ref[valid]).mean()) if valid.any() else 0.0


def with_labels(inp, y):
    """The same inputs as a hard-label CE problem with labels y."""
    from lm_head_loss_streaming_b200 import synthetic
    return synthetic.Inputs("ce", inp.Hq, inp.W, torch.as_tensor(np.asarray(y, np.int32)), None,
                            inp.ignore_index, dict(inp.meta))
