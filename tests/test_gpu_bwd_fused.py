"""The persistent fused backward ("Backward pass": per token chunk, recompute the logits,
form their gradient, produce the chunk's dH and accumulate dW), one launch per chunk.

slm_set_backward_mode(1) (the default) runs each chunk as one launch whose CTA pairs claim
logits-gradient units, then dH and dW units, a dH or dW unit waiting for the logits-gradient
units it reads; mode 0 runs three launches per chunk.  The arithmetic of every tile is the
same in both, so dH and dW must agree bit for bit, for every kind, ragged shapes, several
chunks, accumulation, weighted combinations and the fused single call.  Parity against the
oracle runs in the default mode throughout the other test files.  The failure path: a
withheld accumulator release makes a bounded wait run out, the call reports
SLM_ERR_TIMEOUT and the context stays usable.
"""

import numpy as np
import pytest
import torch

from lm_head_loss_streaming_b200 import _lib, synthetic
from lm_head_loss_streaming_b200.loss import (lm_head_loss_bwd, lm_head_loss_fwd,
                                              lm_head_loss_fwd_bwd, lm_head_loss_combo_bwd,
                                              lm_head_loss_combo_fwd)
from parity_util import assert_grad_close, assert_loss_close, oracle_fwd_bwd, tie_slack

pytestmark = pytest.mark.gpu


def _dev(inp):
    dev = torch.device("cuda", 0)
    return (inp.Hq.to(dev), inp.W.to(dev), None if inp.Hp is None else inp.Hp.to(dev),
            None if inp.labels is None else inp.labels.to(dev))


class _Mode:
    def __init__(self, mode):
        self.mode = mode

    def __enter__(self):
        self.prev = _lib.slm_set_backward_mode(self.mode)
        assert self.prev in (0, 1)

    def __exit__(self, *exc):
        _lib.slm_set_backward_mode(self.prev)


def _bwd_both(kind, inp, chunk, accumulate=False, grad_tok=None):
    Hq, W, Hp, lab = _dev(inp)
    f = lm_head_loss_fwd(kind, Hq, W, lab, Hp, inp.ignore_index, chunk_tokens=chunk)
    base = torch.randn(W.shape, device=W.device, generator=torch.Generator(
        device=W.device).manual_seed(5)) if accumulate else None
    out = []
    for mode in (0, 1):
        dW = base.clone() if accumulate else None
        with _Mode(mode):
            dH, dW = lm_head_loss_bwd(f, Hq, W, lab, Hp, inp.ignore_index, chunk_tokens=chunk,
                                      dW=dW, accumulate_dW=accumulate, grad_tok=grad_tok)
        torch.cuda.synchronize()
        st = _lib.slm_device_status(f.workspace.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == 0, _lib.status_string(st)
        out.append((dH.clone(), dW.clone()))
    return out


@pytest.mark.parametrize("kind", ["ce", "kl_div", "tv", "nla", "lk_hybrid", "rkl", "jsd",
                                  "ce_argmax_p"])
def test_fused_backward_is_bitwise_the_three_launch_backward(kind):
    # Ragged in every dimension: N, V and d off every tile; three chunks, the last short.
    inp = synthetic.make(kind, 700, 264, 3001, w_std=0.05, ignore_frac=0.1, seed=91,
                         with_labels=kind != "ce_argmax_p")
    (h0, w0), (h1, w1) = _bwd_both(kind, inp, chunk=256)
    assert torch.equal(h0, h1)
    assert torch.equal(w0, w1)


@pytest.mark.parametrize("kind,shape,chunk", [("ce", (1, 8, 50), 0), ("kl_div", (129, 64, 257), 0),
                                              ("tv", (300, 16, 4100), 128),
                                              ("ce", (2000, 128, 700), 0),
                                              ("jsd", (513, 520, 1000), 384),
                                              ("kl_div", (2600, 520, 3500), 2304),
                                              ("ce", (2600, 136, 2100), 2560)])
def test_fused_backward_edge_shapes(kind, shape, chunk):
    """One row, fewer units than pairs, one vocabulary tile, a d of two N tiles, chunks that
    are not multiples of 256, and dH / dW unit grids whose last raster group of M tiles is
    short (9 and 10 chunk M tiles, 14 and 9 vocabulary M tiles, in groups of 8)."""
    inp = synthetic.make(kind, *shape, w_std=0.1, ignore_frac=0.1 if shape[0] > 1 else 0.0,
                         seed=92)
    (h0, w0), (h1, w1) = _bwd_both(kind, inp, chunk=chunk)
    assert torch.equal(h0, h1) and torch.equal(w0, w1)


def test_fused_backward_accumulates_and_takes_token_weights():
    inp = synthetic.make("kl_div", 600, 128, 2000, w_std=0.05, seed=93)
    g = torch.rand(inp.N, generator=torch.Generator().manual_seed(3)).to("cuda:0")
    (h0, w0), (h1, w1) = _bwd_both("kl_div", inp, chunk=256, accumulate=True, grad_tok=g)
    assert torch.equal(h0, h1) and torch.equal(w0, w1)


def test_fused_backward_matches_oracle():
    inp = synthetic.make("lk_hybrid", 700, 128, 3000, w_std=0.05, ignore_frac=0.05, seed=94)
    Hq, W, Hp, lab = _dev(inp)
    with _Mode(1):
        f = lm_head_loss_fwd("lk_hybrid", Hq, W, lab, Hp, inp.ignore_index)
        dH, dW = lm_head_loss_bwd(f, Hq, W, lab, Hp, inp.ignore_index, chunk_tokens=256)
    r = oracle_fwd_bwd(inp, "lk_hybrid")
    assert_loss_close(f.loss_tok.double().cpu().numpy(), r["loss_tok"], f.loss_mean.item(),
                      r["loss"], "fused bwd lk_hybrid")
    sh, sw = tie_slack(inp, "lk_hybrid")
    assert_grad_close(dH.double().cpu().numpy(), r["dH"], "fused bwd lk_hybrid dH", sh)
    assert_grad_close(dW.double().cpu().numpy(), r["dW"], "fused bwd lk_hybrid dW", sw)


def test_fused_backward_weighted_combination_and_single_call():
    inp = synthetic.make("kl_div", 700, 136, 3001, w_std=0.05, ignore_frac=0.1, seed=95,
                         with_labels=True)
    Hq, W, Hp, lab = _dev(inp)
    weights = {"ce": 0.1, "tv": 0.9, "kl_div": 0.5}
    res = lm_head_loss_combo_fwd(weights, Hq, W, lab, Hp, inp.ignore_index, chunk_tokens=256)
    outs = []
    for mode in (0, 1):
        with _Mode(mode):
            outs.append(lm_head_loss_combo_bwd(res, Hq, W, lab, Hp, inp.ignore_index,
                                               chunk_tokens=256))
    torch.cuda.synchronize()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    singles = []
    for mode in (0, 1):
        with _Mode(mode):
            _, dH, dW = lm_head_loss_fwd_bwd("tv", Hq, W, lab, Hp, inp.ignore_index,
                                             chunk_tokens=256)
        torch.cuda.synchronize()
        singles.append((dH.clone(), dW.clone()))
    assert torch.equal(singles[0][0], singles[1][0]) and torch.equal(singles[0][1], singles[1][1])


def test_fused_backward_wait_runs_out_and_context_survives():
    from lm_head_loss_streaming_b200.loss import device_status
    inp = synthetic.make("kl_div", 512, 128, 3000, w_std=0.05, seed=96)
    Hq, W, Hp, lab = _dev(inp)
    f = lm_head_loss_fwd("kl_div", Hq, W, lab, Hp, inp.ignore_index)
    assert device_status(f) == 0
    with _Mode(1):
        assert _lib.slm_debug_set(1, 100_000_000) == 0   # ~0.05-0.1 s per wait
        try:
            lm_head_loss_bwd(f, Hq, W, lab, Hp, inp.ignore_index)
            st = device_status(f)
        finally:
            assert _lib.slm_debug_set(0, 0) == 0
    assert st == 7, _lib.status_string(st)   # SLM_ERR_TIMEOUT
    # The context is usable and the next backward is right.
    (h0, w0), (h1, w1) = _bwd_both("kl_div", inp, chunk=0)
    assert torch.equal(h0, h1) and torch.equal(w0, w1)


def test_backward_mode_switch_rejects_bad_modes():
    prev = _lib.slm_set_backward_mode(1)
    assert _lib.slm_set_backward_mode(2) == -1
    assert _lib.slm_set_backward_mode(-1) == -1
    assert _lib.slm_set_backward_mode(prev) == 1
