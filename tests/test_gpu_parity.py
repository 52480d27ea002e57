"""GPU-vs-oracle parity of the streaming LM-head loss, element by element, on seeded
inputs small enough for the float64 oracle but spanning several tiles and ragged tails.
Every call goes through the C ABI."""

import math

import numpy as np
import pytest
import torch

from lm_head_loss_streaming_b200 import synthetic
from parity_util import (argmax_targets_valid, assert_grad_close, assert_loss_close,
                         gpu_fwd_bwd, oracle_fwd_bwd, tie_slack, with_labels)

pytestmark = pytest.mark.gpu

KINDS = ["ce", "kl_div", "tv", "nla", "lk_hybrid", "rkl", "jsd", "ce_argmax_p"]


def _compare_argmax(inp, chunk_tokens=0, what="", fused=False):
    """CE against argmax p: the targets are an argmax decided in fp32 on the GPU.  Check
    they are valid argmaxes of the float64 target logits, then compare the loss and the
    gradients with the oracle's hard-label CE on the GPU's targets."""
    g = gpu_fwd_bwd(inp, "ce_argmax_p", chunk_tokens=chunk_tokens, fused=fused)
    assert g["st_fwd"] == 0 and g["st_bwd"] == 0, (g["st_fwd"], g["st_bwd"])
    y = g["stats32"][1].view(np.int32)
    assert argmax_targets_valid(inp, y) <= 0.01, what
    r = oracle_fwd_bwd(with_labels(inp, y), "ce")
    assert g["n_valid"] == r["n_valid"]
    assert_loss_close(g["loss_tok"], r["loss_tok"], g["loss_mean"], r["loss"], what)
    assert np.allclose(g["stats"][0], r["lse_q"], rtol=1e-5, atol=1e-4), what
    assert_grad_close(g["dH"], r["dH"], what + " dH")
    assert_grad_close(g["dW"], r["dW"], what + " dW")
    return g, r


def _compare(inp, kind, chunk_tokens=0, what="", fused=False):
    if kind == "ce_argmax_p":
        return _compare_argmax(inp, chunk_tokens, what, fused)
    g = gpu_fwd_bwd(inp, kind, chunk_tokens=chunk_tokens, fused=fused)
    r = oracle_fwd_bwd(inp, kind)
    assert g["st_fwd"] == 0 and g["st_bwd"] == 0, (g["st_fwd"], g["st_bwd"])
    assert g["n_valid"] == r["n_valid"]
    assert_loss_close(g["loss_tok"], r["loss_tok"], g["loss_mean"], r["loss"], what)
    assert abs(g["loss_sum"] - r["loss_sum"]) <= 2e-3 * max(abs(r["loss_sum"]), 1e-2)
    assert np.allclose(g["stats"][0], r["lse_q"], rtol=1e-5, atol=1e-4), what
    if kind != "ce":
        assert np.allclose(g["stats"][1], r["lse_p"], rtol=1e-5, atol=1e-4), what
    if kind in ("tv", "nla", "lk_hybrid"):
        assert np.abs(g["alpha"] - r["alpha"]).max() <= 2e-3, what
    sh, sw = tie_slack(inp, kind)
    assert_grad_close(g["dH"], r["dH"], what + " dH", sh)
    assert_grad_close(g["dW"], r["dW"], what + " dW", sw)
    return g, r


def test_tiny_ce_workload():
    """N=256, d=256, V=4096 CE with 10% ignored rows, seed 0: every output element."""
    inp = synthetic.workload("tiny_ce", seed=0)
    _compare(inp, "ce", what="tiny_ce")


@pytest.mark.parametrize("kind", KINDS)
def test_ragged_shapes(kind):
    """Tails in every dimension: N not a multiple of 128, d not a multiple of 64,
    V not a multiple of the vocabulary tile, and a masked fraction."""
    inp = synthetic.make(kind, 300, 264, 1000, w_std=0.05, ignore_frac=0.1, seed=1)
    _compare(inp, kind, what=f"ragged {kind}")


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("shape", [(1, 8, 50), (129, 64, 257), (130, 512, 4100)])
def test_edge_shapes(kind, shape):
    N, d, V = shape
    inp = synthetic.make(kind, N, d, V, w_std=0.1, ignore_frac=0.0, seed=2,
                         with_labels=(kind == "ce"))
    _compare(inp, kind, what=f"edge {kind} {shape}")


@pytest.mark.parametrize("kind", ["ce", "kl_div", "lk_hybrid", "jsd", "ce_argmax_p"])
def test_chunked_backward_matches(kind):
    """The backward's token chunking does not change the result (only reduction order)."""
    inp = synthetic.make(kind, 700, 128, 3000, w_std=0.05, ignore_frac=0.05, seed=3)
    g0, r = _compare(inp, kind, chunk_tokens=0, what="chunk auto")
    g1, _ = _compare(inp, kind, chunk_tokens=200, what="chunk 200")
    assert np.abs(g0["dW"] - g1["dW"]).max() <= 1e-3 * np.abs(r["dW"]).max()


def test_zero_weight_gives_log_v():
    """W = 0: every valid row's CE is log V, dH = 0 (closed form)."""
    inp = synthetic.make("ce", 200, 64, 5000, ignore_frac=0.1, seed=4)
    inp.W.zero_()
    g = gpu_fwd_bwd(inp, "ce")
    valid = inp.labels.numpy() != inp.ignore_index
    assert np.abs(g["loss_tok"][valid] - math.log(5000)).max() <= 2e-3 * math.log(5000)
    assert np.abs(g["dH"]).max() == 0.0


@pytest.mark.parametrize("kind", ["kl_div", "tv", "nla", "lk_hybrid", "rkl", "jsd"])
def test_identical_target_and_draft(kind):
    """p = q: KL = TV = nla = lk = RKL = JSD = 0, alpha = 1, gradients vanish."""
    inp = synthetic.make(kind, 150, 128, 2000, w_std=0.05, draft=("none",), seed=5)
    g = gpu_fwd_bwd(inp, kind)
    assert np.abs(g["loss_tok"]).max() <= 2e-3 * 1e-2 * 50
    if g["alpha"] is not None:
        assert np.abs(g["alpha"] - 1.0).max() <= 2e-3
    assert np.abs(g["dH"]).max() <= 1e-3 * 0.05
    assert np.abs(g["dW"]).max() <= 1e-3


@pytest.mark.parametrize("kind", ["ce", "kl_div"])
def test_all_rows_masked(kind):
    inp = synthetic.make(kind, 140, 64, 700, ignore_frac=1.0, seed=6, with_labels=True)
    g = gpu_fwd_bwd(inp, kind)
    assert g["n_valid"] == 0 and g["loss_sum"] == 0.0 and g["loss_mean"] == 0.0
    assert np.abs(g["loss_tok"]).max() == 0
    assert np.abs(g["dH"]).max() == 0 and np.abs(g["dW"]).max() == 0


def test_label_out_of_range_is_reported_and_masked():
    inp = synthetic.make("ce", 260, 64, 900, ignore_frac=0.0, seed=7)
    inp.labels[5] = 900
    inp.labels[77] = -3
    g = gpu_fwd_bwd(inp, "ce")
    assert g["st_fwd"] == 6  # SLM_ERR_LABEL_RANGE
    assert g["loss_tok"][5] == 0 and g["loss_tok"][77] == 0
    assert g["n_valid"] == 258
    assert np.abs(g["dH"][[5, 77]]).max() == 0


def test_accumulate_dw_and_grad_tok():
    """accumulate_dW adds to the caller's dW; grad_tok scales each row."""
    inp = synthetic.make("ce", 333, 128, 1500, w_std=0.05, ignore_frac=0.1, seed=8)
    rng = np.random.default_rng(8)
    gt = rng.uniform(0.0, 2.0, inp.N).astype(np.float32)
    base = rng.standard_normal((inp.V, inp.d)).astype(np.float32)
    g = gpu_fwd_bwd(inp, "ce", grad_tok=gt, normalize=False, accumulate_dW=base)
    r = oracle_fwd_bwd(inp, "ce", grad_tok=gt.astype(np.float64))
    assert_grad_close(g["dH"], r["dH"], "dH grad_tok")
    assert_grad_close(g["dW"] - base, r["dW"], "dW accumulate")


def test_empty_batch():
    inp = synthetic.make("ce", 0, 64, 300, seed=9)
    g = gpu_fwd_bwd(inp, "ce")
    assert g["n_valid"] == 0 and g["loss_mean"] == 0.0
    assert np.abs(g["dW"]).max() == 0.0


def test_large_logits_finite():
    """Logits in the hundreds: no overflow (max subtraction)."""
    inp = synthetic.make("kl_div", 128, 64, 999, w_std=3.0, seed=10)
    _compare(inp, "kl_div", what="large logits kl")
    inp = synthetic.make("ce", 128, 64, 999, w_std=3.0, seed=10)
    _compare(inp, "ce", what="large logits ce")


@pytest.mark.parametrize("fused", [False, True])
def test_autograd_wrapper(fused):
    from lm_head_loss_streaming_b200 import streaming_lm_head_loss
    inp = synthetic.make("kl_div", 200, 64, 1200, w_std=0.05, seed=11)
    Hq = inp.Hq.cuda().requires_grad_(True)
    W = inp.W.cuda().requires_grad_(True)
    loss = streaming_lm_head_loss(Hq, W, None, inp.Hp.cuda(), kind="kl_div", fused=fused)
    (2.0 * loss).backward()
    r = oracle_fwd_bwd(inp, "kl_div")
    assert abs(loss.item() - r["loss"]) <= 2e-3 * abs(r["loss"])
    assert_grad_close(Hq.grad.double().cpu().numpy(), 2 * r["dH"], "autograd dH")
    assert_grad_close(W.grad.double().cpu().numpy(), 2 * r["dW"], "autograd dW")


def test_jsd_bounded_by_log2_on_disjoint_targets():
    """Target and draft concentrated on different tokens: JSD approaches log 2."""
    inp = synthetic.make("jsd", 128, 64, 512, w_std=1.5, draft=("mix", -1.0, 0.0), seed=12)
    g = gpu_fwd_bwd(inp, "jsd")
    r = oracle_fwd_bwd(inp, "jsd")
    assert (g["loss_tok"] <= math.log(2) + 2e-3).all() and (g["loss_tok"] >= -2e-3).all()
    assert_loss_close(g["loss_tok"], r["loss_tok"], g["loss_mean"], r["loss"], "jsd disjoint")
