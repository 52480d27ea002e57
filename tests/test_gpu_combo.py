"""Weighted combinations ("Loss Functions", "Weighted Combinations") on the GPU against
the oracle: the combined loss and gradients, and every term reported on its own before
its weight is applied."""

import numpy as np
import pytest
import torch

import oracle
from lm_head_loss_streaming_b200 import _lib, synthetic
from parity_util import (argmax_targets_valid, assert_grad_close, assert_loss_close,
                         tie_slack, with_labels)

pytestmark = pytest.mark.gpu


def _gpu(weights, inp, chunk_tokens=0):
    from lm_head_loss_streaming_b200.loss import lm_head_loss_combo_bwd, lm_head_loss_combo_fwd
    dev = torch.device("cuda", 0)
    Hq, W = inp.Hq.to(dev), inp.W.to(dev)
    Hp = inp.Hp.to(dev) if inp.Hp is not None else None
    lab = inp.labels.to(dev) if inp.labels is not None else None
    f = lm_head_loss_combo_fwd(weights, Hq, W, lab, Hp, inp.ignore_index, chunk_tokens)
    st_f = _lib.slm_device_status(f.workspace.data_ptr(), torch.cuda.current_stream().cuda_stream)
    dH, dW = lm_head_loss_combo_bwd(f, Hq, W, lab, Hp, inp.ignore_index,
                                    chunk_tokens=chunk_tokens)
    torch.cuda.synchronize()
    return dict(loss=f.loss_mean.item(), loss_sum=f.loss_sum.item(), n_valid=f.n_valid.item(),
                tok=f.loss_tok.double().cpu().numpy(),
                terms=f.term_loss_tok.double().cpu().numpy(),
                term_sums=f.term_loss_sum.cpu().numpy(), stats32=f.stats.cpu().numpy(),
                dH=dH.double().cpu().numpy(), dW=dW.double().cpu().numpy(), st=st_f,
                means=f.term_means())


def _reference(weights, inp, g):
    """Oracle reference; an argmax-p term is evaluated on the GPU's (validated) targets."""
    w_plain = {k: v for k, v in weights.items() if k != "ce_argmax_p"}
    Hp = inp.Hp
    tok = np.zeros(inp.N)
    dH = np.zeros((inp.N, inp.d))
    dW = np.zeros((inp.V, inp.d))
    terms = {}
    n_valid = None
    if w_plain:
        r = oracle.combo_forward(w_plain, inp.Hq, inp.W, inp.labels, Hp, inp.ignore_index)
        h, w = oracle.combo_backward(w_plain, inp.Hq, inp.W, inp.labels, Hp, None,
                                     inp.ignore_index)
        tok += r["loss_tok"]
        dH += h
        dW += w
        terms.update({k: t["loss_tok"] for k, t in r["terms"].items()})
        n_valid = r["n_valid"]
    if "ce_argmax_p" in weights:
        y = g["stats32"][8].view(np.int32)
        assert argmax_targets_valid(inp, y) <= 0.01
        inp_y = with_labels(inp, y)
        r = oracle.forward("ce", inp_y.Hq, inp_y.W, inp_y.labels, None, inp.ignore_index)
        # The gradient of the mean divides by the combination's valid count.
        nv = n_valid if n_valid is not None else r["n_valid"]
        valid = inp_y.labels.numpy() != inp.ignore_index
        gt = np.where(valid, 1.0 / max(nv, 1), 0.0)
        h, w = oracle.backward("ce", inp_y.Hq, inp_y.W, inp_y.labels, None, gt, inp.ignore_index)
        wa = weights["ce_argmax_p"]
        tok += wa * r["loss_tok"]
        dH += wa * h
        dW += wa * w
        terms["ce_argmax_p"] = r["loss_tok"]
        n_valid = nv
    return tok, dH, dW, terms, n_valid


def _slack(weights, inp):
    sh = sw = 0.0
    for k, w in weights.items():
        a, b = tie_slack(inp, k)
        sh = sh + abs(w) * a
        sw = sw + abs(w) * b
    return sh, sw


def _check(weights, inp, chunk_tokens=0, what=""):
    g = _gpu(weights, inp, chunk_tokens)
    assert g["st"] == 0
    tok, dH, dW, terms, n_valid = _reference(weights, inp, g)
    assert g["n_valid"] == n_valid
    ref_loss = tok.sum() / max(n_valid, 1)
    assert_loss_close(g["tok"], tok, g["loss"], ref_loss, what)
    for k, t in terms.items():
        kid = _lib.KIND[k]
        assert_loss_close(g["terms"][kid], t, what=f"{what} term {k}")
        assert abs(g["term_sums"][kid] - t.sum()) <= 2e-3 * max(abs(t.sum()), 1e-2)
        assert abs(g["means"][k] - t.sum() / max(n_valid, 1)) <= 2e-3 * max(abs(t.sum() / max(n_valid, 1)), 1e-2)
    for k in range(_lib.SLM_NUM_KINDS):   # absent terms report 0
        if not any(_lib.KIND[n] == k for n in weights):
            assert np.abs(g["terms"][k]).max() == 0.0
    sh, sw = _slack(weights, inp)
    assert_grad_close(g["dH"], dH, what + " dH", sh)
    assert_grad_close(g["dW"], dW, what + " dW", sw)
    return g


def test_page_example_ce_and_tv():
    """The page's own example: {"ce": 0.1, "tv": 0.9}."""
    inp = synthetic.make("tv", 300, 264, 1000, w_std=0.05, ignore_frac=0.1, seed=61,
                         with_labels=True)
    _check({"ce": 0.1, "tv": 0.9}, inp, what="ce+tv")


def test_divergence_mix_chunked():
    inp = synthetic.make("kl_div", 700, 128, 3000, w_std=0.05, ignore_frac=0.05, seed=62)
    _check({"kl_div": 1.0, "rkl": 0.5, "jsd": 2.0}, inp, chunk_tokens=200, what="kl+rkl+jsd")


def test_every_kind_at_once():
    inp = synthetic.make("lk_hybrid", 257, 64, 2050, w_std=0.1, ignore_frac=0.1, seed=63,
                         with_labels=True)
    w = {"ce": 0.3, "kl_div": 0.7, "tv": 0.2, "nla": 0.1, "lk_hybrid": 0.5, "rkl": 0.25,
         "jsd": 1.5, "ce_argmax_p": 0.4}
    _check(w, inp, what="all kinds")


@pytest.mark.parametrize("kind", ["ce", "kl_div", "nla", "jsd"])
def test_single_term_matches_single_kind_entry_point(kind):
    from lm_head_loss_streaming_b200.loss import lm_head_loss_bwd, lm_head_loss_fwd
    inp = synthetic.make(kind, 200, 128, 1500, w_std=0.05, ignore_frac=0.1, seed=64)
    g = _gpu({kind: 1.0}, inp)
    dev = torch.device("cuda", 0)
    Hq, W = inp.Hq.to(dev), inp.W.to(dev)
    Hp = inp.Hp.to(dev) if inp.Hp is not None else None
    lab = inp.labels.to(dev) if inp.labels is not None else None
    f = lm_head_loss_fwd(kind, Hq, W, lab, Hp, inp.ignore_index)
    dH, dW = lm_head_loss_bwd(f, Hq, W, lab, Hp, inp.ignore_index)
    ref_tok = f.loss_tok.double().cpu().numpy()
    assert_loss_close(g["tok"], ref_tok, g["loss"], f.loss_mean.item(), f"single {kind}")
    sh, sw = tie_slack(inp, kind)
    assert_grad_close(g["dH"], dH.double().cpu().numpy(), f"single {kind} dH", sh)
    assert_grad_close(g["dW"], dW.double().cpu().numpy(), f"single {kind} dW", sw)


def test_full_size_combination_sampled_rows():
    """{"kl_div": 1, "tv": 0.5} at the Llama-3.1-8B shape: sampled rows against the oracle."""
    from lm_head_loss_streaming_b200.loss import lm_head_loss_combo_bwd, lm_head_loss_combo_fwd
    inp = synthetic.workload("llama8b_kl", seed=0)
    weights = {"kl_div": 1.0, "tv": 0.5}
    dev = torch.device("cuda", 0)
    Hq, W, Hp = inp.Hq.to(dev), inp.W.to(dev), inp.Hp.to(dev)
    f = lm_head_loss_combo_fwd(weights, Hq, W, None, Hp)
    rows = np.sort(np.random.default_rng(7).choice(inp.N, 32, replace=False))
    gt = np.zeros(inp.N, np.float32)
    gt[rows] = 1.0
    dH, dW = lm_head_loss_combo_bwd(f, Hq, W, None, Hp, grad_tok=torch.from_numpy(gt).to(dev),
                                    normalize=False)
    tok = f.loss_tok.double().cpu().numpy()
    sl = torch.from_numpy(rows)
    r = oracle.combo_forward(weights, inp.Hq[sl], inp.W, None, inp.Hp[sl])
    rh, rw = oracle.combo_backward(weights, inp.Hq[sl], inp.W, None, inp.Hp[sl],
                                   np.ones(len(rows)))
    assert_loss_close(tok[rows], r["loss_tok"], what="full-size combo loss")
    sh = sw = 0.0
    for k, w in weights.items():
        a, b = tie_slack(inp, k, rows=sl, grad_tok=np.ones(len(rows)))
        sh = sh + w * a
        sw = sw + w * b
    assert_grad_close(dH[sl.to(dev)].double().cpu().numpy(), rh, "full-size combo dH", sh)
    assert_grad_close(dW.double().cpu().numpy(), rw, "full-size combo dW", sw)
