"""The fused single-call forward + backward (slm_loss_fwd_bwd), which keeps each chunk's
fp32 logits instead of recomputing them, against the oracle: every kind, several chunks
with ragged tails, and sampled rows at the workloads' full sizes."""

import numpy as np
import pytest
import torch

from lm_head_loss_streaming_b200 import synthetic
from parity_util import (argmax_targets_valid, assert_grad_close, assert_loss_close,
                         gpu_fwd_bwd, oracle_fwd_bwd, tie_slack, with_labels)
from test_gpu_parity import KINDS, _compare

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", KINDS)
def test_fused_ragged_several_chunks(kind):
    inp = synthetic.make(kind, 700, 264, 3001, w_std=0.05, ignore_frac=0.1, seed=71)
    _compare(inp, kind, chunk_tokens=256, what=f"fused {kind}", fused=True)


@pytest.mark.parametrize("kind", ["ce", "kl_div", "tv", "jsd"])
def test_fused_single_chunk_and_edges(kind):
    for shape in [(1, 8, 50), (300, 64, 257)]:
        inp = synthetic.make(kind, *shape, w_std=0.1, seed=72, with_labels=(kind == "ce"))
        _compare(inp, kind, what=f"fused {kind} {shape}", fused=True)


@pytest.mark.parametrize("kind", ["ce", "kl_div", "lk_hybrid"])
def test_fused_matches_two_call_path(kind):
    inp = synthetic.make(kind, 900, 256, 4097, w_std=0.05, ignore_frac=0.05, seed=73)
    a = gpu_fwd_bwd(inp, kind, fused=True, chunk_tokens=512)
    b = gpu_fwd_bwd(inp, kind, chunk_tokens=512)
    if kind in ("tv", "nla", "lk_hybrid", "jsd"):
        # The second pass sums over the kept logits in another order than the GEMM
        # epilogue's second pass: equal up to fp32 rounding.
        assert np.allclose(a["loss_tok"], b["loss_tok"], rtol=1e-5, atol=1e-6)
    else:
        assert np.array_equal(a["loss_tok"], b["loss_tok"])  # the same forward epilogue
    assert a["n_valid"] == b["n_valid"]
    # Same logits either way; a two-pass kind's alpha and S differ by fp32 rounding, which
    # can move a bf16-rounded dz by one unit: then the gradient tolerance of the tests.
    tol = 1e-2 if kind in ("tv", "nla", "lk_hybrid", "jsd") else 1e-3
    assert np.abs(a["dH"] - b["dH"]).max() <= tol * np.abs(b["dH"]).max()
    assert np.abs(a["dW"] - b["dW"]).max() <= tol * np.abs(b["dW"]).max()


def test_fused_grad_tok_and_accumulate():
    inp = synthetic.make("kl_div", 333, 128, 1500, w_std=0.05, ignore_frac=0.1, seed=74)
    rng = np.random.default_rng(74)
    gt = rng.uniform(0.0, 2.0, inp.N).astype(np.float32)
    base = rng.standard_normal((inp.V, inp.d)).astype(np.float32)
    g = gpu_fwd_bwd(inp, "kl_div", grad_tok=gt, accumulate_dW=base, fused=True)
    valid = inp.labels.numpy() != inp.ignore_index
    r = oracle_fwd_bwd(inp, "kl_div", grad_tok=gt.astype(np.float64) / valid.sum())
    assert_grad_close(g["dH"], r["dH"], "fused dH grad_tok")
    assert_grad_close(g["dW"] - base, r["dW"], "fused dW accumulate")


@pytest.mark.parametrize("name,kind", [("llama8b_kl", "kl_div"), ("alpha_losses", "tv"),
                                       ("llama1b_ce", "ce")])
def test_fused_full_size_sampled_rows(name, kind):
    from lm_head_loss_streaming_b200.loss import lm_head_loss_fwd_bwd
    inp = synthetic.workload(name, kind=kind, seed=0)
    dev = torch.device("cuda", 0)
    Hq, W = inp.Hq.to(dev), inp.W.to(dev)
    Hp = inp.Hp.to(dev) if kind != "ce" else None
    lab = inp.labels.to(dev) if inp.labels is not None else None
    rows = np.sort(np.random.default_rng(9).choice(inp.N, 40, replace=False))
    gt = np.zeros(inp.N, np.float32)
    gt[rows] = 1.0
    fwd, dH, dW = lm_head_loss_fwd_bwd(kind, Hq, W, lab, Hp, inp.ignore_index,
                                       grad_tok=torch.from_numpy(gt).to(dev))
    nv = int(fwd.n_valid.item())
    sl = torch.from_numpy(rows)
    # grad_tok is divided by the valid count inside the call: the oracle gets the same.
    ref = oracle_fwd_bwd(inp, kind, rows=sl, grad_tok=np.full(len(rows), 1.0 / nv))
    tok = fwd.loss_tok.double().cpu().numpy()
    assert_loss_close(tok[rows], ref["loss_tok"], what=f"fused full {name}")
    sh, sw = tie_slack(inp, kind, rows=sl, grad_tok=np.full(len(rows), 1.0 / nv))
    assert_grad_close(dH[sl.to(dev)].double().cpu().numpy(), ref["dH"], f"fused full {name} dH", sh)
    assert_grad_close(dW.double().cpu().numpy(), ref["dW"], f"fused full {name} dW", sw)
