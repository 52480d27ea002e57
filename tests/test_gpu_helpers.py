"""Draft-head helpers on the GPU against the oracle: target alignment before chunking
(integer work: bit-exact) and the per-token flatness of the target distribution."""

import math

import numpy as np
import pytest
import torch

import oracle
from lm_head_loss_streaming_b200 import synthetic

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shift", [0, 1, 2, 5, 2000])
@pytest.mark.parametrize("with_mask,with_seq", [(False, False), (True, False), (True, True)])
def test_align_labels_bit_exact(shift, with_mask, with_seq):
    from lm_head_loss_streaming_b200.loss import align_labels
    rng = np.random.default_rng(80 + shift)
    B, S = 3, 1000
    tok = rng.integers(0, 128256, (B, S)).astype(np.int32)
    mask = (rng.random((B, S)) < 0.8) if with_mask else None
    seq = np.cumsum(rng.random((B, S)) < 0.01, axis=1).astype(np.int32) if with_seq else None
    dev = torch.device("cuda", 0)
    got = align_labels(torch.from_numpy(tok).to(dev), shift,
                       None if mask is None else torch.from_numpy(mask).to(dev),
                       None if seq is None else torch.from_numpy(seq).to(dev))
    ref = oracle.align_labels(tok, shift, mask, seq).reshape(-1)
    assert np.array_equal(got.cpu().numpy().astype(np.int64), ref)


def test_align_labels_feeds_the_loss():
    """Aligned labels straight into the streaming loss equal the oracle's dense loss."""
    from lm_head_loss_streaming_b200.loss import align_labels, lm_head_loss_fwd
    rng = np.random.default_rng(90)
    B, S, d, V = 2, 300, 128, 2000
    tok = rng.integers(0, V, (B, S)).astype(np.int32)
    seq = np.cumsum(rng.random((B, S)) < 0.05, axis=1).astype(np.int32)
    inp = synthetic.make("ce", B * S, d, V, w_std=0.05, seed=91)
    dev = torch.device("cuda", 0)
    lab = align_labels(torch.from_numpy(tok).to(dev), 3, None, torch.from_numpy(seq).to(dev))
    f = lm_head_loss_fwd("ce", inp.Hq.to(dev), inp.W.to(dev), lab)
    ref = oracle.forward("ce", inp.Hq, inp.W, oracle.align_labels(tok, 3, None, seq).reshape(-1))
    assert int(f.n_valid.item()) == ref["n_valid"]
    assert abs(f.loss_mean.item() - ref["loss"]) <= 2e-3 * abs(ref["loss"])


@pytest.mark.parametrize("shape", [(300, 264, 3001), (1, 8, 50), (513, 128, 4096)])
def test_flatness_matches_oracle(shape):
    from lm_head_loss_streaming_b200.loss import target_flatness
    N, d, V = shape
    inp = synthetic.make("kl_div", N, d, V, w_std=0.1, seed=92)
    got = target_flatness(inp.Hp.cuda(), inp.W.cuda()).double().cpu().numpy()
    ref = oracle.flatness(oracle.logits(inp.Hp, inp.W))
    assert np.abs(got - ref).max() <= 2e-3 * np.abs(ref).max()


def test_flatness_closed_forms():
    from lm_head_loss_streaming_b200.loss import target_flatness
    inp = synthetic.make("kl_div", 130, 64, 1000, w_std=0.1, seed=93)
    W0 = torch.zeros_like(inp.W)
    assert np.allclose(target_flatness(inp.Hp.cuda(), W0.cuda()).cpu().numpy(), 1.0, atol=1e-5)
    # Peaked targets (logits in the hundreds): flatness -> 1/sqrt(V).
    inp = synthetic.make("kl_div", 130, 64, 1000, w_std=20.0, seed=94)
    got = target_flatness(inp.Hp.cuda(), inp.W.cuda()).cpu().numpy()
    ref = oracle.flatness(oracle.logits(inp.Hp, inp.W))
    assert np.allclose(got, ref, rtol=2e-3)
    # ||p||_2 <= 1, so 1/sqrt(V) <= flatness <= 1; peaked rows sit at the lower bound.
    assert (got >= 1 / math.sqrt(1000) - 1e-6).all() and (got <= 1 + 1e-6).all()
    assert np.median(got) < 1.01 / math.sqrt(1000)


def test_flatness_full_size_sampled():
    from lm_head_loss_streaming_b200.loss import target_flatness
    inp = synthetic.workload("llama8b_kl", seed=0)
    got = target_flatness(inp.Hp.cuda(), inp.W.cuda()).double().cpu().numpy()
    rows = np.sort(np.random.default_rng(95).choice(inp.N, 64, replace=False))
    ref = oracle.flatness(oracle.logits(inp.Hp[torch.from_numpy(rows)], inp.W))
    assert np.abs(got[rows] - ref).max() <= 2e-3 * np.abs(ref).max()
