"""Randomised properties of the float64 oracle (CPU only, hypothesis).

The fixed-shape pins in test_oracle_pins.py tie the oracle to closed forms, library
routines and the pages' figures.  These draw many small random shapes, scales, masks and
kinds and check what must hold for every input ("Loss Functions", "Available Losses";
"Training speculative decoders: removing the logits and attention bottlenecks",
"Streaming Cross Entropy"):
  * ranges: KL, RKL, JSD, CE >= 0, JSD <= log 2, 0 <= alpha <= 1, tv = 1 - alpha;
  * <dH, H> = <dW, W> and sum_v dW[v] = 0 (the target is detached; softmax-Jacobian rows
    sum to zero);
  * masked rows contribute nothing to the loss sum, the count or either gradient;
  * the streamed result does not depend on the chunk size;
  * CE and forward KL agree with torch's float64 definitions.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import slm_oracle as orc

KINDS = ["ce", "kl_div", "tv", "nla", "lk_hybrid", "rkl", "jsd"]
SETTINGS = settings(max_examples=40, deadline=None,
                    suppress_health_check=[HealthCheck.too_slow])


@st.composite
def problems(draw):
    n = draw(st.integers(1, 9))
    d = draw(st.integers(1, 7))
    V = draw(st.integers(2, 23))
    w_std = draw(st.sampled_from([0.05, 0.5, 2.0]))
    corr = draw(st.sampled_from([0.0, 0.6, 0.95]))
    seed = draw(st.integers(0, 2**31 - 1))
    kind = draw(st.sampled_from(KINDS))
    rng = np.random.default_rng(seed)
    Hp = rng.standard_normal((n, d))
    Hq = corr * Hp + math.sqrt(1 - corr**2) * rng.standard_normal((n, d))
    W = w_std * rng.standard_normal((V, d))
    y = rng.integers(0, V, n)
    mask = rng.random(n) < 0.3
    y = np.where(mask, -100, y)
    g = rng.uniform(0.1, 2.0, n)
    return kind, Hq, Hp, W, y, g


@SETTINGS
@given(problems())
def test_ranges(p):
    kind, Hq, Hp, W, y, _ = p
    r = orc.forward(kind, Hq, W, y, None if kind == "ce" else Hp)
    tok = np.asarray(r["loss_tok"])
    assert np.isfinite(tok).all()
    tol = 1e-12
    if kind in ("ce", "kl_div", "rkl", "jsd"):
        assert (tok >= -tol).all()
    if kind == "jsd":
        assert (tok <= math.log(2) + tol).all()
    if kind in ("tv", "nla", "lk_hybrid"):
        t = orc.token_terms(kind, orc.logits(Hq, W), orc.logits(Hp, W), y)
        alpha = np.asarray(t["alpha"])
        valid = y != -100
        assert ((alpha >= -tol) & (alpha <= 1 + tol)).all()
        if kind == "tv":
            assert np.allclose(tok[valid], 1 - alpha[valid], atol=1e-12)
    # Masked rows contribute nothing, and the count is the number of valid rows.
    assert np.all(tok[y == -100] == 0)
    assert r["n_valid"] == int((y != -100).sum())


@SETTINGS
@given(problems())
def test_gradient_identities_and_masking(p):
    kind, Hq, Hp, W, y, g = p
    Hp_ = None if kind == "ce" else Hp
    dH, dW = orc.backward(kind, Hq, W, y, Hp=Hp_, grad_tok=g)
    a, b = (dH * Hq).sum(), (dW * W).sum()
    assert abs(a - b) <= 1e-10 * max(1.0, abs(a), abs(b))
    assert np.abs(dW.sum(axis=0)).max() <= 1e-10 * max(1.0, np.abs(dW).max())
    assert np.all(dH[y == -100] == 0)
    # dW is the same with the masked rows removed altogether.
    keep = y != -100
    if keep.any():
        _, dW2 = orc.backward(kind, Hq[keep], W, y[keep], Hp=None if Hp_ is None else Hp[keep],
                              grad_tok=g[keep])
        assert np.allclose(dW, dW2, rtol=1e-10, atol=1e-13)


@SETTINGS
@given(problems(), st.integers(1, 5))
def test_chunk_size_invariance(p, chunk):
    kind, Hq, Hp, W, y, g = p
    Hp_ = None if kind == "ce" else Hp
    a = orc.forward(kind, Hq, W, y, Hp_)
    b = orc.forward(kind, Hq, W, y, Hp_, chunk_size=chunk)
    assert a["n_valid"] == b["n_valid"]
    assert abs(a["loss_sum"] - b["loss_sum"]) <= 1e-12 * max(1.0, abs(a["loss_sum"]))
    dHa, dWa = orc.backward(kind, Hq, W, y, Hp=Hp_, grad_tok=g)
    dHb, dWb = orc.backward(kind, Hq, W, y, Hp=Hp_, grad_tok=g, chunk_size=chunk)
    assert np.allclose(dHa, dHb, rtol=1e-12, atol=1e-14)
    assert np.allclose(dWa, dWb, rtol=1e-12, atol=1e-14)


@SETTINGS
@given(problems())
def test_ce_and_kl_match_torch(p):
    _, Hq, Hp, W, y, _ = p
    zq = torch.from_numpy(Hq @ W.T)
    zp = torch.from_numpy(Hp @ W.T)
    lab = torch.from_numpy(y)
    ce = orc.forward("ce", Hq, W, y)
    ref = F.cross_entropy(zq, lab, ignore_index=-100, reduction="sum").item()
    assert abs(ce["loss_sum"] - ref) <= 1e-10 * max(1.0, abs(ref))
    kl = orc.forward("kl_div", Hq, W, y, Hp)
    valid = lab != -100
    per = F.kl_div(F.log_softmax(zq, -1), F.log_softmax(zp, -1), log_target=True,
                   reduction="none").sum(-1)
    ref = per[valid].sum().item()
    assert abs(kl["loss_sum"] - ref) <= 1e-10 * max(1.0, abs(ref))
