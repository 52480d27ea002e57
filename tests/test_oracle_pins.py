"""Pins of the float64 oracle to things other than itself (CPU only).

Every check here comes from the pages' definitions and printed figures, from closed forms,
from library routines (torch autograd in float64, scipy) or from brute force on tiny
inputs.  They are chosen so that a dropped term, a wrong sign or index or a transposed
operand anywhere in the oracle fails at least one of them.
"""

import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import slm_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LN2 = math.log(2.0)


def _rand(n, d, V, seed, w_std=0.5, corr=0.7):
    rng = np.random.default_rng(seed)
    Hp = rng.standard_normal((n, d))
    Hq = corr * Hp + math.sqrt(1 - corr**2) * rng.standard_normal((n, d))
    W = w_std * rng.standard_normal((V, d))
    y = rng.integers(0, V, n)
    return Hq, Hp, W, y


# --------------------------------------------------------------------------------------
# Golden figures printed on the pages (memory arithmetic of the LM loss path).
# --------------------------------------------------------------------------------------
def test_paper_memory_figures():
    with open(os.path.join(GOLDEN, "paper_memory.json")) as f:
        gold = json.load(f)
    gib = float(1 << 30)
    e = gold["logits_fp32"]
    got = oracle.logits_bytes(e["batch"], e["seq"], e["vocab"], e["dtype_bytes"]) / gib
    assert abs(got - e["printed_gib"]) <= e["printed_tolerance_gib"]
    e = gold["hidden_bf16"]
    got = oracle.logits_bytes(e["batch"], e["seq"], e["hidden"], e["dtype_bytes"]) / gib
    assert abs(got - e["printed_gib"]) <= e["printed_tolerance_gib"]
    e = gold["logits_plus_grad"]
    got = 2 * oracle.logits_bytes(e["batch"], e["seq"], e["vocab"], e["dtype_bytes"]) / gib
    assert abs(got - e["printed_gib"]) <= e["printed_tolerance_gib"]
    e = gold["chunk_buffer"]
    got = oracle.chunk_buffer_bytes(e["chunk"], e["vocab_stated"], e["dtype_bytes"]) / gib
    assert abs(got - e["printed_gib"]) <= e["printed_tolerance_gib"]
    # The page's own formula with 150000 does not give its printed figure (garbled line).
    bad = oracle.chunk_buffer_bytes(e["chunk"], e["vocab_in_formula"], e["dtype_bytes"]) / gib
    assert abs(bad - e["printed_gib"]) > 0.1


# --------------------------------------------------------------------------------------
# C1: all-zero logits (W = 0): CE = log V, dH = 0, closed-form dW.
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("V", [4096, 128256])
def test_zero_logits_ce_is_log_v(V):
    n, d = 6, 8
    rng = np.random.default_rng(1)
    H = rng.standard_normal((n, d))
    W = np.zeros((V, d))
    y = rng.integers(0, V, n)
    y[2] = -100
    out = orc.forward("ce", H, W, y)
    valid = y != -100
    assert np.allclose(out["loss_tok"][valid], math.log(V), rtol=0, atol=1e-12)
    assert out["loss_tok"][2] == 0.0
    assert out["n_valid"] == n - 1
    g = rng.standard_normal(n)
    dH, dW = orc.backward("ce", H, W, y, grad_tok=g)
    assert np.abs(dH).max() == 0.0
    # dW_v = sum_n g_n (1/V - [v = y_n]) H_n over valid rows, built row by row here.
    exp = np.zeros((V, d))
    for i in range(n):
        if not valid[i]:
            continue
        exp += g[i] * (1.0 / V) * H[i][None, :]
        exp[y[i]] -= g[i] * H[i]
    assert np.allclose(dW, exp, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------------------
# C2: p = q gives KL = 0, alpha = 1, TV = nla = lk = jsd = rkl = 0 and zero gradients.
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("kind", orc.DISTRIBUTION_KINDS)
def test_identical_target_and_draft(kind):
    Hq, _, W, _ = _rand(5, 7, 13, seed=2)
    out = orc.forward(kind, Hq, W, Hp=Hq)
    assert np.abs(out["loss_tok"]).max() <= 1e-14
    assert np.allclose(out["alpha"], 1.0, atol=1e-14)
    dH, dW = orc.backward(kind, Hq, W, Hp=Hq, grad_tok=np.ones(5))
    assert np.abs(dH).max() <= 1e-14 and np.abs(dW).max() <= 1e-14


# --------------------------------------------------------------------------------------
# C3/C4: bounds ("jsd ... bounded by log 2"; alpha is an acceptance rate).
# --------------------------------------------------------------------------------------
def test_ranges_and_jsd_bound():
    Hq, Hp, W, _ = _rand(32, 16, 50, seed=3, w_std=1.0, corr=0.2)
    res = {k: orc.forward(k, Hq, W, Hp=Hp) for k in orc.DISTRIBUTION_KINDS}
    a = res["tv"]["alpha"]
    assert (a >= 0).all() and (a <= 1).all()
    assert (res["tv"]["loss_tok"] >= 0).all() and (res["tv"]["loss_tok"] <= 1).all()
    assert (res["kl_div"]["loss_tok"] >= -1e-12).all()
    assert (res["rkl"]["loss_tok"] >= -1e-12).all()
    assert (res["nla"]["loss_tok"] >= 0).all()
    j = res["jsd"]["loss_tok"]
    assert (j >= -1e-12).all() and (j <= LN2 + 1e-12).all()


def test_jsd_and_alpha_near_disjoint():
    # Two rows whose target and draft put their mass on different tokens.
    V, d = 6, 6
    W = np.eye(V, d) * 60.0
    Hp = np.zeros((2, d)); Hq = np.zeros((2, d))
    Hp[0, 0] = 1; Hq[0, 1] = 1
    Hp[1, 2] = 1; Hq[1, 5] = 1
    j = orc.forward("jsd", Hq, W, Hp=Hp)["loss_tok"]
    assert np.allclose(j, LN2, atol=1e-12)
    out = orc.forward("lk_hybrid", Hq, W, Hp=Hp)
    assert (out["alpha"] < 1e-20).all()
    # lambda = exp(-3 alpha) -> 1 as the overlap vanishes: lk_hybrid reduces to KL.
    kl = orc.forward("kl_div", Hq, W, Hp=Hp)["loss_tok"]
    assert np.allclose(out["loss_tok"], kl, rtol=1e-12)


def test_lk_hybrid_weighting_at_known_alpha():
    # Two-token vocabulary where alpha has a closed form: p = (a, 1-a), q = (b, 1-b).
    for a, b in [(0.9, 0.6), (0.3, 0.45), (0.5, 0.5)]:
        zp = np.array([[math.log(a), math.log(1 - a)]])
        zq = np.array([[math.log(b), math.log(1 - b)]])
        t = orc.token_terms("lk_hybrid", zq, zp)
        alpha = min(a, b) + min(1 - a, 1 - b)
        kl = a * math.log(a / b) + (1 - a) * math.log((1 - a) / (1 - b))
        lam = math.exp(-3 * alpha)
        assert abs(t["alpha"][0] - alpha) < 1e-14
        # S = sum of q over the tokens where the draft is below the target.
        S = (b if b < a else 0.0) + ((1 - b) if (1 - b) < (1 - a) else 0.0)
        assert abs(t["S"][0] - S) < 1e-14
        assert abs(t["loss"][0] - (lam * kl + (1 - lam) * (1 - alpha))) < 1e-14
        assert abs(orc.token_terms("tv", zq, zp)["loss"][0] - 0.5 * (abs(a - b) * 2)) < 1e-14
        assert abs(orc.token_terms("nla", zq, zp)["loss"][0] + math.log(alpha)) < 1e-14


# --------------------------------------------------------------------------------------
# C5: masked rows contribute nothing; an all-masked batch gives 0.
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("kind", ["ce", "kl_div", "tv", "nla", "lk_hybrid"])
def test_masked_rows(kind):
    Hq, Hp, W, y = _rand(6, 5, 9, seed=4)
    y[[1, 4]] = -100
    lab = y
    out = orc.forward(kind, Hq, W, lab, Hp=Hp)
    assert out["loss_tok"][1] == 0 and out["loss_tok"][4] == 0
    assert out["n_valid"] == 4
    dH, dW = orc.backward(kind, Hq, W, lab, Hp=Hp)
    assert np.abs(dH[[1, 4]]).max() == 0
    # Same as running without the masked rows at all (dW gets nothing from them).
    keep = [0, 2, 3, 5]
    out2 = orc.forward(kind, Hq[keep], W, lab[keep], Hp=Hp[keep])
    dH2, dW2 = orc.backward(kind, Hq[keep], W, lab[keep], Hp=Hp[keep])
    assert abs(out["loss"] - out2["loss"]) < 1e-13
    assert np.allclose(dW, dW2, atol=1e-14)
    assert np.allclose(dH[keep], dH2, atol=1e-14)
    # Everything masked.
    allm = np.full(6, -100)
    out3 = orc.forward(kind, Hq, W, allm, Hp=Hp)
    assert out3["loss"] == 0.0 and out3["n_valid"] == 0
    dH3, dW3 = orc.backward(kind, Hq, W, allm, Hp=Hp)
    assert np.abs(dH3).max() == 0 and np.abs(dW3).max() == 0


def test_label_out_of_range_is_an_error():
    Hq, _, W, y = _rand(3, 4, 5, seed=5)
    y[0] = 5
    with pytest.raises(ValueError):
        orc.forward("ce", Hq, W, y)


# --------------------------------------------------------------------------------------
# C6: central finite differences on tiny shapes for every kind.
# --------------------------------------------------------------------------------------
def _objective(kind, Hq, W, y, zp, g, lam0=None):
    # The target logits zp are passed in fixed: the target is detached, so perturbing W
    # must not move p.
    zq = orc.logits(Hq, W)
    t = orc.token_terms(kind, zq, zp, y)
    if kind == "lk_hybrid":
        # lambda is detached: hold it at its value at the base point.
        return float((g * (lam0 * t["kl"] + (1 - lam0) * (1 - t["alpha"]))).sum())
    return float((g * t["loss"]).sum())


@pytest.mark.parametrize("kind", orc.KINDS)
def test_finite_differences(kind):
    n, d, V = 4, 6, 11
    for seed in range(10, 60):
        Hq, Hp, W, y = _rand(n, d, V, seed=seed, w_std=0.6, corr=0.5)
        zq, zp = orc.logits(Hq, W), orc.logits(Hp, W)
        p = np.exp(orc.log_softmax(zp)); q = np.exp(orc.log_softmax(zq))
        if np.abs(p - q).min() > 1e-3:   # keep the min() kink out of reach
            break
    Hp_ = None if kind == "ce" else Hp
    g = np.random.default_rng(seed).uniform(0.5, 1.5, n)
    lam0 = None
    if kind == "lk_hybrid":
        lam0 = orc.token_terms(kind, zq, zp)["lam"]
    dH, dW = orc.backward(kind, Hq, W, y, Hp=Hp_, grad_tok=g)
    zp0 = None if kind == "ce" else orc.logits(Hp, W)
    h = 1e-6
    for X, dX in ((Hq, dH), (W, dW)):
        num = np.zeros_like(X)
        for idx in np.ndindex(*X.shape):
            old = X[idx]
            X[idx] = old + h
            fp = _objective(kind, Hq, W, y, zp0, g, lam0)
            X[idx] = old - h
            fm = _objective(kind, Hq, W, y, zp0, g, lam0)
            X[idx] = old
            num[idx] = (fp - fm) / (2 * h)
        assert np.abs(num - dX).max() <= 1e-7 * max(1.0, np.abs(dX).max()), kind


# --------------------------------------------------------------------------------------
# C7: library routines (torch float64 losses and autograd; scipy).
# --------------------------------------------------------------------------------------
def test_ce_matches_torch_cross_entropy_and_autograd():
    Hq, _, W, y = _rand(9, 12, 31, seed=6)
    y[3] = -100
    H_t = torch.tensor(Hq, requires_grad=True)
    W_t = torch.tensor(W, requires_grad=True)
    ref = F.cross_entropy(H_t @ W_t.T, torch.tensor(y), ignore_index=-100, reduction="mean")
    ref.backward()
    L, dH, dW, f = orc.loss_and_grads("ce", Hq, W, y)
    assert abs(L - ref.item()) < 1e-13
    assert np.allclose(dH, H_t.grad.numpy(), atol=1e-14)
    assert np.allclose(dW, W_t.grad.numpy(), atol=1e-14)
    s = F.cross_entropy(torch.tensor(Hq @ W.T), torch.tensor(y), ignore_index=-100,
                        reduction="sum")
    assert abs(f["loss_sum"] - s.item()) < 1e-12
    lse = torch.logsumexp(torch.tensor(Hq @ W.T), dim=1).numpy()
    assert np.allclose(f["lse_q"], lse, atol=1e-13)


def _torch_loss(kind, zq, zp):
    lq = torch.log_softmax(zq, 1)
    lp = torch.log_softmax(zp, 1)
    q, p = lq.exp(), lp.exp()
    if kind == "kl_div":
        return F.kl_div(lq, lp, log_target=True, reduction="none").sum(1)
    if kind == "rkl":
        return F.kl_div(lp, lq, log_target=True, reduction="none").sum(1)
    alpha = torch.minimum(p, q).sum(1)
    if kind == "tv":
        return 0.5 * (p - q).abs().sum(1)      # total variation distance
    if kind == "nla":
        return -torch.log(alpha)
    if kind == "lk_hybrid":
        lam = torch.exp(-3 * alpha).detach()
        kl = F.kl_div(lq, lp, log_target=True, reduction="none").sum(1)
        return lam * kl + (1 - lam) * 0.5 * (p - q).abs().sum(1)
    if kind == "jsd":
        m = 0.5 * (p + q)
        return 0.5 * (F.kl_div(m.log(), lp, log_target=True, reduction="none").sum(1)
                      + F.kl_div(m.log(), lq, log_target=True, reduction="none").sum(1))
    raise ValueError(kind)


@pytest.mark.parametrize("kind", orc.DISTRIBUTION_KINDS)
def test_distribution_losses_match_torch_autograd(kind):
    n, d, V = 7, 10, 23
    Hq, Hp, W, _ = _rand(n, d, V, seed=7, w_std=0.7)
    g = np.random.default_rng(8).uniform(0.2, 2.0, n)
    H_t = torch.tensor(Hq, requires_grad=True)
    W_t = torch.tensor(W, requires_grad=True)
    zp = (torch.tensor(Hp) @ W_t.T).detach()   # the target is detached
    per = _torch_loss(kind, H_t @ W_t.T, zp)
    (per * torch.tensor(g)).sum().backward()
    out = orc.forward(kind, Hq, W, Hp=Hp)
    dH, dW = orc.backward(kind, Hq, W, Hp=Hp, grad_tok=g)
    assert np.allclose(out["loss_tok"], per.detach().numpy(), atol=1e-13)
    assert np.allclose(dH, H_t.grad.numpy(), atol=1e-12)
    assert np.allclose(dW, W_t.grad.numpy(), atol=1e-12)


def test_jsd_matches_scipy():
    from scipy.spatial.distance import jensenshannon
    Hq, Hp, W, _ = _rand(5, 8, 17, seed=9, w_std=1.0)
    out = orc.forward("jsd", Hq, W, Hp=Hp)
    p = np.exp(orc.log_softmax(orc.logits(Hp, W)))
    q = np.exp(orc.log_softmax(orc.logits(Hq, W)))
    for i in range(5):
        assert abs(out["loss_tok"][i] - jensenshannon(p[i], q[i]) ** 2) < 1e-12


# --------------------------------------------------------------------------------------
# Brute force on a tiny case with Python floats.
# --------------------------------------------------------------------------------------
def test_brute_force_python_floats():
    Hq, Hp, W, y = _rand(3, 4, 5, seed=11)
    ce = orc.forward("ce", Hq, W, y)["loss_tok"]
    kl = orc.forward("kl_div", Hq, W, Hp=Hp)["loss_tok"]
    for i in range(3):
        zq = [sum(Hq[i][k] * W[v][k] for k in range(4)) for v in range(5)]
        zp = [sum(Hp[i][k] * W[v][k] for k in range(4)) for v in range(5)]
        sq = sum(math.exp(z) for z in zq)
        sp = sum(math.exp(z) for z in zp)
        assert abs(ce[i] - (math.log(sq) - zq[y[i]])) < 1e-12
        brute = sum(math.exp(zp[v]) / sp * ((zp[v] - math.log(sp)) - (zq[v] - math.log(sq)))
                    for v in range(5))
        assert abs(kl[i] - brute) < 1e-12


# --------------------------------------------------------------------------------------
# C8/C9: invariants that tie dH and dW together (used at full scale on the GPU path).
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("kind", orc.KINDS)
def test_gradient_invariants(kind):
    Hq, Hp, W, y = _rand(12, 9, 19, seed=12)
    g = np.random.default_rng(13).uniform(0.1, 1.0, 12)
    Hp_ = None if kind == "ce" else Hp
    dH, dW = orc.backward(kind, Hq, W, y, Hp=Hp_, grad_tok=g)
    # <dH, H> = <dW, W> = sum_n g_n sum_v dz_nv z_nv.
    a, b = (dH * Hq).sum(), (dW * W).sum()
    assert abs(a - b) <= 1e-12 * max(1.0, abs(a))
    # Softmax-Jacobian rows sum to zero, so the columns of dW sum to zero.
    assert np.abs(dW.sum(axis=0)).max() <= 1e-12


# --------------------------------------------------------------------------------------
# C10: streaming equals dense up to reduction order, for any chunk size.
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("kind", ["ce", "kl_div", "lk_hybrid"])
def test_chunk_size_does_not_change_result(kind):
    Hq, Hp, W, y = _rand(23, 8, 29, seed=14)
    y[[0, 5, 22]] = -100
    Hp_ = None if kind == "ce" else Hp
    lab = y
    ref = orc.forward(kind, Hq, W, lab, Hp=Hp_, chunk_size=23)
    dHr, dWr = orc.backward(kind, Hq, W, lab, Hp=Hp_, chunk_size=23)
    for cs in (1, 7, 1000):
        out = orc.forward(kind, Hq, W, lab, Hp=Hp_, chunk_size=cs)
        assert abs(out["loss"] - ref["loss"]) <= 1e-12 * abs(ref["loss"])
        dH, dW = orc.backward(kind, Hq, W, lab, Hp=Hp_, chunk_size=cs)
        assert np.allclose(dH, dHr, atol=1e-14) and np.allclose(dW, dWr, atol=1e-14)


# --------------------------------------------------------------------------------------
# C11 (loose statistical sanity) and C12 (overflow safety).
# --------------------------------------------------------------------------------------
def test_ce_statistical_scale():
    # Gaussian logits of variance s2: E[CE] ~ log V + s2/2 for large V.
    n, d, V = 64, 256, 4096
    rng = np.random.default_rng(15)
    H = rng.standard_normal((n, d))
    W = 0.05 * rng.standard_normal((V, d))
    y = rng.integers(0, V, n)
    s2 = d * 0.05**2
    L = orc.forward("ce", H, W, y)["loss"]
    assert abs(L - (math.log(V) + s2 / 2)) < 0.15


def test_large_logits_are_finite_and_match_torch():
    Hq, Hp, W, y = _rand(6, 8, 40, seed=16, w_std=1.0)
    W = W * 100.0
    out = orc.forward("ce", Hq, W, y)
    assert np.isfinite(out["loss_tok"]).all()
    ref = F.cross_entropy(torch.tensor(Hq @ W.T), torch.tensor(y), reduction="none").numpy()
    assert np.allclose(out["loss_tok"], ref, rtol=1e-12)
    kl = orc.forward("kl_div", Hq, W, Hp=Hp)["loss_tok"]
    assert np.isfinite(kl).all()


# --------------------------------------------------------------------------------------
# "ce" row of the loss table: cross entropy against argmax p (hard labels from the target).
# --------------------------------------------------------------------------------------
def test_ce_argmax_p_matches_torch():
    Hq, Hp, W, y = _rand(11, 9, 21, seed=40, w_std=0.8)
    lab = y.copy()
    lab[[2, 7]] = -100                      # optional row mask
    H_t = torch.tensor(Hq, requires_grad=True)
    W_t = torch.tensor(W, requires_grad=True)
    zp = torch.tensor(Hp) @ W_t.T.detach()
    target = torch.argmax(zp, dim=1)        # first maximal index on ties
    target[[2, 7]] = -100
    ref = F.cross_entropy(H_t @ W_t.T, target, ignore_index=-100, reduction="mean")
    ref.backward()
    L, dH, dW, f = orc.loss_and_grads("ce_argmax_p", Hq, W, lab, Hp)
    assert abs(L - ref.item()) < 1e-13
    assert np.allclose(dH, H_t.grad.numpy(), atol=1e-14)
    assert np.allclose(dW, W_t.grad.numpy(), atol=1e-14)
    assert f["n_valid"] == 9


def test_ce_argmax_p_ties_go_to_lowest_index():
    # Target logits with an exact three-way tie at columns 1, 3 and 4.
    zp = np.array([[0.0, 2.0, 1.0, 2.0, 2.0]])
    zq = np.array([[0.3, -0.1, 0.2, 0.5, 0.0]])
    t = orc.token_terms("ce_argmax_p", zq, zp)
    assert int(t["target"][0]) == 1
    lse = math.log(sum(math.exp(v) for v in zq[0]))
    assert abs(t["loss"][0] - (lse - zq[0, 1])) < 1e-14


# --------------------------------------------------------------------------------------
# "Weighted Combinations": weights used as given, each term reported before weighting.
# --------------------------------------------------------------------------------------
def test_combination_against_torch_autograd():
    # {"ce": 0.1, "tv": 0.9} as on the page, plus a three-term mix, against torch.
    Hq, Hp, W, y = _rand(8, 10, 19, seed=50, w_std=0.7)
    y[3] = -100
    for weights in ({"ce": 0.1, "tv": 0.9}, {"kl_div": 1.0, "rkl": 0.5, "jsd": 2.0}):
        H_t = torch.tensor(Hq, requires_grad=True)
        W_t = torch.tensor(W, requires_grad=True)
        zq = H_t @ W_t.T
        zp = (torch.tensor(Hp) @ W_t.T).detach()
        valid = torch.tensor(y != -100)
        total = torch.zeros(8, dtype=torch.float64)
        for k, w in weights.items():
            if k == "ce":
                per = F.cross_entropy(zq, torch.tensor(y), ignore_index=-100, reduction="none")
            else:
                per = _torch_loss(k, zq, zp)
            total = total + w * torch.where(valid, per, torch.zeros_like(per))
        L = total.sum() / valid.sum()
        L.backward()
        out = orc.combo_forward(weights, Hq, W, y, Hp)
        dH, dW = orc.combo_backward(weights, Hq, W, y, Hp)
        assert abs(out["loss"] - L.item()) < 1e-12
        assert np.allclose(out["loss_tok"], total.detach().numpy(), atol=1e-12)
        assert np.allclose(dH, H_t.grad.numpy(), atol=1e-12)
        assert np.allclose(dW, W_t.grad.numpy(), atol=1e-12)
        assert set(out["terms"]) == set(weights)   # each term also reported on its own
        for k in weights:
            assert np.allclose(out["terms"][k]["loss_tok"],
                               orc.forward(k, Hq, W, y, Hp)["loss_tok"], atol=0)


# --------------------------------------------------------------------------------------
# Draft-head helpers: alignment before chunking, and flatness.
# --------------------------------------------------------------------------------------
def test_align_labels_worked_examples():
    tok = np.array([[10, 11, 12, 13, 14, 15]])
    # Standard next-token targets (shift 1): the last position has none.
    assert orc.align_labels(tok, 1).tolist() == [[11, 12, 13, 14, 15, -100]]
    # A draft head two tokens ahead.
    assert orc.align_labels(tok, 2).tolist() == [[12, 13, 14, 15, -100, -100]]
    # Packed sequences [10 11 12 | 13 14 15]: targets never cross the boundary.
    seq = np.array([[0, 0, 0, 1, 1, 1]])
    assert orc.align_labels(tok, 1, seq_ids=seq).tolist() == [[11, 12, -100, 14, 15, -100]]
    assert orc.align_labels(tok, 2, seq_ids=seq).tolist() == [[12, -100, -100, 15, -100, -100]]
    # A loss mask on the target positions (e.g. only the answer tokens count).
    mask = np.array([[0, 0, 1, 1, 0, 1]])
    assert orc.align_labels(tok, 1, loss_mask=mask).tolist() == [[-100, 12, 13, -100, 15, -100]]


def test_align_then_chunk_equals_dense():
    # Aligning before chunking keeps the streaming loss equal to the dense one ([SD]).
    rng = np.random.default_rng(70)
    B, S, d, V = 3, 17, 8, 29
    tok = rng.integers(0, V, (B, S))
    seq = np.cumsum(rng.random((B, S)) < 0.2, axis=1)
    lab = orc.align_labels(tok, 2, seq_ids=seq).reshape(-1)
    H = rng.standard_normal((B * S, d))
    W = 0.5 * rng.standard_normal((V, d))
    dense = F.cross_entropy(torch.tensor(H @ W.T), torch.tensor(lab), ignore_index=-100)
    for cs in (1, 5, 51):
        assert abs(orc.forward("ce", H, W, lab, chunk_size=cs)["loss"] - dense.item()) < 1e-12


def test_flatness_closed_forms_and_scipy():
    from scipy.spatial.distance import cosine
    V = 37
    assert np.allclose(orc.flatness(np.zeros((2, V))), 1.0)           # uniform p
    z = np.zeros((1, V)); z[0, 5] = 800.0                               # one-hot p
    assert np.allclose(orc.flatness(z), 1.0 / math.sqrt(V))
    rng = np.random.default_rng(71)
    z = rng.standard_normal((4, V)) * 2
    p = np.exp(orc.log_softmax(z))
    ref = [1.0 - cosine(p[i], np.full(V, 1.0 / V)) for i in range(4)]
    assert np.allclose(orc.flatness(z), ref, atol=1e-12)
    assert np.allclose(orc.flatness(z), 1.0 / (math.sqrt(V) * np.linalg.norm(p, axis=1)))
