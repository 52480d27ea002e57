"""Plain float64 CPU definition of the streaming LM-head loss and its gradients.

TEST INFRASTRUCTURE.  This module is the checker, not the product: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may call it.  It is
slow on purpose.  It materialises the logits of a block of rows, works in float64
throughout, and shares no code, constant or helper with the CUDA path.

Sources, cited by page title and section:

[SD] "Training speculative decoders: removing the logits and attention bottlenecks"
     - "The logits bottleneck in long-context draft-head training": the LM loss path
       hidden states -> LM head -> logits -> cross entropy -> loss, and the memory
       arithmetic of the logits tensor.
     - "Streaming Cross Entropy": the loss is a sum of independent per-token terms;
       tokens are processed in chunks, the masked per-chunk loss sum and valid-token
       count are accumulated, and the total is divided by the total count at the end.
     - "Correctness: alignment before chunking": targets and masks are aligned first,
       then chunked; the result equals the dense loss up to reduction order.
     - "Backward pass": per chunk, the logits are recomputed, the hidden-state gradient
       of the chunk is produced and the LM-head weight gradient is accumulated; the
       chunk buffer arithmetic chunk x vocab x dtype x 2.
     - Gradient-accumulation and streaming normalisation equations: normalise by the
       number of valid, non-masked tokens, never by the number of chunks.
[FT] "Flatter Tokens are More Valuable for Speculative Draft Model Training" (summary):
     flatness of a token = cosine similarity of the target distribution to uniform.
[LF] "Loss Functions" (speculators user guide), table "Available Losses": p is the
     target distribution, q the draft distribution, alpha = sum_v min(p_v, q_v);
     kl_div = forward KL target->draft, rkl = reverse KL, jsd = Jensen-Shannon,
     ce = cross entropy against argmax p (hard labels from the target),
     tv = 1 - alpha, nla = -log(alpha), lk_hybrid = lambda*KL + (1-lambda)*TV with
     lambda = exp(-3*alpha) detached.

Readings taken where the pages are silent (each one is also listed in the design notes):
  * Row mask: a row whose label equals ``ignore_index`` is masked.  For "ce" the labels
    are required and every other label must lie in [0, V).  For the distribution losses
    and "ce_argmax_p" the labels are optional and only act as a row mask.
  * "ce_argmax_p" is the table's "ce" row (cross entropy against argmax p); it is named
    apart from the hard-label "ce" of the streaming cross entropy page.  Ties of the
    argmax go to the lowest vocabulary index.
  * Denominator: the number of unmasked rows.  With every row masked the loss is 0 and
    every gradient is 0 (the pages do not say; a mean over zero rows is undefined).
  * KL direction: "Forward KL, target to draft" is KL(p || q).
  * The target p is detached: gradients flow to the draft hidden states H_q and to W
    through z_q only; there is no gradient for H_p.
  * alpha is per token, so lambda_n = exp(-3 alpha_n) is per token and detached.
  * d alpha / d q_v uses the strict indicator m_v = [q_v < p_v] (a tie gives 0).
  * Upstream gradient: token n's loss is scaled by g_n (``grad_tok``); the normalised
    mean loss uses g_n = 1/n_valid on valid rows.

Notation (per token row): z_q = H_q W^T, z_p = H_p W^T, L = logsumexp(z),
q = softmax(z_q), p = softmax(z_p), m_v = [q_v < p_v], S = sum_v m_v q_v.
"""

from __future__ import annotations

import numpy as np

KINDS = ("ce", "kl_div", "tv", "nla", "lk_hybrid", "rkl", "jsd", "ce_argmax_p")
DISTRIBUTION_KINDS = ("kl_div", "tv", "nla", "lk_hybrid", "rkl", "jsd")
# Kinds that read the target logits z_p (every kind but hard-label "ce").
TARGET_KINDS = DISTRIBUTION_KINDS + ("ce_argmax_p",)
ALPHA_KINDS = ("tv", "nla", "lk_hybrid")

GIB = float(1 << 30)


def _f64(x):
    """Widen to float64 (exact for bf16 / fp32 inputs)."""
    if hasattr(x, "detach"):  # a torch tensor: widen through float64 on the CPU
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def _labels(labels, n):
    if labels is None:
        return None
    if hasattr(labels, "detach"):
        labels = labels.detach().to("cpu").numpy()
    lab = np.asarray(labels).astype(np.int64).reshape(-1)
    if lab.shape[0] != n:
        raise ValueError("labels must have one entry per token row")
    return lab


# ----------------------------------------------------------------------------------------
# [SD] "The logits bottleneck...": hidden states -> LM head -> logits.
# ----------------------------------------------------------------------------------------
def logits(H, W):
    """Logits of a block of rows: H [n, d] times the LM head W [V, d] transposed -> [n, V]."""
    return _f64(H) @ _f64(W).T


def log_softmax(z):
    """Row-wise log-softmax with the row maximum subtracted before exponentiation."""
    z = _f64(z)
    m = z.max(axis=1, keepdims=True)
    s = np.exp(z - m).sum(axis=1, keepdims=True)
    return z - m - np.log(s)


def _logsumexp(z):
    m = z.max(axis=1)
    return m + np.log(np.exp(z - m[:, None]).sum(axis=1))


# ----------------------------------------------------------------------------------------
# [LF] "Available Losses": per-token objective of every loss kind.
# ----------------------------------------------------------------------------------------
def token_terms(kind, zq, zp=None, labels=None):
    """Per-token loss and the quantities the loss is built from, for one block of rows.

    ``labels`` is only read for "ce"; rows are not masked here (see ``forward``).
    Returns a dict with ``loss`` [n] and, where defined, ``lse_q``, ``lse_p``, ``kl``,
    ``alpha``, ``S`` (all [n]).
    """
    if kind not in KINDS:
        raise ValueError(f"unknown loss kind {kind!r}")
    zq = _f64(zq)
    n, V = zq.shape
    out = {"lse_q": _logsumexp(zq)}
    lq = zq - out["lse_q"][:, None]
    if kind == "ce":
        # Hard-label cross entropy: -log q_y.
        y = np.asarray(labels, dtype=np.int64)
        safe = np.clip(y, 0, V - 1)
        out["loss"] = -lq[np.arange(n), safe]
        return out
    zp = _f64(zp)
    if kind == "ce_argmax_p":
        # Cross entropy against the target's most likely token (lowest index on ties).
        y = argmax_target(zp)
        out["target"] = y
        out["loss"] = -lq[np.arange(n), y]
        return out
    out["lse_p"] = _logsumexp(zp)
    lp = zp - out["lse_p"][:, None]
    q = np.exp(lq)
    p = np.exp(lp)
    # Forward KL, target to draft: KL(p || q) = sum_v p_v (log p_v - log q_v).
    kl = (p * (lp - lq)).sum(axis=1)
    out["kl"] = kl
    # Distributional overlap alpha = sum_v min(p_v, q_v).
    alpha = np.minimum(p, q).sum(axis=1)
    out["alpha"] = alpha
    out["S"] = np.where(q < p, q, 0.0).sum(axis=1)
    if kind == "kl_div":
        out["loss"] = kl
    elif kind == "tv":
        out["loss"] = 1.0 - alpha
    elif kind == "nla":
        out["loss"] = -np.log(alpha)
    elif kind == "lk_hybrid":
        lam = np.exp(-3.0 * alpha)
        out["lam"] = lam
        out["loss"] = lam * kl + (1.0 - lam) * (1.0 - alpha)
    elif kind == "rkl":
        # Reverse KL, draft to target: KL(q || p).
        out["loss"] = (q * (lq - lp)).sum(axis=1)
    elif kind == "jsd":
        mix = 0.5 * (p + q)
        lm = np.log(mix)
        out["loss"] = 0.5 * (p * (lp - lm)).sum(axis=1) + 0.5 * (q * (lq - lm)).sum(axis=1)
    return out


def argmax_target(zp):
    """Hard labels from the target: argmax_v z_p (first, i.e. lowest, index on ties)."""
    return np.argmax(_f64(zp), axis=1)


def dlogits(kind, zq, zp=None, labels=None):
    """d(per-token loss)/d z_q for one block of rows (upstream gradient 1 per row).

    The target logits z_p are constants (detached).  For lk_hybrid lambda is held
    constant at its value (detached), as the loss table states.
    """
    zq = _f64(zq)
    n, V = zq.shape
    lq = log_softmax(zq)
    q = np.exp(lq)
    if kind == "ce":
        y = np.asarray(labels, dtype=np.int64)
        dz = q.copy()
        dz[np.arange(n), np.clip(y, 0, V - 1)] -= 1.0
        return dz
    if kind == "ce_argmax_p":
        dz = q.copy()
        dz[np.arange(n), argmax_target(zp)] -= 1.0
        return dz
    lp = log_softmax(zp)
    p = np.exp(lp)
    if kind == "kl_div":
        return q - p
    mask = (q < p).astype(np.float64)
    S = (mask * q).sum(axis=1, keepdims=True)
    dalpha = q * (mask - S)  # d alpha / d z_q,j
    if kind == "tv":
        return -dalpha
    if kind == "nla":
        alpha = np.minimum(p, q).sum(axis=1, keepdims=True)
        return -dalpha / alpha
    if kind == "lk_hybrid":
        alpha = np.minimum(p, q).sum(axis=1, keepdims=True)
        lam = np.exp(-3.0 * alpha)
        return lam * (q - p) - (1.0 - lam) * dalpha
    if kind == "rkl":
        r = (q * (lq - lp)).sum(axis=1, keepdims=True)
        return q * (lq - lp - r)
    if kind == "jsd":
        a = 0.5 * (lq - np.log(0.5 * (p + q)))
        return q * (a - (q * a).sum(axis=1, keepdims=True))
    raise ValueError(f"unknown loss kind {kind!r}")


# ----------------------------------------------------------------------------------------
# [SD] "Streaming Cross Entropy" / "Backward pass": the chunk loops.
# ----------------------------------------------------------------------------------------
def _row_mask(kind, lab, n, V, ignore_index):
    """Valid rows.  For "ce" a label outside [0, V) other than ignore_index is an error."""
    if lab is None:
        if kind == "ce":
            raise ValueError("ce needs labels")
        return np.ones(n, dtype=bool)
    valid = lab != ignore_index
    if kind == "ce":
        bad = valid & ((lab < 0) | (lab >= V))
        if bad.any():
            raise ValueError("label out of range")
    return valid


def forward(kind, Hq, W, labels=None, Hp=None, ignore_index=-100, chunk_size=512):
    """Streaming forward: loop over token chunks, accumulate the masked loss sum and the
    valid-token count, divide once at the end ([SD] "Streaming Cross Entropy").

    Returns a dict: ``loss`` (normalised mean), ``loss_sum``, ``n_valid``, ``loss_tok``
    [N] (0 on masked rows) and the per-token statistics ``lse_q``, ``lse_p``, ``kl``,
    ``alpha``, ``S`` where the kind defines them.
    """
    Hq = _f64(Hq)
    W = _f64(W)
    n, V = Hq.shape[0], W.shape[0]
    Hp_ = _f64(Hp) if (kind != "ce") else None
    lab = _labels(labels, n)
    valid = _row_mask(kind, lab, n, V, ignore_index)
    keys = ("lse_q", "lse_p", "kl", "alpha", "S", "target")
    res = {k: np.zeros(n) for k in keys}
    res["loss_tok"] = np.zeros(n)
    total_loss = 0.0
    total_weight = 0
    for c0 in range(0, n, max(1, int(chunk_size))):
        c1 = min(n, c0 + max(1, int(chunk_size)))
        zq = logits(Hq[c0:c1], W)
        zp = logits(Hp_[c0:c1], W) if Hp_ is not None else None
        terms = token_terms(kind, zq, zp, None if lab is None else lab[c0:c1])
        v = valid[c0:c1]
        tok = np.where(v, terms["loss"], 0.0)
        res["loss_tok"][c0:c1] = tok
        for k in keys:
            if k in terms:
                res[k][c0:c1] = terms[k]
        total_loss += tok.sum()          # chunk_loss_sum
        total_weight += int(v.sum())     # chunk_weight
    res["target"] = res["target"].astype(np.int64)
    res["loss_sum"] = total_loss
    res["n_valid"] = total_weight
    res["loss"] = total_loss / total_weight if total_weight > 0 else 0.0
    return res


def backward(kind, Hq, W, labels=None, Hp=None, grad_tok=None, ignore_index=-100,
             chunk_size=512):
    """Streaming backward ([SD] "Backward pass"): per chunk, recompute the logits, form
    the per-token loss gradient w.r.t. the logits scaled by g_n, produce the chunk's
    hidden-state gradient dH = dZ W and accumulate dW += dZ^T H.

    ``grad_tok`` [N] is g_n = d(total)/d(loss_n); masked rows get no gradient.  Default:
    the normalised mean (g_n = 1/n_valid).  Returns (dHq [N, d], dW [V, d]) in float64.
    """
    Hq = _f64(Hq)
    W = _f64(W)
    n, V = Hq.shape[0], W.shape[0]
    Hp_ = _f64(Hp) if (kind != "ce") else None
    lab = _labels(labels, n)
    valid = _row_mask(kind, lab, n, V, ignore_index)
    if grad_tok is None:
        nv = int(valid.sum())
        g = np.full(n, 1.0 / nv if nv > 0 else 0.0)
    else:
        g = _f64(grad_tok).reshape(-1)
    g = np.where(valid, g, 0.0)
    dH = np.zeros_like(Hq)
    dW = np.zeros_like(W)
    for c0 in range(0, n, max(1, int(chunk_size))):
        c1 = min(n, c0 + max(1, int(chunk_size)))
        zq = logits(Hq[c0:c1], W)
        zp = logits(Hp_[c0:c1], W) if Hp_ is not None else None
        dz = dlogits(kind, zq, zp, None if lab is None else lab[c0:c1]) * g[c0:c1, None]
        dH[c0:c1] = dz @ W
        dW += dz.T @ Hq[c0:c1]
    return dH, dW


def loss_and_grads(kind, Hq, W, labels=None, Hp=None, ignore_index=-100, chunk_size=512):
    """Normalised mean loss and its gradients w.r.t. H_q and W."""
    f = forward(kind, Hq, W, labels, Hp, ignore_index, chunk_size)
    dH, dW = backward(kind, Hq, W, labels, Hp, None, ignore_index, chunk_size)
    return f["loss"], dH, dW, f


# ----------------------------------------------------------------------------------------
# [SD] memory arithmetic of the LM loss path.
# ----------------------------------------------------------------------------------------
def logits_bytes(batch, seq, vocab, dtype_bytes=4):
    """Bytes of a materialised [batch, seq, vocab] logits tensor."""
    return int(batch) * int(seq) * int(vocab) * int(dtype_bytes)


def chunk_buffer_bytes(chunk, vocab, dtype_bytes=4):
    """Peak bytes of one chunk's logits plus their gradient: chunk x vocab x dtype x 2."""
    return int(chunk) * int(vocab) * int(dtype_bytes) * 2


# ----------------------------------------------------------------------------------------
# [LF] "Weighted Combinations": a weighted sum of several losses; the weights are used as
# given (not normalised) and every term is also reported on its own, before weighting.
# ----------------------------------------------------------------------------------------
def combo_forward(weights, Hq, W, labels=None, Hp=None, ignore_index=-100, chunk_size=512):
    """Weighted combination {kind: weight}.  Every term shares the row mask and the valid
    count; the combined per-token loss is sum_k w_k l_k and the mean divides it by the
    valid count.  Returns the combined results plus ``terms`` = {kind: per-term forward}."""
    terms = {}
    for kind, w in weights.items():
        if kind not in KINDS:
            raise ValueError(f"unknown loss kind {kind!r}")
        terms[kind] = forward(kind, Hq, W, labels, Hp if kind != "ce" else None, ignore_index,
                              chunk_size)
    first = next(iter(terms.values()))
    tok = sum(float(w) * terms[k]["loss_tok"] for k, w in weights.items())
    n_valid = first["n_valid"]
    loss_sum = float(tok.sum())
    return {"loss_tok": tok, "loss_sum": loss_sum, "n_valid": n_valid,
            "loss": loss_sum / n_valid if n_valid > 0 else 0.0, "terms": terms}


def combo_backward(weights, Hq, W, labels=None, Hp=None, grad_tok=None, ignore_index=-100,
                   chunk_size=512):
    """Gradients of the weighted combination: the weighted sum of the terms' gradients."""
    dH = np.zeros(np.shape(Hq))
    dW = np.zeros(np.shape(W))
    for kind, w in weights.items():
        h, g = backward(kind, Hq, W, labels, Hp if kind != "ce" else None, grad_tok,
                        ignore_index, chunk_size)
        dH += float(w) * h
        dW += float(w) * g
    return dH, dW


# ----------------------------------------------------------------------------------------
# Draft-head helpers either side of the path.
# [SD] "Correctness: alignment before chunking": hidden states, targets and masks are
# aligned for the objective first (for draft heads the target shift depends on the head),
# masks applied, and only then split into chunks.
# [FT] "Flatter Tokens are More Valuable for Speculative Draft Model Training": a token's
# flatness is the cosine similarity of the target distribution to the uniform one.
# ----------------------------------------------------------------------------------------
def align_labels(tokens, shift, loss_mask=None, seq_ids=None, ignore_index=-100):
    """Labels for a head that predicts the token ``shift`` positions ahead.

    tokens [B, S] int; loss_mask [B, S] (nonzero = the token may be a target) or None;
    seq_ids [B, S] (packed sequences: position t may only target a token of the same
    sequence) or None.  Returns int64 [B, S]: tokens[b, t + shift] where t + shift < S, the
    target position is unmasked and in the same sequence; ignore_index elsewhere.
    Written as a plain loop over positions."""
    tok = np.asarray(tokens)
    B, S = tok.shape
    out = np.full((B, S), ignore_index, dtype=np.int64)
    for b in range(B):
        for t in range(S):
            u = t + shift
            if u >= S:
                continue
            if loss_mask is not None and not np.asarray(loss_mask)[b, u]:
                continue
            if seq_ids is not None and np.asarray(seq_ids)[b, u] != np.asarray(seq_ids)[b, t]:
                continue
            out[b, t] = tok[b, u]
    return out


def flatness(zp):
    """Cosine similarity of softmax(zp) (per row) to the uniform distribution:
    <p, u> / (||p|| ||u||) with u = 1/V, which equals 1 / (sqrt(V) ||p||_2)."""
    p = np.exp(log_softmax(zp))
    V = p.shape[1]
    u = np.full(V, 1.0 / V)
    return (p @ u) / (np.linalg.norm(p, axis=1) * np.linalg.norm(u))
