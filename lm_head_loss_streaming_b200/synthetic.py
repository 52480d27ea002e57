"""Seeded synthetic inputs for the streaming LM-head loss.

This module only draws random numbers: it holds none of the loss arithmetic.  Both the
CUDA path (tests, benchmark) and the float64 oracle (tests) read their inputs from here.

Recipe (all draws fp32 from a seeded ``torch.Generator``, rounded to bf16 with
round-to-nearest-even by ``.to(torch.bfloat16)``):

  * W  ~ N(0, w_std^2)                      [V, d]
  * H_p ~ N(0, 1)                            [N, d]   (the target's hidden states)
  * draft H_q:  "add": H_q = H_p + s * eps;  "mix": H_q = a * H_p + b * eps;  "none": H_q = H_p
    with eps ~ N(0, 1), the combination formed in fp32 before rounding.
  * labels uniform int32 in [0, V); exactly round(ignore_frac * N) rows, chosen by a seeded
    permutation, are set to ``ignore_index``.

The named workloads are the shapes of the LM heads of Llama-3.2-1B (d=2048), Llama-3.1-8B
(d=4096) and Llama-3.1-405B (d=16384), all with a 128256-entry vocabulary.  No weights or
datasets are used: every value is synthetic.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

IGNORE_INDEX = -100

WORKLOADS = {
    # Tiny hard-label CE: N=256, d=256, V=4096, 10% ignored.
    "tiny_ce": dict(kinds=("ce",), N=256, d=256, V=4096, w_std=0.02, ignore_frac=0.10,
                    draft=None),
    # Llama-3.2-1B-shaped CE: N=8192, d=2048, V=128256, 5% ignored.
    "llama1b_ce": dict(kinds=("ce",), N=8192, d=2048, V=128256, w_std=0.02,
                       ignore_frac=0.05, draft=None),
    # Llama-3.1-8B-shaped forward KL(p||q): correlated draft H_q = H_p + 0.5 eps.
    "llama8b_kl": dict(kinds=("kl_div",), N=16384, d=4096, V=128256, w_std=0.02,
                       ignore_frac=0.0, draft=("add", 0.5)),
    # alpha-based losses (tv, nla, lk_hybrid): H_q = 0.8 H_p + 0.6 eps.
    "alpha_losses": dict(kinds=("tv", "nla", "lk_hybrid"), N=32768, d=4096, V=128256,
                         w_std=0.02, ignore_frac=0.0, draft=("mix", 0.8, 0.6)),
    # Llama-3.1-405B-shaped CE at scale: N=65536 (2 x 32768), d=16384, 10% ignored.
    "llama405b_ce": dict(kinds=("ce",), N=65536, d=16384, V=128256, w_std=0.01,
                         ignore_frac=0.10, draft=None),
}

# Row slab used to bound the fp32 temporaries of large draws.
_SLAB_ELEMS = 1 << 26


@dataclass
class Inputs:
    kind: str
    Hq: torch.Tensor
    W: torch.Tensor
    labels: torch.Tensor | None
    Hp: torch.Tensor | None
    ignore_index: int = IGNORE_INDEX
    meta: dict = field(default_factory=dict)

    @property
    def N(self):
        return self.Hq.shape[0]

    @property
    def d(self):
        return self.Hq.shape[1]

    @property
    def V(self):
        return self.W.shape[0]


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal_bf16(rows, cols, std, g, device):
    """[rows, cols] N(0, std^2) drawn in fp32 slab by slab, rounded to bf16."""
    out = torch.empty(rows, cols, dtype=torch.bfloat16, device=device)
    slab = max(1, _SLAB_ELEMS // max(1, cols))
    for r0 in range(0, rows, slab):
        r1 = min(rows, r0 + slab)
        x = torch.randn(r1 - r0, cols, generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        out[r0:r1].copy_(x)
    return out


def _draft_bf16(Hp, draft, g, device):
    """Draft hidden states from the target's, combined in fp32 slab by slab."""
    rows, cols = Hp.shape
    out = torch.empty_like(Hp)
    slab = max(1, _SLAB_ELEMS // max(1, cols))
    for r0 in range(0, rows, slab):
        r1 = min(rows, r0 + slab)
        eps = torch.randn(r1 - r0, cols, generator=g, device=device, dtype=torch.float32)
        hp = Hp[r0:r1].float()
        if draft[0] == "add":
            x = hp + draft[1] * eps
        elif draft[0] == "mix":
            x = draft[1] * hp + draft[2] * eps
        else:
            raise ValueError(f"unknown draft recipe {draft!r}")
        out[r0:r1].copy_(x)
    return out


def _labels(N, V, ignore_frac, g, device, ignore_index):
    lab = torch.randint(0, V, (N,), generator=g, device=device, dtype=torch.int64)
    n_ign = int(round(ignore_frac * N))
    if n_ign > 0:
        perm = torch.randperm(N, generator=g, device=device)
        lab[perm[:n_ign]] = ignore_index
    return lab.to(torch.int32)


def make(kind, N, d, V, *, w_std=0.02, h_std=1.0, ignore_frac=0.0, draft=None,
         with_labels=None, seed=0, device="cpu", ignore_index=IGNORE_INDEX,
         w_scale=None) -> Inputs:
    """Draw one input set.

    ``kind`` selects which tensors are produced: "ce" gets (H, W, labels); the
    distribution kinds get (H_q, H_p, W) and, when ``with_labels`` or ``ignore_frac > 0``,
    a label row mask.  ``draft`` defaults to ("add", 0.5) for the distribution kinds.
    ``w_scale`` multiplies W after rounding (used for overflow-safety cases).
    """
    g = _gen(seed, device)
    W = _normal_bf16(V, d, w_std, g, device)
    if w_scale is not None:
        W = (W.float() * w_scale).to(torch.bfloat16)
    H = _normal_bf16(N, d, h_std, g, device)
    if kind == "ce":
        labels = _labels(N, V, ignore_frac, g, device, ignore_index)
        return Inputs(kind, H, W, labels, None, ignore_index,
                      dict(N=N, d=d, V=V, seed=seed, w_std=w_std, ignore_frac=ignore_frac))
    if draft is None:
        draft = ("add", 0.5)
    Hp = H
    Hq = Hp.clone() if draft[0] == "none" else _draft_bf16(Hp, draft, g, device)
    labels = None
    if with_labels or ignore_frac > 0:
        labels = _labels(N, V, ignore_frac, g, device, ignore_index)
    return Inputs(kind, Hq, W, labels, Hp, ignore_index,
                  dict(N=N, d=d, V=V, seed=seed, w_std=w_std, ignore_frac=ignore_frac,
                       draft=list(draft)))


def workload(name, *, kind=None, seed=0, device="cpu", N=None) -> Inputs:
    """Draw the named workload (optionally with fewer token rows ``N``).

    ``kind`` defaults to the workload's first kind.  Any other kind draws the workload's
    shapes and distributions: hard-label CE adds uniform labels; the distribution kinds
    draw a draft with the workload's recipe (H_q = H_p + 0.5 eps when it has none)."""
    cfg = WORKLOADS[name]
    k = kind or cfg["kinds"][0]
    inp = make(k, N or cfg["N"], cfg["d"], cfg["V"], w_std=cfg["w_std"],
               ignore_frac=cfg["ignore_frac"], draft=cfg["draft"], seed=seed,
               device=device)
    inp.meta["workload"] = name
    return inp
