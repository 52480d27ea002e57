"""Launch schedule and execution modes of the GEMMs: none may change a result.

  * The CTA pairs' loose lockstep only shapes performance: with every wait giving up at
    once (test hook slm_debug_set(2, ...)), loss and gradients are bit for bit the same.
  * Two calls running at once on two streams (their lockstep records carry different
    launch tags) give what they give one after the other.
  * A forward + backward captured into a CUDA graph and replayed gives what the eager calls
    give ("Backward pass": the streamed step is a fixed sequence of launches on one stream,
    with no allocation or host synchronisation inside).
"""

import pytest
import torch

from lm_head_loss_streaming_b200 import _lib, synthetic
from lm_head_loss_streaming_b200.loss import lm_head_loss_bwd, lm_head_loss_fwd

pytestmark = pytest.mark.gpu


def _dev(inp):
    dev = torch.device("cuda", 0)
    return (inp.Hq.to(dev), inp.W.to(dev), None if inp.Hp is None else inp.Hp.to(dev),
            None if inp.labels is None else inp.labels.to(dev))


def _step(kind, Hq, W, lab, Hp, chunk=0):
    f = lm_head_loss_fwd(kind, Hq, W, lab, Hp, chunk_tokens=chunk)
    dH, dW = lm_head_loss_bwd(f, Hq, W, lab, Hp, chunk_tokens=chunk)
    return f, dH, dW


# Big enough for every pair to hold several vocabulary runs, so that pairs do wait.
SHAPE = dict(N=4096, d=512, V=40000)


@pytest.mark.parametrize("kind", ["kl_div", "tv"])
def test_lockstep_giving_up_changes_nothing(kind):
    inp = synthetic.make(kind, SHAPE["N"], SHAPE["d"], SHAPE["V"], w_std=0.05, seed=81)
    Hq, W, Hp, lab = _dev(inp)
    f0, h0, w0 = _step(kind, Hq, W, lab, Hp)
    assert _lib.slm_debug_set(2, 0) == 0
    try:
        f1, h1, w1 = _step(kind, Hq, W, lab, Hp)
        torch.cuda.synchronize()
    finally:
        assert _lib.slm_debug_set(0, 0) == 0
    assert _lib.slm_device_status(f1.workspace.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream) == 0
    assert torch.equal(f0.loss_tok, f1.loss_tok) and torch.equal(f0.stats, f1.stats)
    assert torch.equal(h0, h1) and torch.equal(w0, w1)


def test_two_streams_at_once_match_one_after_the_other():
    a = synthetic.make("kl_div", SHAPE["N"], SHAPE["d"], SHAPE["V"], w_std=0.05, seed=82)
    b = synthetic.make("ce", SHAPE["N"], SHAPE["d"], SHAPE["V"], w_std=0.05,
                       ignore_frac=0.1, seed=83)
    A, B = _dev(a), _dev(b)
    ref_a = _step("kl_div", A[0], A[1], A[3], A[2])
    ref_b = _step("ce", B[0], B[1], B[3], B[2])
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    s1.wait_stream(torch.cuda.current_stream())
    s2.wait_stream(torch.cuda.current_stream())
    for _ in range(3):
        with torch.cuda.stream(s1):
            got_a = _step("kl_div", A[0], A[1], A[3], A[2])
        with torch.cuda.stream(s2):
            got_b = _step("ce", B[0], B[1], B[3], B[2])
        torch.cuda.synchronize()
        for ref, got in ((ref_a, got_a), (ref_b, got_b)):
            assert torch.equal(ref[0].loss_tok, got[0].loss_tok)
            assert torch.equal(ref[1], got[1]) and torch.equal(ref[2], got[2])


@pytest.mark.parametrize("kind", ["ce", "kl_div", "nla"])
def test_cuda_graph_replay_matches_eager(kind):
    inp = synthetic.make(kind, 1024, 256, 9000, w_std=0.05, ignore_frac=0.1, seed=84)
    Hq, W, Hp, lab = _dev(inp)
    ref = _step(kind, Hq, W, lab, Hp, chunk=512)   # also the warm-up before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        out = _step(kind, Hq, W, lab, Hp, chunk=512)
    for _ in range(2):
        out[1].zero_()
        out[2].zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(ref[0].loss_tok, out[0].loss_tok)
        assert torch.equal(ref[0].loss_sum, out[0].loss_sum)
        assert torch.equal(ref[1], out[1]) and torch.equal(ref[2], out[2])
    # New inputs copied into the captured buffers flow through the replay.
    inp2 = synthetic.make(kind, 1024, 256, 9000, w_std=0.05, ignore_frac=0.1, seed=85)
    H2, _, Hp2, lab2 = _dev(inp2)
    Hq.copy_(H2)
    if Hp is not None:
        Hp.copy_(Hp2)
    if lab is not None:
        lab.copy_(lab2)
    ref2 = _step(kind, Hq, W, lab, Hp, chunk=512)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(ref2[0].loss_tok, out[0].loss_tok)
    assert torch.equal(ref2[1], out[1]) and torch.equal(ref2[2], out[2])
