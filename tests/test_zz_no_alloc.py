"""The allocation-free forward entry point, slm_loss_fwd_noalloc, called through the C ABI.

It is meant for callers that cannot allocate device memory: hosts with no allocator of
their own to hand out a workspace, runtimes whose enqueue path must not call cudaMalloc,
and processes held to a fixed memory budget.  Its scratch is a fixed device array inside
the library, shared by every call, so these tests check two calls in a row (and a third
that repeats the first) against the regular workspace-based slm_loss_fwd, within the
parity tests' loss tolerance, and against the float64 oracle; that a call which raises a
device flag reports it and the next clean call on the same array does not; and that sizes
beyond the array are refused.
"""

import numpy as np
import pytest
import torch

import oracle
from lm_head_loss_streaming_b200 import _lib, synthetic
from lm_head_loss_streaming_b200.loss import lm_head_loss_fwd

pytestmark = pytest.mark.gpu

LOSS_RTOL = 2e-3


def _on_gpu(inp):
    dev = torch.device("cuda", 0)
    return (inp.Hq.to(dev), inp.W.to(dev),
            inp.Hp.to(dev) if inp.Hp is not None else None,
            inp.labels.to(dev) if inp.labels is not None else None)


def _noalloc_fwd(inp):
    Hq, W, Hp, lab = _on_gpu(inp)
    k = _lib.KIND[inp.kind]
    dev = Hq.device
    N, d, V = inp.N, inp.d, inp.V
    loss_tok = torch.full((N,), float("nan"), device=dev)
    alpha = torch.full((N,), float("nan"), device=dev) if k in _lib.ALPHA_KINDS else None
    loss_sum = torch.zeros(1, dtype=torch.float64, device=dev)
    n_valid = torch.zeros(1, dtype=torch.int64, device=dev)
    loss_mean = torch.zeros(1, device=dev)
    stats = torch.full((_lib.slm_stats_floats(k), N), float("nan"), device=dev)
    flags = torch.full((1,), -1, dtype=torch.int32, device=dev)
    ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    st = _lib.slm_loss_fwd_noalloc(k, ptr(Hq), ptr(Hp), ptr(W), ptr(lab), inp.ignore_index,
                                   N, d, V, ptr(loss_tok), ptr(alpha), ptr(loss_sum),
                                   ptr(n_valid), ptr(loss_mean), ptr(stats), ptr(flags),
                                   torch.cuda.current_stream().cuda_stream)
    assert st == _lib.SLM_OK, _lib.status_string(st)
    torch.cuda.synchronize()
    return dict(loss_tok=loss_tok.double().cpu().numpy(), loss_sum=loss_sum.item(),
                n_valid=n_valid.item(), loss_mean=loss_mean.item(),
                stats=stats.double().cpu().numpy(), flags=int(flags.item()))


def _workspace_fwd(inp):
    Hq, W, Hp, lab = _on_gpu(inp)
    r = lm_head_loss_fwd(inp.kind, Hq, W, lab, Hp, inp.ignore_index)
    torch.cuda.synchronize()
    return dict(loss_tok=r.loss_tok.double().cpu().numpy(), loss_sum=r.loss_sum.item(),
                n_valid=r.n_valid.item(), loss_mean=r.loss_mean.item(),
                stats=r.stats.double().cpu().numpy())


def _assert_same(got, ref):
    assert got["flags"] == 0
    assert got["n_valid"] == ref["n_valid"]
    scale = max(np.abs(ref["loss_tok"]).max(), 1e-2)
    assert np.abs(got["loss_tok"] - ref["loss_tok"]).max() <= LOSS_RTOL * scale
    assert abs(got["loss_mean"] - ref["loss_mean"]) <= LOSS_RTOL * max(abs(ref["loss_mean"]), 1e-2)
    assert abs(got["loss_sum"] - ref["loss_sum"]) <= LOSS_RTOL * max(abs(ref["loss_sum"]), 1e-2)
    assert np.allclose(got["stats"], ref["stats"], rtol=1e-5, atol=1e-4)


def test_noalloc_forward_matches_workspace_forward_two_calls_in_a_row():
    first = synthetic.make("ce", 700, 256, 5000, w_std=0.05, ignore_frac=0.1, seed=21)
    second = synthetic.make("kl_div", 513, 128, 3001, w_std=0.05, seed=22)
    ref1 = _workspace_fwd(first)
    ref2 = _workspace_fwd(second)
    got1 = _noalloc_fwd(first)
    _assert_same(got1, ref1)
    got2 = _noalloc_fwd(second)
    _assert_same(got2, ref2)
    # The shared scratch keeps the previous call's contents; a repeat of the first call
    # must not see them.
    again = _noalloc_fwd(first)
    _assert_same(again, ref1)
    assert np.array_equal(again["loss_tok"], got1["loss_tok"])


def _assert_oracle(got, inp):
    """Loss and kept statistics against the float64 oracle (the parity tolerance)."""
    ref = oracle.forward(inp.kind, inp.Hq, inp.W, inp.labels, inp.Hp, inp.ignore_index)
    assert got["n_valid"] == ref["n_valid"]
    scale = max(np.abs(ref["loss_tok"]).max(), 1e-2)
    assert np.abs(got["loss_tok"] - ref["loss_tok"]).max() <= LOSS_RTOL * scale
    assert abs(got["loss_mean"] - ref["loss"]) <= LOSS_RTOL * max(abs(ref["loss"]), 1e-2)
    # stats[0] = L_q for every kind; stats[1] = L_p for the target kinds.
    assert np.abs(got["stats"][0] - ref["lse_q"]).max() <= 1e-4 * max(np.abs(ref["lse_q"]).max(), 1.0)
    if inp.kind != "ce":
        assert np.abs(got["stats"][1] - ref["lse_p"]).max() <= 1e-4 * max(np.abs(ref["lse_p"]).max(), 1.0)


def test_noalloc_forward_matches_oracle():
    for inp in (synthetic.make("ce", 700, 256, 5000, w_std=0.05, ignore_frac=0.1, seed=21),
                synthetic.make("kl_div", 513, 128, 3001, w_std=0.05, seed=22)):
        _assert_oracle(_noalloc_fwd(inp), inp)


def test_noalloc_flag_then_clean_call():
    # One CE label equal to V is out of range: the kernels mask the row and set bit 1 of the
    # status word, which this call copies out of the shared array.  A clean call on the same
    # array right after must start from a cleared word and report 0.
    clean = synthetic.make("ce", 300, 128, 2000, w_std=0.05, ignore_frac=0.1, seed=24)
    bad_labels = clean.labels.clone()
    row = int(np.flatnonzero(bad_labels.numpy() != clean.ignore_index)[0])
    bad_labels[row] = clean.V
    bad = synthetic.Inputs("ce", clean.Hq, clean.W, bad_labels, None, clean.ignore_index,
                           dict(clean.meta))
    got_bad = _noalloc_fwd(bad)
    assert got_bad["flags"] == 1
    assert got_bad["loss_tok"][row] == 0.0
    got_clean = _noalloc_fwd(clean)
    assert got_clean["flags"] == 0
    _assert_same(got_clean, _workspace_fwd(clean))


def test_noalloc_alpha_kind():
    inp = synthetic.make("lk_hybrid", 300, 128, 2000, w_std=0.05, seed=23)
    _assert_same(_noalloc_fwd(inp), _workspace_fwd(inp))


def test_noalloc_refuses_sizes_beyond_its_scratch():
    # KL at V = 128256 needs ~1.26 KB of forward scratch per row: 100000 rows do not fit.
    fake = 1 << 20  # aligned, never dereferenced: the call returns before enqueuing work
    st = _lib.slm_loss_fwd_noalloc(_lib.SLM_KL, fake, fake, fake, None, -100, 100000, 8,
                                   128256, None, None, fake, fake, None, fake, None,
                                   torch.cuda.current_stream().cuda_stream)
    assert st == 5  # SLM_ERR_WORKSPACE
    assert _lib.slm_loss_fwd_noalloc(9, None, None, None, None, -100, 1, 8, 8, None, None,
                                     None, None, None, None, None, None) == 4  # SLM_ERR_KIND
    # A valid kind with an invalid shape (d not a multiple of 8) is a shape error, for
    # every kind.
    for k in range(8):
        assert _lib.slm_loss_fwd_noalloc(k, None, None, None, None, -100, 1, 12, 8, None,
                                         None, None, None, None, None, None, None) == 2
