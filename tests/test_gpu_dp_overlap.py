"""The data-parallel backward with the dW reduction overlapped ("Training speculative
decoders: removing the logits and attention bottlenecks", "Streaming Cross Entropy": the
streaming loss composes with data parallelism).

slm_loss_bwd_overlap must give the same dH and dW as slm_loss_bwd, bit for bit (it only
reorders the last chunk's dH and dW GEMMs and runs that dH GEMM on fewer SMs), and must
record its event once dW is final.  The data-parallel step over NCCL with the overlap must
equal the one without it, and both the oracle; one GPU runs it as a one-rank NCCL group.
"""

import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from lm_head_loss_streaming_b200 import _lib, dp, synthetic
from lm_head_loss_streaming_b200.loss import lm_head_loss_bwd, lm_head_loss_fwd
from parity_util import assert_grad_close, tie_slack

pytestmark = pytest.mark.gpu


def _dev(inp):
    dev = torch.device("cuda", 0)
    return (inp.Hq.to(dev), inp.W.to(dev), None if inp.Hp is None else inp.Hp.to(dev),
            None if inp.labels is None else inp.labels.to(dev))


@pytest.mark.parametrize("kind,chunk,reserve", [("ce", 128, 8), ("kl_div", 200, 0),
                                                ("tv", 256, 32), ("ce_argmax_p", 0, 128)])
def test_overlap_backward_is_bitwise_the_plain_backward(kind, chunk, reserve):
    inp = synthetic.make(kind, 600, 128, 2000, w_std=0.05, ignore_frac=0.1, seed=71,
                         with_labels=kind != "ce_argmax_p")
    Hq, W, Hp, lab = _dev(inp)
    f = lm_head_loss_fwd(kind, Hq, W, lab, Hp, inp.ignore_index, chunk_tokens=chunk)
    dH0, dW0 = lm_head_loss_bwd(f, Hq, W, lab, Hp, inp.ignore_index, chunk_tokens=chunk)
    ev = torch.cuda.Event()
    dH1, dW1 = lm_head_loss_bwd(f, Hq, W, lab, Hp, inp.ignore_index, chunk_tokens=chunk,
                                dw_ready=ev, reserve_sms=reserve)
    torch.cuda.synchronize()
    assert ev.query()
    assert _lib.slm_device_status(f.workspace.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream) == 0
    assert torch.equal(dH0, dH1)
    assert torch.equal(dW0, dW1)


def test_overlap_backward_accumulates_and_handles_empty_batch():
    inp = synthetic.make("kl_div", 300, 64, 1000, w_std=0.05, seed=72)
    Hq, W, Hp, lab = _dev(inp)
    f = lm_head_loss_fwd("kl_div", Hq, W, lab, Hp)
    base = torch.randn(W.shape, device=W.device)
    dW0 = base.clone()
    lm_head_loss_bwd(f, Hq, W, lab, Hp, dW=dW0, accumulate_dW=True, chunk_tokens=128)
    dW1 = base.clone()
    lm_head_loss_bwd(f, Hq, W, lab, Hp, dW=dW1, accumulate_dW=True, chunk_tokens=128,
                     dw_ready=torch.cuda.Event(), reserve_sms=16)
    assert torch.equal(dW0, dW1)
    # No rows: dW is zeroed and the event still recorded.
    e = synthetic.make("ce", 0, 64, 1000, seed=73)
    Hq, W, _, lab = _dev(e)
    f = lm_head_loss_fwd("ce", Hq, W, lab)
    ev = torch.cuda.Event()
    dH, dW = lm_head_loss_bwd(f, Hq, W, lab, dw_ready=ev, reserve_sms=8)
    torch.cuda.synchronize()
    assert ev.query() and dW.abs().max().item() == 0.0


def test_overlap_rejects_reserve_outside_range():
    inp = synthetic.make("ce", 64, 64, 500, seed=74)
    Hq, W, _, lab = _dev(inp)
    f = lm_head_loss_fwd("ce", Hq, W, lab)
    for bad in (-1, 129):
        with pytest.raises(_lib.SLMError):
            lm_head_loss_bwd(f, Hq, W, lab, reserve_sms=bad)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("kind", ["ce", "kl_div"])
def test_nccl_step_with_overlap_equals_plain_step_and_oracle(kind):
    inp = synthetic.make(kind, 700, 128, 3000, w_std=0.05, ignore_frac=0.1, seed=75)
    Hq, W, Hp, lab = _dev(inp)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        runs = []
        for overlap in (False, True):
            r = dp.cuda_step(kind, Hq, W, lab, Hp, inp.ignore_index, chunk_tokens=256,
                             overlap=overlap, reserve_sms=8)
            torch.cuda.synchronize()
            runs.append((r.loss_mean.item(), r.n_valid.item(), r.dH.clone(), r.dW.clone()))
    finally:
        dist.destroy_process_group()
    (l0, n0, h0, w0), (l1, n1, h1, w1) = runs
    assert l0 == l1 and n0 == n1
    assert torch.equal(h0, h1) and torch.equal(w0, w1)
    ref = oracle.forward(kind, inp.Hq, inp.W, inp.labels, inp.Hp, inp.ignore_index)
    assert n0 == ref["n_valid"]
    assert abs(l0 - ref["loss_sum"] / ref["n_valid"]) <= 2e-3 * abs(ref["loss_sum"] / ref["n_valid"])
    valid = inp.labels.numpy() != inp.ignore_index
    gt = np.where(valid, 1.0 / ref["n_valid"], 0.0)
    rh, rw = oracle.backward(kind, inp.Hq, inp.W, inp.labels, inp.Hp, gt, inp.ignore_index)
    sh, sw = tie_slack(inp, kind)
    assert_grad_close(h1.double().cpu().numpy(), rh, "dp dH", sh)
    assert_grad_close(w1.double().cpu().numpy(), rw, "dp dW", sw)


@pytest.mark.parametrize("kind", ["ce", "kl_div"])
def test_nccl_fused_step_matches_oracle(kind):
    """The data-parallel step over the fused single call (valid counts summed first and
    passed in as the gradient's scale), as a one-rank NCCL group."""
    inp = synthetic.make(kind, 700, 128, 3000, w_std=0.05, ignore_frac=0.1, seed=76)
    Hq, W, Hp, lab = _dev(inp)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        r = dp.cuda_step_fused(kind, Hq, W, lab, Hp, inp.ignore_index, chunk_tokens=256)
        torch.cuda.synchronize()
        loss, n, h, w = r.loss_mean.item(), r.n_valid.item(), r.dH.clone(), r.dW.clone()
    finally:
        dist.destroy_process_group()
    ref = oracle.forward(kind, inp.Hq, inp.W, inp.labels, inp.Hp, inp.ignore_index)
    assert n == ref["n_valid"]
    mean = ref["loss_sum"] / ref["n_valid"]
    assert abs(loss - mean) <= 2e-3 * abs(mean)
    valid = inp.labels.numpy() != inp.ignore_index
    gt = np.where(valid, 1.0 / ref["n_valid"], 0.0)
    rh, rw = oracle.backward(kind, inp.Hq, inp.W, inp.labels, inp.Hp, gt, inp.ignore_index)
    assert_grad_close(h.double().cpu().numpy(), rh, "dp fused dH")
    assert_grad_close(w.double().cpu().numpy(), rw, "dp fused dW")


@pytest.mark.parametrize("fused", [False, True])
def test_nccl_step_with_dW_sharded_by_vocabulary_rows(fused):
    """dW reduce-scattered by vocabulary rows (FSDP-style) over a one-rank NCCL group: the
    single shard is the whole summed dW, equal bit for bit to the all-reduced one."""
    inp = synthetic.make("kl_div", 500, 128, 3001, w_std=0.05, ignore_frac=0.1, seed=77,
                         with_labels=True)
    Hq, W, Hp, lab = _dev(inp)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        step = dp.cuda_step_fused if fused else dp.cuda_step
        a = step("kl_div", Hq, W, lab, Hp, inp.ignore_index, chunk_tokens=256)
        wa = a.dW.clone()
        b = step("kl_div", Hq, W, lab, Hp, inp.ignore_index, chunk_tokens=256, shard_dW=True)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert b.dW_rows == (0, inp.V) and b.dW.shape == wa.shape
    assert torch.equal(b.dW, wa)
    assert a.n_valid.item() == b.n_valid.item()


def test_fused_dp_count_leaves_out_rows_the_kernels_mask():
    """The fused data-parallel step takes its valid count from the library: a CE label
    outside [0, V) is masked by the kernels and left out of the count, so the mean and the
    gradient agree with the oracle on the remaining rows."""
    inp = synthetic.make("ce", 400, 128, 2000, w_std=0.05, ignore_frac=0.1, seed=78)
    labels = inp.labels.clone()
    bad = int(np.flatnonzero(labels.numpy() != inp.ignore_index)[3])
    labels[bad] = inp.V + 5
    Hq, W, _, _ = _dev(inp)
    lab = labels.to(Hq.device)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        ws = torch.empty(_lib.slm_fused_workspace_bytes(_lib.SLM_CE, inp.N, inp.d, inp.V, 256),
                         dtype=torch.uint8, device=Hq.device)
        r = dp.cuda_step_fused("ce", Hq, W, lab, None, inp.ignore_index, chunk_tokens=256,
                               workspace=ws)
        torch.cuda.synchronize()
        n, loss = r.n_valid.item(), r.loss_mean.item()
        w = r.dW.clone()
        st = _lib.slm_device_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    finally:
        dist.destroy_process_group()
    assert st == 6  # SLM_ERR_LABEL_RANGE
    keep = labels.numpy().copy()
    keep[bad] = inp.ignore_index      # the oracle's reading: that row is masked
    ref = oracle.forward("ce", inp.Hq, inp.W, torch.from_numpy(keep), None, inp.ignore_index)
    assert n == ref["n_valid"]
    assert abs(loss - ref["loss"]) <= 2e-3 * abs(ref["loss"])
    rh, rw = oracle.backward("ce", inp.Hq, inp.W, torch.from_numpy(keep), None, None,
                             inp.ignore_index)
    assert_grad_close(w.double().cpu().numpy(), rw, "dp fused dW, masked label")
