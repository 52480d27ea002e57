"""Two small entry points on the GPU: the library's valid-row count (slm_count_valid) and
its kernel-class timing (slm_trace_enable / slm_trace_read).

The count must equal the forward's own n_valid, and the oracle's reading of the mask
("Streaming Cross Entropy": the mean divides by the valid, non-masked tokens).  The trace
must report one launch per GEMM of the launch sequence (forward statistics GEMM, then per
token chunk the logits-gradient, dH and dW GEMMs, or one persistent launch for all three)
with positive device times.
"""

import numpy as np
import pytest
import torch

from lm_head_loss_streaming_b200 import _lib, synthetic
from lm_head_loss_streaming_b200.loss import count_valid, lm_head_loss_bwd, lm_head_loss_fwd

pytestmark = pytest.mark.gpu


def _dev(inp):
    dev = torch.device("cuda", 0)
    return (inp.Hq.to(dev), inp.W.to(dev), None if inp.Hp is None else inp.Hp.to(dev),
            None if inp.labels is None else inp.labels.to(dev))


def test_count_valid_matches_forward_and_mask():
    inp = synthetic.make("ce", 3000, 64, 777, w_std=0.05, ignore_frac=0.15, seed=81)
    labels = inp.labels.clone()
    valid_rows = np.flatnonzero(labels.numpy() != inp.ignore_index)
    labels[int(valid_rows[0])] = inp.V          # out of range: masked for CE
    labels[int(valid_rows[1])] = -7             # out of range: masked for CE
    Hq, W, _, _ = _dev(inp)
    lab = labels.to(Hq.device)
    lab_np = labels.numpy()
    in_range = (lab_np >= 0) & (lab_np < inp.V)
    n_ce = int(((lab_np != inp.ignore_index) & in_range).sum())
    assert count_valid("ce", lab, inp.N, inp.V, inp.ignore_index).item() == n_ce
    f = lm_head_loss_fwd("ce", Hq, W, lab, None, inp.ignore_index)
    assert f.n_valid.item() == n_ce
    # Distribution kinds: the labels are a row mask only (no range check), or absent.
    n_mask = int((lab_np != inp.ignore_index).sum())
    assert count_valid("kl_div", lab, inp.N, inp.V, inp.ignore_index).item() == n_mask
    assert count_valid("kl_div", None, inp.N, inp.V, inp.ignore_index).item() == inp.N
    assert count_valid("tv", None, 0, inp.V, inp.ignore_index).item() == 0


@pytest.mark.parametrize("kind,mode,launches", [
    ("kl_div", 0, {"fwd_gemm": 1, "dz_gemm": 3, "dh_gemm": 3, "dw_gemm": 3, "row": 2}),
    ("tv", 0, {"fwd_gemm": 1, "pass2_gemm": 1, "dz_gemm": 3, "dh_gemm": 3, "dw_gemm": 3,
               "row": 3}),
    ("kl_div", 1, {"fwd_gemm": 1, "bwd_fused": 3, "row": 2}),
    ("ce", 1, {"fwd_gemm": 1, "bwd_fused": 3, "row": 2})])
def test_trace_reports_every_gemm_launch(kind, mode, launches):
    inp = synthetic.make(kind, 700, 128, 3000, w_std=0.05, seed=82)
    Hq, W, Hp, lab = _dev(inp)
    torch.cuda.synchronize()
    _lib.check(_lib.slm_trace_read()[0])
    prev = _lib.slm_set_backward_mode(mode)
    _lib.slm_trace_enable(True)
    try:
        f = lm_head_loss_fwd(kind, Hq, W, lab, Hp, inp.ignore_index, chunk_tokens=256)
        lm_head_loss_bwd(f, Hq, W, lab, Hp, inp.ignore_index, chunk_tokens=256)
    finally:
        _lib.slm_trace_enable(False)
        _lib.slm_set_backward_mode(prev)
    st, got = _lib.slm_trace_read()
    assert st == 0
    for name, (ms, n) in got.items():
        assert n == launches.get(name, 0), (name, n)
        if n:
            assert ms > 0.0, name
    # Read clears the record; tracing is off again.
    lm_head_loss_fwd(kind, Hq, W, lab, Hp, inp.ignore_index)
    st, got = _lib.slm_trace_read()
    assert st == 0 and all(n == 0 for _, n in got.values())
