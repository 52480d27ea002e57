"""The device-side failure path: a bounded pipeline wait that runs out.

The test hook slm_debug_set(1, ...) makes the epilogue withhold its first accumulator
release, so the MMA issuer's wait for it runs out.  The kernel must record
SLM_ERR_TIMEOUT, unwind (its own copies and MMAs land, its tensor memory is freed) and
return; the CUDA context must stay usable, which the follow-up call checks against the
oracle.  No GPU fault, trap or hang is involved: every wait in the kernel is bounded.
"""

import numpy as np
import pytest
import torch

from lm_head_loss_streaming_b200 import _lib, synthetic
from parity_util import gpu_fwd_bwd, oracle_fwd_bwd, assert_loss_close

pytestmark = pytest.mark.gpu


# CE: the forward tile releases its accumulator in two sub-tiles (the hook withholds the
# first); kl_div: the two-operand tile releases it at once.
@pytest.mark.parametrize("kind", ["ce", "kl_div"])
def test_wait_runs_out_reports_timeout_and_context_survives(kind):
    from lm_head_loss_streaming_b200.loss import device_status, lm_head_loss_fwd
    inp = synthetic.make(kind, 512, 256, 4096, w_std=0.05, ignore_frac=0.1, seed=31)
    dev = torch.device("cuda", 0)
    Hq, W, lab = inp.Hq.to(dev), inp.W.to(dev), inp.labels.to(dev)
    Hp = inp.Hp.to(dev) if inp.Hp is not None else None
    assert _lib.slm_debug_set(1, 100_000_000) == 0   # ~0.05-0.1 s per wait
    try:
        fwd = lm_head_loss_fwd(kind, Hq, W, lab, Hp, inp.ignore_index)
        st = device_status(fwd)
    finally:
        assert _lib.slm_debug_set(0, 0) == 0
    assert st == 7, _lib.status_string(st)   # SLM_ERR_TIMEOUT
    # The context is usable and the next call is correct.
    g = gpu_fwd_bwd(inp, kind)
    assert g["st_fwd"] == 0 and g["st_bwd"] == 0
    r = oracle_fwd_bwd(inp, kind)
    assert_loss_close(g["loss_tok"], r["loss_tok"], g["loss_mean"], r["loss"],
                      f"{kind} after timeout")
