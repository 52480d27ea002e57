"""Double-buffered host-to-device staging (lm_head_loss_streaming_b200.staging).

Every step must see its own batch: the copy of step k+1, which overlaps step k, may not
overwrite the buffers step k is still reading, and step k may not start before its own copy
has landed.  Checked with batches that differ per step and a deliberately long compute per
step, and end to end through the loss.
"""

import pytest
import torch

from lm_head_loss_streaming_b200 import synthetic
from lm_head_loss_streaming_b200.loss import lm_head_loss_fwd
from lm_head_loss_streaming_b200.staging import InputStager

pytestmark = pytest.mark.gpu


def test_each_step_sees_its_own_batch():
    dev = torch.device("cuda", 0)
    n = 1 << 22
    batches = [{"x": torch.full((n,), float(k + 1)).pin_memory(),
                "y": torch.arange(k, k + 64, dtype=torch.int32).pin_memory()}
               for k in range(6)]
    stager = InputStager({"x": torch.empty(n, device=dev),
                          "y": torch.empty(64, dtype=torch.int32, device=dev)})
    slow = torch.randn(2048, 2048, device=dev)
    sums, firsts = [], []
    slot = stager.put(batches[0])
    for k in range(len(batches)):
        nxt = stager.put(batches[k + 1]) if k + 1 < len(batches) else None
        b = stager.get(slot)
        for _ in range(20):          # keep the compute stream busy while the next copy runs
            slow = torch.tanh(slow @ slow)
        sums.append(b["x"].sum())
        firsts.append(b["y"][0].clone())
        stager.done(slot)
        slot = nxt
    torch.cuda.synchronize()
    for k in range(len(batches)):
        assert sums[k].item() == float(k + 1) * n
        assert firsts[k].item() == k


def test_loss_through_staged_inputs_matches_direct():
    dev = torch.device("cuda", 0)
    inp = synthetic.make("kl_div", 600, 128, 3000, w_std=0.05, seed=91)
    W = inp.W.to(dev)
    ref = lm_head_loss_fwd("kl_div", inp.Hq.to(dev), W, None, inp.Hp.to(dev))
    host = {"Hq": inp.Hq.pin_memory(), "Hp": inp.Hp.pin_memory()}
    stager = InputStager({"Hq": ref.stats.new_empty(inp.Hq.shape, dtype=torch.bfloat16),
                          "Hp": ref.stats.new_empty(inp.Hp.shape, dtype=torch.bfloat16)})
    slot = stager.put(host)
    for k in range(3):
        nxt = stager.put(host) if k < 2 else None
        b = stager.get(slot)
        got = lm_head_loss_fwd("kl_div", b["Hq"], W, None, b["Hp"])
        stager.done(slot)
        torch.cuda.synchronize()
        assert torch.equal(got.loss_tok, ref.loss_tok)
        slot = nxt
