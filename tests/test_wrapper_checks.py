"""The Python wrappers refuse tensors whose device, dtype, layout or extent differ from what
the kernels are told, before anything is launched (the C ABI sees raw pointers only, so a
CPU tensor or a short buffer would otherwise be read or written past its end)."""

import pytest
import torch

from lm_head_loss_streaming_b200 import loss as L


def _cpu_bf16(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def test_cpu_tensors_are_refused():
    h, w = _cpu_bf16(4, 16), _cpu_bf16(32, 16)
    lab = torch.zeros(4, dtype=torch.int32)
    with pytest.raises(ValueError):
        L.lm_head_loss_fwd("ce", h, w, lab)
    with pytest.raises(ValueError):
        L.lm_head_loss_fwd_bwd("kl_div", h, w, None, h)
    with pytest.raises(ValueError):
        L.lm_head_loss_combo_fwd({"ce": 1.0}, h, w, lab)
    with pytest.raises(ValueError):
        L.target_flatness(h, w)
    with pytest.raises(ValueError):
        L.align_labels(torch.zeros(2, 3, dtype=torch.int32), 1)


def test_unknown_kind_is_refused():
    with pytest.raises(ValueError):
        L.lm_head_loss_fwd("mse", _cpu_bf16(4, 16), _cpu_bf16(32, 16))


@pytest.mark.gpu
def test_mismatched_shapes_and_devices_are_refused():
    dev = torch.device("cuda", 0)
    N, d, V = 64, 32, 100
    h = torch.zeros(N, d, dtype=torch.bfloat16, device=dev)
    w = torch.zeros(V, d, dtype=torch.bfloat16, device=dev)
    lab = torch.zeros(N, dtype=torch.int32, device=dev)
    bad = [
        dict(kind="ce", hidden=h, weight=torch.zeros(V, d + 8, dtype=torch.bfloat16, device=dev),
             labels=lab),
        dict(kind="ce", hidden=h, weight=w, labels=lab[:-1]),
        dict(kind="ce", hidden=h, weight=w, labels=lab.cpu()),
        dict(kind="ce", hidden=h, weight=w, labels=lab.to(torch.int64)),
        dict(kind="kl_div", hidden=h, weight=w, target_hidden=h[:-1]),
        dict(kind="kl_div", hidden=h, weight=w, target_hidden=h.t().contiguous().t()),
    ]
    for kw in bad:
        with pytest.raises(ValueError):
            L.lm_head_loss_fwd(**kw)
    f = L.lm_head_loss_fwd("ce", h, w, lab)
    with pytest.raises(ValueError):
        L.lm_head_loss_bwd(f, h, w, lab, dW=torch.zeros(V, d, device=dev)[:-1])
    with pytest.raises(ValueError):
        L.lm_head_loss_bwd(f, h, w, lab, dH=torch.zeros(N, d, device=dev))   # fp32, not bf16
    with pytest.raises(ValueError):
        L.lm_head_loss_bwd(f, h[:32], w, lab[:32])                           # another N
    with pytest.raises(ValueError):
        L.lm_head_loss_bwd(f, h, w, lab, grad_tok=torch.ones(N))            # on the CPU
    with pytest.raises(ValueError):
        L.lm_head_loss_fwd_bwd("ce", h, w, lab, grad_scale=torch.ones(2, device=dev))
    with pytest.raises(ValueError):
        L.align_labels(lab.reshape(8, 8), 1, loss_mask=torch.ones(8, 8, dtype=torch.uint8))
