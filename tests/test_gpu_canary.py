"""Out-of-bounds writes: every output buffer and the workspace sit inside a larger
allocation whose margins hold a canary pattern; after the calls the margins must be
unchanged.  Ragged shapes (N, V and d not multiples of any tile) exercise every tail path
of the kernels, the two-call path and the fused single call alike.
"""

import pytest
import torch

from lm_head_loss_streaming_b200 import _lib, synthetic
from lm_head_loss_streaming_b200.loss import (FwdResult, lm_head_loss_bwd, lm_head_loss_fwd,
                                              lm_head_loss_fwd_bwd)

pytestmark = pytest.mark.gpu

M = 64  # margin, in elements (bytes for the workspace: 64 KiB)


def _padded(shape, dtype, dev, fill):
    """A contiguous tensor of `shape` at offset M of a flat buffer pre-filled with `fill`."""
    n = 1
    for s in shape:
        n *= s
    flat = torch.full((n + 2 * M,), fill, dtype=dtype, device=dev)
    return flat, flat[M:M + n].view(*shape)


def _margins_intact(flat, fill):
    ref = torch.full((M,), fill, dtype=flat.dtype, device=flat.device)
    return torch.equal(flat[:M], ref) and torch.equal(flat[-M:], ref)


@pytest.mark.parametrize("kind,N,d,V", [("ce", 301, 72, 1037), ("kl_div", 259, 136, 2051),
                                        ("tv", 130, 64, 777), ("jsd", 67, 40, 3001),
                                        ("ce_argmax_p", 513, 24, 4099)])
@pytest.mark.parametrize("fused", [False, True])
def test_no_write_outside_outputs_and_workspace(kind, N, d, V, fused):
    dev = torch.device("cuda", 0)
    inp = synthetic.make(kind, N, d, V, w_std=0.1, ignore_frac=0.1, seed=101,
                         with_labels=kind != "ce_argmax_p")
    Hq, W = inp.Hq.to(dev), inp.W.to(dev)
    Hp = inp.Hp.to(dev) if inp.Hp is not None else None
    lab = inp.labels.to(dev) if inp.labels is not None else None
    k = _lib.KIND[kind]
    bufs = {}
    bufs["loss_tok"] = _padded((N,), torch.float32, dev, 7.25)
    bufs["alpha"] = _padded((N,), torch.float32, dev, 7.25)
    bufs["stats"] = _padded((_lib.slm_stats_floats(k), N), torch.float32, dev, 7.25)
    bufs["dH"] = _padded((N, d), torch.bfloat16, dev, 7.25)
    bufs["dW"] = _padded((V, d), torch.float32, dev, 7.25)
    need = (_lib.slm_fused_workspace_bytes(k, N, d, V, 128) if fused
            else _lib.slm_workspace_bytes(k, N, d, V, 128))
    ws = torch.full((need + 65536,), 0xA5, dtype=torch.uint8, device=dev)
    out = FwdResult(k, torch.empty(1, device=dev),
                    torch.empty(1, dtype=torch.float64, device=dev),
                    torch.empty(1, dtype=torch.int64, device=dev), bufs["loss_tok"][1],
                    bufs["alpha"][1] if k in _lib.ALPHA_KINDS else None, bufs["stats"][1], ws)
    if fused:
        lm_head_loss_fwd_bwd(kind, Hq, W, lab, Hp, inp.ignore_index, chunk_tokens=128,
                             workspace=ws, out=out, dH=bufs["dH"][1], dW=bufs["dW"][1])
    else:
        f = lm_head_loss_fwd(kind, Hq, W, lab, Hp, inp.ignore_index, workspace=ws,
                             chunk_tokens=128, out=out)
        lm_head_loss_bwd(f, Hq, W, lab, Hp, inp.ignore_index, dH=bufs["dH"][1],
                         dW=bufs["dW"][1], chunk_tokens=128)
    torch.cuda.synchronize()
    assert _lib.slm_device_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream) == 0
    for name, (flat, _) in bufs.items():
        assert _margins_intact(flat, 7.25), name
    tail = ws[need:]
    assert torch.equal(tail, torch.full_like(tail, 0xA5)), "workspace tail"
