"""The FMA-pipe exponential of the loss epilogues (slm_debug_exp2), checked against CUDA's
exp2f and against the exact 2^x.

The epilogues compute part of their exponentials 2^x (x <= 0, the softmax weights
2^(z log2 e - m)) on the FMA pipe: x = j + r with j = round(x), 2^r from a degree-5
polynomial fitted to 2^r on [-0.5, 0.5], and j added into the exponent field.  Its fitted
relative error is 2.2e-7 in fp32 Horner form, about the accuracy of exp2f itself.  Here it
must stay within 4e-7 of the exact value and of exp2f over [-125, 0], and give a result
no larger than 2^-126 below -126, where it clamps.
"""

import numpy as np
import pytest
import torch

from lm_head_loss_streaming_b200 import _lib

pytestmark = pytest.mark.gpu


def _run(x_np):
    dev = torch.device("cuda", 0)
    x = torch.from_numpy(x_np.astype(np.float32)).to(dev)
    yf = torch.empty_like(x)
    ym = torch.empty_like(x)
    st = _lib.slm_debug_exp2(x.data_ptr(), yf.data_ptr(), ym.data_ptr(), x.numel(),
                             torch.cuda.current_stream().cuda_stream)
    assert st == 0, _lib.status_string(st)
    torch.cuda.synchronize()
    return yf.cpu().numpy().astype(np.float64), ym.cpu().numpy().astype(np.float64)


def test_fma_exp2_matches_exp2f_and_the_exact_value():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        -rng.random(200_000) * 125.0,               # the whole range
        -rng.random(200_000) * 4.0,                 # where the softmax weights live
        np.arange(0, -126, -1, dtype=np.float64),   # integers (r = 0)
        np.arange(0, -126, -1) - 0.5,               # halfway points (r = +-0.5)
        [0.0, -1e-7, -0.49999997, -0.5, -0.50000006, -1.5, -124.999],
    ]).astype(np.float32)
    yf, ym = _run(x)
    exact = np.exp2(x.astype(np.float64))
    rel_exact = np.abs(yf / exact - 1.0)
    rel_mufu = np.abs(yf / ym - 1.0)
    assert rel_exact.max() <= 4e-7, (rel_exact.max(), x[rel_exact.argmax()])
    assert rel_mufu.max() <= 4e-7, (rel_mufu.max(), x[rel_mufu.argmax()])
    assert (yf > 0).all()


def test_fma_exp2_clamps_below_minus_126():
    x = np.array([-126.0, -126.5, -127.0, -150.0, -1e4, -3e38], dtype=np.float32)
    yf, _ = _run(x)
    assert (yf >= 0).all() and (yf <= 2.0 ** -126 * 1.0000005).all()


def test_debug_exp2_rejects_bad_arguments():
    assert _lib.slm_debug_exp2(None, None, None, 0, None) == 0
    assert _lib.slm_debug_exp2(None, None, None, 5, None) == 1
    assert _lib.slm_debug_exp2(None, None, None, -1, None) == 2
