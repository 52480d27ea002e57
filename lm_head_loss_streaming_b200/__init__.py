"""Streaming LM-head loss for B200 (sm_100a).

Hidden states [N, d] are projected by the LM head W [V, d] and reduced to a per-token loss
and its gradients without materialising the [N, V] logits.  The arithmetic runs in the
hand-written kernels of ``libslm.so`` behind a C ABI (``include/slm.h``); this package
only marshals arguments and allocates device memory through PyTorch.
"""

from .synthetic import IGNORE_INDEX  # noqa: F401

KINDS = ("ce", "kl_div", "tv", "nla", "lk_hybrid", "rkl", "jsd", "ce_argmax_p")


def __getattr__(name):
    # The binding and the autograd wrapper load the native library lazily, so the
    # input generators stay importable on machines without the built extension.
    if name in ("streaming_lm_head_loss", "StreamingLMHeadLoss", "lm_head_loss_fwd",
                "lm_head_loss_bwd"):
        from . import loss as _loss
        return getattr(_loss, name)
    if name == "lib":
        from . import _lib
        return _lib
    raise AttributeError(name)
