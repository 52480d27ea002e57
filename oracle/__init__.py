"""Float64 CPU oracle for the streaming LM-head loss (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  The product package ``lm_head_loss_streaming_b200`` never imports it
and it never imports the product package: the two share no code.
"""

from .slm_oracle import (  # noqa: F401
    KINDS,
    DISTRIBUTION_KINDS,
    ALPHA_KINDS,
    TARGET_KINDS,
    argmax_target,
    logits,
    log_softmax,
    token_terms,
    dlogits,
    forward,
    backward,
    loss_and_grads,
    combo_forward,
    combo_backward,
    align_labels,
    flatness,
    logits_bytes,
    chunk_buffer_bytes,
)
