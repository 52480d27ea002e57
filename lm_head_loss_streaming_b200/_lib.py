"""ctypes binding of ``libslm.so`` (the C ABI declared in ``include/slm.h``).

Argument marshalling only: every function here forwards plain integers (device
addresses, sizes, a stream handle) to the C entry point of the same name and returns its
status.  Loading fails loudly when the library has not been built: there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# The in-tree build, or a variant built with `build --out PATH -D ...` named by SLM_LIBRARY.
LIB_PATH = os.path.abspath(os.environ.get("SLM_LIBRARY") or os.path.join(HERE, "libslm.so"))

SLM_CE, SLM_KL, SLM_TV, SLM_NLA, SLM_LK_HYBRID = 0, 1, 2, 3, 4
SLM_RKL, SLM_JSD, SLM_CE_ARGMAX_P = 5, 6, 7
KIND = {"ce": SLM_CE, "kl_div": SLM_KL, "tv": SLM_TV, "nla": SLM_NLA,
        "lk_hybrid": SLM_LK_HYBRID, "rkl": SLM_RKL, "jsd": SLM_JSD,
        "ce_argmax_p": SLM_CE_ARGMAX_P}
ALPHA_KINDS = (SLM_TV, SLM_NLA, SLM_LK_HYBRID)
SLM_NUM_KINDS = 8
SLM_COMBO_STATS = 9

SLM_OK = 0
STATUS_NAMES = {
    0: "SLM_OK", 1: "SLM_ERR_NULL", 2: "SLM_ERR_SHAPE", 3: "SLM_ERR_ALIGN",
    4: "SLM_ERR_KIND", 5: "SLM_ERR_WORKSPACE", 6: "SLM_ERR_LABEL_RANGE",
    7: "SLM_ERR_TIMEOUT", 8: "SLM_ERR_CUDA", 9: "SLM_ERR_UNSUPPORTED_ARCH",
}

# Every symbol the header declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_INT = ctypes.c_int
_SZ = ctypes.c_size_t
SIGNATURES = {
    "slm_version": (_INT, []),
    "slm_status_string": (ctypes.c_char_p, [_INT]),
    "slm_stats_floats": (_SZ, [_INT]),
    "slm_workspace_bytes": (_SZ, [_INT, _I64, _I64, _I64, _I64]),
    "slm_loss_fwd": (_INT, [_INT, _P, _P, _P, _P, _I32, _I64, _I64, _I64,
                            _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "slm_loss_bwd": (_INT, [_INT, _P, _P, _P, _P, _I32, _I64, _I64, _I64,
                            _P, _P, _P, _P, _P, _P, _INT, _I64, _P, _SZ, _P]),
    "slm_loss_bwd_overlap": (_INT, [_INT, _P, _P, _P, _P, _I32, _I64, _I64, _I64,
                                    _P, _P, _P, _P, _P, _P, _INT, _I64, _P, _SZ, _P,
                                    _P, _INT]),
    "slm_chunk_for_budget": (_I64, [_INT, _I64, _I64, _I64, _SZ, _INT]),
    "slm_device_status": (_INT, [_P, _P]),
    "slm_debug_set": (_INT, [_INT, ctypes.c_longlong]),
    "slm_fused_workspace_bytes": (_SZ, [_INT, _I64, _I64, _I64, _I64]),
    "slm_loss_fwd_bwd": (_INT, [_INT, _P, _P, _P, _P, _I32, _I64, _I64, _I64, _P, _P,
                                _P, _P, _P, _P, _P, _P, _P, _P, _INT, _I64, _P, _SZ, _P]),
    "slm_combo_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I64]),
    "slm_align_labels": (_INT, [_P, _P, _P, _I64, _I64, _I32, _I32, _P, _P]),
    "slm_flatness_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "slm_target_flatness": (_INT, [_P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "slm_combo_fwd": (_INT, [_P, _P, _P, _P, _P, _I32, _I64, _I64, _I64,
                             _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "slm_combo_bwd": (_INT, [_P, _P, _P, _P, _P, _I32, _I64, _I64, _I64,
                             _P, _P, _P, _P, _P, _P, _INT, _I64, _P, _SZ, _P]),
    "slm_loss_fwd_noalloc": (_INT, [_INT, _P, _P, _P, _P, _I32, _I64, _I64, _I64,
                                    _P, _P, _P, _P, _P, _P, _P, _P]),
    "slm_count_valid": (_INT, [_INT, _P, _I32, _I64, _I64, _P, _P]),
    "slm_set_backward_mode": (_INT, [_INT]),
    "slm_debug_exp2": (_INT, [_P, _P, _P, _I64, _P]),
    "slm_trace_enable": (_INT, [_INT]),
    "slm_trace_read": (_INT, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_I64), _INT]),
}

# Kernel classes of slm_trace_read, in order.
TRACE_CLASSES = ("fwd_gemm", "pass2_gemm", "dz_gemm", "dh_gemm", "dw_gemm", "bwd_fused",
                 "logits_row", "row")


class SLMError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}" if where else status_string(status))


_lib = None


def load():
    """Load ``libslm.so`` (raises if it is missing: there is no CPU fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built; run `python -m lm_head_loss_streaming_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status):
    try:
        return load().slm_status_string(int(status)).decode()
    except ImportError:
        return STATUS_NAMES.get(int(status), f"status {status}")


def check(status, where=""):
    if status != SLM_OK:
        raise SLMError(status, where)
    return status


def slm_version():
    return load().slm_version()


def slm_status_string(status):
    return load().slm_status_string(int(status)).decode()


def slm_stats_floats(kind):
    return load().slm_stats_floats(int(kind))


def slm_workspace_bytes(kind, N, d, V, chunk_tokens=0):
    return load().slm_workspace_bytes(int(kind), int(N), int(d), int(V), int(chunk_tokens))


def slm_loss_fwd(kind, Hq, Hp, W, labels, ignore_index, N, d, V, loss_tok, alpha_tok,
                 loss_sum, n_valid, loss_mean, stats, workspace, ws_bytes, stream):
    return load().slm_loss_fwd(int(kind), Hq, Hp, W, labels, int(ignore_index), int(N),
                               int(d), int(V), loss_tok, alpha_tok, loss_sum, n_valid,
                               loss_mean, stats, workspace, int(ws_bytes), stream)


def slm_loss_bwd(kind, Hq, Hp, W, labels, ignore_index, N, d, V, grad_tok, grad_scale,
                 n_valid, stats, dHq, dW, accumulate_dW, chunk_tokens, workspace, ws_bytes,
                 stream):
    return load().slm_loss_bwd(int(kind), Hq, Hp, W, labels, int(ignore_index), int(N),
                               int(d), int(V), grad_tok, grad_scale, n_valid, stats, dHq, dW,
                               int(accumulate_dW), int(chunk_tokens), workspace,
                               int(ws_bytes), stream)


def slm_loss_bwd_overlap(kind, Hq, Hp, W, labels, ignore_index, N, d, V, grad_tok,
                         grad_scale, n_valid, stats, dHq, dW, accumulate_dW, chunk_tokens,
                         workspace, ws_bytes, stream, dw_ready_event, reserve_sms):
    return load().slm_loss_bwd_overlap(int(kind), Hq, Hp, W, labels, int(ignore_index),
                                       int(N), int(d), int(V), grad_tok, grad_scale, n_valid,
                                       stats, dHq, dW, int(accumulate_dW), int(chunk_tokens),
                                       workspace, int(ws_bytes), stream, dw_ready_event,
                                       int(reserve_sms))


def slm_chunk_for_budget(kind, N, d, V, budget_bytes, fused=False):
    return load().slm_chunk_for_budget(int(kind), int(N), int(d), int(V), int(budget_bytes),
                                       1 if fused else 0)


def slm_device_status(workspace, stream):
    return load().slm_device_status(workspace, stream)


def slm_debug_set(fault_mode, timeout_cycles=0):
    """Test hook: make the next launches run a bounded wait out (fault_mode=1), or restore
    normal operation (0); timeout_cycles bounds every pipeline wait (0 = default)."""
    return load().slm_debug_set(int(fault_mode), int(timeout_cycles))


def slm_loss_fwd_noalloc(kind, Hq, Hp, W, labels, ignore_index, N, d, V, loss_tok, alpha_tok,
                         loss_sum, n_valid, loss_mean, stats, device_flags, stream):
    """Forward with the library's own fixed device scratch (no workspace argument), for
    callers that cannot allocate device memory."""
    return load().slm_loss_fwd_noalloc(int(kind), Hq, Hp, W, labels, int(ignore_index),
                                       int(N), int(d), int(V), loss_tok, alpha_tok,
                                       loss_sum, n_valid, loss_mean, stats, device_flags,
                                       stream)


def _weights(weights):
    """Host float[SLM_NUM_KINDS] array from a {kind name or id: weight} mapping."""
    arr = (ctypes.c_float * SLM_NUM_KINDS)()
    for k, w in weights.items():
        arr[KIND[k] if isinstance(k, str) else int(k)] = float(w)
    return arr


def slm_combo_workspace_bytes(N, d, V, chunk_tokens=0):
    return load().slm_combo_workspace_bytes(int(N), int(d), int(V), int(chunk_tokens))


def slm_combo_fwd(weights, Hq, Hp, W, labels, ignore_index, N, d, V, loss_tok, term_loss_tok,
                  loss_sum, term_loss_sum, n_valid, loss_mean, stats, workspace, ws_bytes,
                  stream):
    return load().slm_combo_fwd(_weights(weights), Hq, Hp, W, labels, int(ignore_index),
                                int(N), int(d), int(V), loss_tok, term_loss_tok, loss_sum,
                                term_loss_sum, n_valid, loss_mean, stats, workspace,
                                int(ws_bytes), stream)


def slm_combo_bwd(weights, Hq, Hp, W, labels, ignore_index, N, d, V, grad_tok, grad_scale,
                  n_valid, stats, dHq, dW, accumulate_dW, chunk_tokens, workspace, ws_bytes,
                  stream):
    return load().slm_combo_bwd(_weights(weights), Hq, Hp, W, labels, int(ignore_index),
                                int(N), int(d), int(V), grad_tok, grad_scale, n_valid, stats,
                                dHq, dW, int(accumulate_dW), int(chunk_tokens), workspace,
                                int(ws_bytes), stream)


def slm_fused_workspace_bytes(kind, N, d, V, chunk_tokens=0):
    return load().slm_fused_workspace_bytes(int(kind), int(N), int(d), int(V),
                                            int(chunk_tokens))


def slm_loss_fwd_bwd(kind, Hq, Hp, W, labels, ignore_index, N, d, V, grad_tok, grad_scale,
                     loss_tok, alpha_tok, loss_sum, n_valid, loss_mean, stats, dHq, dW,
                     accumulate_dW, chunk_tokens, workspace, ws_bytes, stream):
    return load().slm_loss_fwd_bwd(int(kind), Hq, Hp, W, labels, int(ignore_index), int(N),
                                   int(d), int(V), grad_tok, grad_scale, loss_tok, alpha_tok,
                                   loss_sum, n_valid, loss_mean, stats, dHq, dW,
                                   int(accumulate_dW), int(chunk_tokens), workspace,
                                   int(ws_bytes), stream)


def slm_align_labels(tokens, loss_mask, seq_ids, B, S, shift, ignore_index, labels, stream):
    return load().slm_align_labels(tokens, loss_mask, seq_ids, int(B), int(S), int(shift),
                                   int(ignore_index), labels, stream)


def slm_flatness_workspace_bytes(N, d, V):
    return load().slm_flatness_workspace_bytes(int(N), int(d), int(V))


def slm_target_flatness(Hp, W, N, d, V, flat, workspace, ws_bytes, stream):
    return load().slm_target_flatness(Hp, W, int(N), int(d), int(V), flat, workspace,
                                      int(ws_bytes), stream)


def slm_count_valid(kind, labels, ignore_index, N, V, n_valid, stream):
    return load().slm_count_valid(int(kind), labels, int(ignore_index), int(N), int(V),
                                  n_valid, stream)


def slm_trace_enable(on):
    return load().slm_trace_enable(1 if on else 0)


def slm_trace_read():
    """(status, {class name: (ms, launches)}) since the previous read."""
    n = len(TRACE_CLASSES)
    ms = (ctypes.c_double * n)()
    cnt = (_I64 * n)()
    st = load().slm_trace_read(ms, cnt, n)
    return st, {name: (ms[i], int(cnt[i])) for i, name in enumerate(TRACE_CLASSES)}


def slm_set_backward_mode(mode):
    """1: one persistent launch per backward chunk (default); 0: three launches per chunk.
    Returns the previous mode (-1: invalid mode, nothing changed)."""
    return load().slm_set_backward_mode(int(mode))


def slm_debug_exp2(x, y_fma, y_mufu, n, stream):
    """Test hook: the epilogues' FMA-pipe 2^x and CUDA's exp2f on the same device inputs."""
    return load().slm_debug_exp2(x, y_fma, y_mufu, int(n), stream)
