"""The C ABI library on a machine without a GPU: it loads, exports every symbol the header
declares, and rejects invalid arguments on the host before touching CUDA."""

import ctypes
import os
import re

import pytest

from lm_head_loss_streaming_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "slm.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(slm_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from lm_head_loss_streaming_b200.build import build
        build()
    return _lib.load()


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert set(names) == set(_lib.SIGNATURES), names
    for n in names:
        assert hasattr(lib, n), n


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libslm.so"))
    with pytest.raises(ImportError):
        _lib.load()


def test_library_override_names_the_missing_file(tmp_path):
    """SLM_LIBRARY points the binding at a variant build; a wrong path fails on load, naming
    the path, and never falls back to the in-tree build."""
    import subprocess
    import sys

    missing = str(tmp_path / "variant" / "libslm.so")
    code = ("from lm_head_loss_streaming_b200 import _lib\n"
            "try:\n    _lib.load()\nexcept ImportError as e:\n    print('IMPORTERROR', e)\n")
    env = dict(os.environ, SLM_LIBRARY=missing)
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "IMPORTERROR" in r.stdout and missing in r.stdout


def test_variant_build_rejects_bad_definitions(tmp_path):
    from lm_head_loss_streaming_b200.build import build

    for bad in ("SLM_GROUP_B=1;rm", "A B", "X=$(y)"):
        with pytest.raises(ValueError):
            build(out=str(tmp_path / "libslm.so"), defines=[bad])


def test_status_strings_and_sizes(lib):
    assert _lib.slm_version() >= 100
    for code, name in _lib.STATUS_NAMES.items():
        assert _lib.slm_status_string(code).startswith(name)
    assert _lib.slm_stats_floats(_lib.SLM_CE) == 1
    assert _lib.slm_stats_floats(_lib.SLM_KL) == 3
    for k in (_lib.SLM_TV, _lib.SLM_NLA, _lib.SLM_LK_HYBRID):
        assert _lib.slm_stats_floats(k) == 5
    assert _lib.slm_stats_floats(_lib.SLM_RKL) == 3
    assert _lib.slm_stats_floats(_lib.SLM_JSD) == 5
    assert _lib.slm_stats_floats(_lib.SLM_CE_ARGMAX_P) == 2
    assert _lib.slm_stats_floats(8) == 0
    assert _lib.slm_workspace_bytes(_lib.SLM_CE, 16, 12, 100) == 0  # d % 8 != 0
    assert _lib.slm_workspace_bytes(9, 16, 16, 100) == 0


def test_workspace_holds_chunk_buffer(lib):
    # The backward's chunk buffer: chunk x V x bf16 (V padded to 8), chunk = min(N, 2d).
    N, d, V = 16384, 4096, 128256
    ws = _lib.slm_workspace_bytes(_lib.SLM_KL, N, d, V)
    assert ws >= 8192 * V * 2
    # O(N d + V d): far below the fp32 logits of the whole batch.
    assert ws < N * V * 4 / 3
    ws_small = _lib.slm_workspace_bytes(_lib.SLM_KL, N, d, V, 1024)
    assert 1024 * V * 2 <= ws_small < ws
    assert _lib.slm_workspace_bytes(_lib.SLM_CE, 0, 8, 10) > 0


@pytest.mark.parametrize("kind", range(8))
def test_workspace_is_linear_in_tokens_and_bounded_by_dw(lib, kind):
    """Memory stays O(N d + V d): the backward's chunk buffer is capped by the size of the
    fp32 dW (chunk = min(N, 2d) rows of bf16 logit gradients), and everything else grows
    by a fixed number of bytes per token (the forward's per-row partial statistics).  The
    fused call's buffer holds a fixed number of chunk rows, whatever N and d are."""
    V = 128256
    for d in (256, 2048, 4096, 16384):
        for N in (256, 8192, 65536, 1 << 20):
            ws = _lib.slm_workspace_bytes(kind, N, d, V, 0)
            assert 0 < ws <= 4 * V * d + 1536 * N + (1 << 20), (d, N, ws)
            assert ws < N * V * 4 or N <= 2 * d   # never the whole batch's fp32 logits
            fws = _lib.slm_fused_workspace_bytes(kind, N, d, V, 0)
            # fp32 q and p logits plus bf16 dZ for 4096 rows, and the chunk's partials.
            assert 0 < fws <= 10 * 4096 * V + 64 * N + (16 << 20), (d, N, fws)
    # Doubling the batch past the chunk size adds only per-token bytes.
    a = _lib.slm_workspace_bytes(kind, 1 << 16, 4096, V, 0)
    b = _lib.slm_workspace_bytes(kind, 1 << 17, 4096, V, 0)
    assert 0 <= b - a <= 1536 * (1 << 16)


A = 1 << 20  # a 256-byte aligned fake address; never dereferenced on these paths


def _fwd(**kw):
    args = dict(kind=0, Hq=A, Hp=None, W=A, labels=A, ignore_index=-100, N=4, d=16, V=32,
                loss_tok=A, alpha_tok=None, loss_sum=A, n_valid=A, loss_mean=None, stats=A,
                workspace=A, ws_bytes=1 << 30, stream=None)
    args.update(kw)
    return _lib.slm_loss_fwd(*args.values())


def _bwd(**kw):
    args = dict(kind=0, Hq=A, Hp=None, W=A, labels=A, ignore_index=-100, N=4, d=16, V=32,
                grad_tok=None, grad_scale=None, n_valid=None, stats=A, dHq=A, dW=A,
                accumulate_dW=0, chunk_tokens=0, workspace=A, ws_bytes=1 << 30, stream=None)
    args.update(kw)
    return _lib.slm_loss_bwd(*args.values())


@pytest.mark.parametrize("fn", [_fwd, _bwd])
def test_host_errors(lib, fn):
    assert fn(kind=8) == 4                   # SLM_ERR_KIND
    assert fn(kind=-1) == 4
    assert fn(d=12) == 2                     # SLM_ERR_SHAPE: d % 8
    assert fn(d=0) == 2
    assert fn(V=0) == 2
    assert fn(N=-1) == 2
    assert fn(W=None) == 1                   # SLM_ERR_NULL
    assert fn(Hq=None) == 1
    assert fn(labels=None) == 1              # CE needs labels
    assert fn(kind=1) == 1                   # KL needs Hp
    assert fn(kind=7) == 1                   # CE against argmax p needs Hp
    assert fn(workspace=None) == 1
    assert fn(W=A + 8) == 3                  # SLM_ERR_ALIGN
    assert fn(Hq=A + 2) == 3
    assert fn(workspace=A + 16) == 5         # SLM_ERR_WORKSPACE: alignment
    assert fn(ws_bytes=16) == 5              # SLM_ERR_WORKSPACE: size


def test_fwd_output_pointer_errors(lib):
    assert _fwd(loss_sum=None) == 1
    assert _fwd(n_valid=None) == 1
    assert _fwd(stats=None) == 1


def test_bwd_output_pointer_errors(lib):
    assert _bwd(dW=None) == 1
    assert _bwd(dHq=None) == 1
    assert _bwd(dW=A + 4) == 3


def test_debug_hook_arguments(lib):
    assert _lib.slm_debug_set(3, 0) == 2     # SLM_ERR_SHAPE: unknown mode
    assert _lib.slm_debug_set(2, 0) == 0     # lockstep gives up at once
    assert _lib.slm_debug_set(-1, 0) == 2
    assert _lib.slm_debug_set(0, -1) == 2    # SLM_ERR_SHAPE: negative bound
    assert _lib.slm_debug_set(0, 0) == 0     # back to normal operation
    for fn in (_lib.slm_debug_exp2,):
        assert fn(None, None, None, 0, None) == 0          # nothing to do
        assert fn(None, None, None, 5, None) == 1          # SLM_ERR_NULL
        assert fn(None, None, None, -1, None) == 2         # SLM_ERR_SHAPE
        assert fn(None, None, None, 1 << 31, None) == 2


def _combo_fwd(weights, **kw):
    args = dict(Hq=A, Hp=A, W=A, labels=A, ignore_index=-100, N=4, d=16, V=32, loss_tok=A,
                term_loss_tok=None, loss_sum=A, term_loss_sum=None, n_valid=A, loss_mean=None,
                stats=A, workspace=A, ws_bytes=1 << 30, stream=None)
    args.update(kw)
    return _lib.slm_combo_fwd(weights, *args.values())


def test_combo_host_errors(lib):
    assert _lib.slm_combo_workspace_bytes(4, 16, 32) > 0
    assert _lib.slm_combo_workspace_bytes(4, 12, 32) == 0
    assert _combo_fwd({}) == 4                          # no term: SLM_ERR_KIND
    assert _combo_fwd({"kl_div": float("nan")}) == 4    # NaN weight
    assert _combo_fwd({"kl_div": float("inf")}) == 4
    assert _combo_fwd({"ce": 1.0}, labels=None) == 1    # CE term needs labels
    assert _combo_fwd({"tv": 1.0}, Hp=None) == 1        # distribution term needs Hp
    assert _combo_fwd({"tv": 1.0}, d=12) == 2
    assert _combo_fwd({"tv": 1.0}, W=A + 8) == 3
    assert _combo_fwd({"tv": 1.0}, ws_bytes=16) == 5
    assert _combo_fwd({"tv": 1.0}, stats=None) == 1


def test_helper_host_errors(lib):
    assert _lib.slm_align_labels(A, None, None, 2, 3, -1, -100, A, None) == 2   # shift < 0
    assert _lib.slm_align_labels(A, None, None, -1, 3, 1, -100, A, None) == 2
    assert _lib.slm_align_labels(None, None, None, 0, 3, 1, -100, None, None) == 0  # empty
    assert _lib.slm_align_labels(None, None, None, 2, 3, 1, -100, A, None) == 1
    assert _lib.slm_flatness_workspace_bytes(4, 12, 10) == 0
    assert _lib.slm_target_flatness(A, A, 4, 12, 10, A, A, 1 << 30, None) == 2
    assert _lib.slm_target_flatness(None, A, 4, 16, 10, A, A, 1 << 30, None) == 1
    assert _lib.slm_target_flatness(A, A, 4, 16, 10, A, A, 16, None) == 5


def test_overlap_backward_host_errors(lib):
    def bwd_ov(reserve, **kw):
        args = dict(kind=0, Hq=A, Hp=None, W=A, labels=A, ignore_index=-100, N=4, d=16, V=32,
                    grad_tok=None, grad_scale=None, n_valid=None, stats=A, dHq=A, dW=A,
                    accumulate_dW=0, chunk_tokens=0, workspace=A, ws_bytes=1 << 30,
                    stream=None, event=None)
        args.update(kw)
        return _lib.slm_loss_bwd_overlap(*args.values(), reserve)
    assert bwd_ov(-1) == 2                   # SLM_ERR_SHAPE: reserve_sms out of range
    assert bwd_ov(129) == 2
    assert bwd_ov(8, kind=8) == 4            # then the backward's own checks
    assert bwd_ov(8, d=12) == 2
    assert bwd_ov(8, dW=None) == 1
    assert bwd_ov(8, ws_bytes=16) == 5


@pytest.mark.parametrize("fused", [False, True])
def test_chunk_for_budget_is_the_largest_chunk_that_fits(lib, fused):
    """The chunk-size rule: the largest chunk whose workspace stays within the budget."""
    ws = _lib.slm_fused_workspace_bytes if fused else _lib.slm_workspace_bytes
    step = 256 if fused else 128
    for kind, N, d, V in ((_lib.SLM_KL, 16384, 4096, 128256), (_lib.SLM_CE, 8192, 2048, 128256),
                          (_lib.SLM_TV, 1000, 64, 3000)):
        for budget in (1 << 28, 1 << 30, 3 << 30, 1 << 40):
            c = _lib.slm_chunk_for_budget(kind, N, d, V, budget, fused)
            if c == 0:
                assert ws(kind, N, d, V, step) > budget
                continue
            assert c % step == 0 or c == N
            assert c <= N
            assert ws(kind, N, d, V, c) <= budget
            if c < N:
                assert ws(kind, N, d, V, c + step) > budget
        # An unlimited budget takes every row in one chunk.
        assert _lib.slm_chunk_for_budget(kind, N, d, V, 1 << 60, fused) == N
    # N not a multiple of the step: the chunk is never reported larger than N, and the
    # workspace of the reported chunk is the one the call uses.
    for N in (1, 127, 129, 300, 1000, 4097):
        c = _lib.slm_chunk_for_budget(_lib.SLM_KL, N, 64, 3000, 1 << 40, fused)
        assert c == N
    # With a budget between two steps the chunk stays a multiple of the step below N.
    N = 1000
    c = _lib.slm_chunk_for_budget(_lib.SLM_KL, N, 64, 3000, ws(_lib.SLM_KL, N, 64, 3000, 3 * step),
                                  fused)
    assert c == min(3 * step, N)
    assert _lib.slm_chunk_for_budget(_lib.SLM_KL, 1024, 12, 100, 1 << 30, fused) == 0  # d % 8
    assert _lib.slm_chunk_for_budget(9, 1024, 16, 100, 1 << 30, fused) == 0
    assert _lib.slm_chunk_for_budget(_lib.SLM_KL, 16384, 4096, 128256, 1, fused) == 0


def test_count_valid_rejects_bad_arguments_on_the_host(lib):
    fake = 1 << 20  # aligned, never dereferenced: every call below returns before enqueuing
    assert _lib.slm_count_valid(9, fake, -100, 10, 100, fake, None) == 4       # kind
    assert _lib.slm_count_valid(_lib.SLM_CE, fake, -100, -1, 100, fake, None) == 2  # N < 0
    assert _lib.slm_count_valid(_lib.SLM_CE, fake, -100, 10, 0, fake, None) == 2    # V <= 0
    assert _lib.slm_count_valid(_lib.SLM_CE, fake, -100, 1 << 31, 100, fake, None) == 2
    assert _lib.slm_count_valid(_lib.SLM_CE, None, -100, 10, 100, fake, None) == 1   # labels
    assert _lib.slm_count_valid(_lib.SLM_KL, fake, -100, 10, 100, None, None) == 1   # out


def test_trace_switch_and_empty_read(lib):
    assert _lib.slm_trace_enable(False) == 0
    st, got = _lib.slm_trace_read()
    assert st == 0
    assert set(got) == set(_lib.TRACE_CLASSES)
    assert all(ms == 0.0 and n == 0 for ms, n in got.values())
    assert lib.slm_trace_read(None, None, 3) == 1
    assert lib.slm_trace_read(None, None, 0) == 0
