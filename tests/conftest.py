import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")
    config.addinivalue_line("markers", "slow: long-running case")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


@pytest.fixture(autouse=True)
def _margin_test_name(request):
    """Tags the tolerance-headroom records of tests/parity_util.py with the running test."""
    try:
        import parity_util
    except ImportError:  # pragma: no cover
        yield
        return
    parity_util.CURRENT_TEST[0] = request.node.nodeid
    yield


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Prints, per test, the largest fraction of a parity tolerance that any comparison
    used (1.0 = at the tolerance), and for the near-tie comparisons the entries inside the
    band and the largest slack drawn; writes every record to $SLM_MARGINS_OUT if set."""
    try:
        import parity_util
    except ImportError:  # pragma: no cover
        return
    recs = parity_util.MARGINS
    if not recs:
        return
    out = os.environ.get("SLM_MARGINS_OUT")
    if out:
        import json
        with open(out, "w") as f:
            json.dump(recs, f, indent=0)
    worst = {}
    for r in recs:
        if r["test"] not in worst or r["frac_of_tol"] > worst[r["test"]]["frac_of_tol"]:
            worst[r["test"]] = r
    tw = terminalreporter
    tw.section("parity tolerance headroom (largest error / tolerance per test)")
    for t, r in sorted(worst.items(), key=lambda kv: -kv[1]["frac_of_tol"]):
        tw.line(f"{r['frac_of_tol']:7.3f}  {t}  [{r['what']}]")
    ties = [r for r in recs if "slack_used_frac" in r]
    if ties:
        tw.line("near-tie comparisons (entries in band / entries, slack used / tolerance, "
                "error without slack / tolerance):")
        for r in ties:
            off = r.get("raw_frac_off_tie_rows")
            off_s = "" if off is None else f"  off-tie-rows raw {off:.3f} ({r.get('tie_rows')} tie rows)"
            tw.line(f"  {r['near_ties']}/{r['entries']}  slack {r['slack_used_frac']:.4f}  "
                    f"raw {r['raw_frac']:.3f}{off_s}  {r['test']} [{r['what']}]")
