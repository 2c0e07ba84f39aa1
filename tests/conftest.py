import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter):
    """Worst error and cosine of each whole-encoder parity comparison."""
    try:
        from parity_util import PARITY_REPORT
    except ImportError:
        return
    if not PARITY_REPORT:
        return
    terminalreporter.write_sep("-", "encoder parity against the fp64 oracle (worst over valid rows)")
    for label, n_seq, n_tok, err, cos, kind in PARITY_REPORT:
        c = "" if cos is None else f"  min per-token cosine {cos:.6f}"
        terminalreporter.write_line(f"{label}: {n_seq} seqs, {n_tok} tokens, max {kind} err {err:.3e}{c}")
