import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Counts of every GPU-vs-oracle comparison of the session: boundary mismatches
    of codes and signs (and the vectors excluded for them), the largest norm and
    gamma errors, and the decode max-abs errors."""
    try:
        import parity
    except Exception:
        return
    if not parity.STATS:
        return
    tr = terminalreporter
    tr.section("parity counts (GPU vs oracle)")
    for label, s in parity.STATS:
        if "decode_max_abs" in s:
            extra = "".join("  %s %.3e" % (k, v) for k, v in s.items() if k not in ("decode_max_abs", "outputs"))
            tr.write_line("%-58s decode max-abs %.3e over %d outputs%s" % (label[:58], s["decode_max_abs"],
                                                                         s["outputs"], extra))
        elif "coords" not in s:
            tr.write_line("%-58s %s" % (label[:58], "  ".join("%s %.4g" % (k, v) for k, v in s.items())))
        else:
            tr.write_line("%-58s coords %d: code mism %d (bad %d), sign mism %d (bad %d), excluded vec %d, "
                          "norm %.1e, gamma %.1e" % (label[:58], s["coords"], s["code_mismatch"], s["code_bad"],
                                                     s.get("sign_mismatch", 0), s.get("sign_bad", 0),
                                                     s["excluded_vectors"], s["norm_max_rel"],
                                                     s.get("gamma_max_rel", 0.0)))
