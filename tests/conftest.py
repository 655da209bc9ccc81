import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print the counts of every GPU <-> oracle comparison of the session (near ties and
    diverged groups included), so that a run's log keeps them even when the tests pass."""
    parity = sys.modules.get("parity")
    if parity is None or not parity.RECORDS:
        return
    tw = terminalreporter
    tw.section("parity counts (GPU against the oracle)")
    tot = dict(groups=0, exact=0, tie=0, div=0, codes=0, off=0)
    for label, r in parity.RECORDS:
        tw.write_line(f"{label}: {r.summary()}")
        tot["groups"] += r.n_groups
        tot["exact"] += r.zero_exact
        tot["tie"] += r.zero_near_tie
        tot["div"] += r.zero_diverged
        tot["codes"] += r.n_codes
        tot["off"] += r.code_diff
    tw.write_line(f"TOTAL: {len(parity.RECORDS)} comparisons, {tot['groups']} groups, zeros "
                  f"bit-exact {tot['exact']}, near ties {tot['tie']}, diverged {tot['div']}; "
                  f"codes off {tot['off']}/{tot['codes']}")
