import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built libsas.so")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Report the bf16 output comparisons: the stated bar is max-abs <= 1e-2 against the
    fp64 oracle; elements over it pass only where |o| >= 4 and they are within 1e-2 of
    the oracle rounded to bf16 (the output format's own rounding). Their count is shown."""
    from tests.parity_util import OUT_LOG
    if not OUT_LOG:
        return
    tr = terminalreporter
    n_el = sum(r[1] for r in OUT_LOG)
    n_q = sum(r[4] for r in OUT_LOG)
    worst = max(OUT_LOG, key=lambda r: r[2])
    tr.write_sep("-", "bf16 outputs against the fp64 oracle")
    tr.write_line(f"{len(OUT_LOG)} comparisons, {n_el} elements; max-abs {worst[2]:.3e} ({worst[0]}); "
                  f"{n_q} elements over 1e-2 pass only through the bf16 output-rounding exemption")
    for what, size, m, mq, q in OUT_LOG:
        if q or m > 1e-2:
            tr.write_line(f"  {what}: {size} elements, max-abs {m:.3e}, vs rounded {mq:.3e}, exempted {q}")
