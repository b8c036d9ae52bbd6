"""Run the oracle pins against one compiled copy of the oracle.

Usage: python _mutant_runner.py <path to .so> [--all].  Exit status 0 when
every pin passes, 1 as soon as one fails (one failing pin is enough to catch
a planted mistake; --all runs every pin regardless).  Run in a child process
so that a copy that crashes counts as caught without taking the test session
down.
"""
import functools
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import oracle  # noqa: E402
from oracle_pins import ALL_PINS, BWD_PINS  # noqa: E402


def main(path, run_all):
    lib = oracle.open_library(path)
    fwd = functools.partial(oracle.attention_forward, _lib_override=lib)
    bwd = functools.partial(oracle.attention_backward, _lib_override=lib)
    calls = [(pin, (fwd,)) for pin in ALL_PINS] + [(pin, (fwd, bwd)) for pin in BWD_PINS]
    failed = []
    for pin, args in calls:
        try:
            pin(*args)
        except AssertionError:
            failed.append(pin.__name__)
            if not run_all:
                break
    print("failed:", ",".join(failed) if failed else "none")
    return 1 if failed else 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1], "--all" in sys.argv[2:]))
