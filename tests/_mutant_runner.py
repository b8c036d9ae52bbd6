"""Run every oracle pin against one compiled copy of the oracle.

Usage: python _mutant_runner.py <path to .so>.  Exit status 0 when every pin
passes, 1 when at least one fails.  Run in a child process so that a copy
that crashes counts as caught without taking the test session down.
"""
import functools
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import oracle  # noqa: E402
from oracle_pins import ALL_PINS  # noqa: E402


def main(path):
    fwd = functools.partial(oracle.attention_forward, _lib_override=oracle.open_library(path))
    failed = []
    for pin in ALL_PINS:
        try:
            pin(fwd)
        except AssertionError:
            failed.append(pin.__name__)
    print("failed:", ",".join(failed) if failed else "none")
    return 1 if failed else 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1]))
