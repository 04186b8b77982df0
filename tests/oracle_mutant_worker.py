"""Runs tests/test_oracle_pins.py once per oracle library named on the command
line, all in this one process (the imports are paid once), and prints one JSON
line per library: {"lib": path, "rc": pytest's exit code}.

With ``--oracle-dir DIR`` first, the oracle package is imported from DIR (a copy
whose Python glue may carry a planted mistake) instead of the repository's.  A
helper of tests/test_oracle_mutants.py, which builds the libraries and copies;
not a test module itself."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
if len(sys.argv) > 2 and sys.argv[1] == "--oracle-dir":
    sys.path.insert(0, sys.argv[2])
    del sys.argv[1:3]

import oracle  # noqa: E402

PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")


def main(paths):
    for path in paths:
        oracle.use_library(path)
        rc = pytest.main([PINS, "-x", "-q", "-p", "no:cacheprovider", "--no-header", "-o", "console_output_style=classic"])
        print("ZCMOE-MUTANT " + json.dumps({"lib": path, "rc": int(rc)}), flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
