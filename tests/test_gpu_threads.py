"""Layers created and run from several host threads at once: fresh handles on
four threads, each on its own stream, give the same bits as the serial run.
The worker runs in a fresh process so that the library's one-time set-up
(encoder lookup, the GEMM kernels' per-device shared-memory attributes) is
first reached by the racing threads."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def test_concurrent_handles_on_four_threads_match_serial(cuda_ok):
    r = subprocess.run([sys.executable, "-m", "tests.threads_worker"], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "OK" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]
