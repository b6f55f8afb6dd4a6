"""A bounded device wait that runs out is reported, not hung on.

The scan's staging ring waits on mbarriers with a poll limit.  A correct
launch never reaches it, so the test uses a build of the library made for it
(``build(test_hooks=True)``: a poll limit of 65536 and a switch that withholds
one ring arrival).  Nothing faults: the waiting warps give up, set the
device fault word, let their copies land and return, and the context stays
usable.  The test runs in a child process so that the product library
loaded by the other tests is not touched."""
import json
import os
import subprocess
import sys

import pytest
import torch

from long_context_decode_bit_b200 import build, fathom

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_withheld_ring_arrival_reports_timeout_and_context_recovers():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = build.build(test_hooks=True)
    env = dict(os.environ, FATHOM_LIB=lib)
    env.pop("FATHOM_TEST_WITHHOLD_ARRIVAL", None)
    r = subprocess.run([sys.executable, os.path.join(HERE, "_timeout_child.py")], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-4000:]
    out = json.loads(r.stdout.strip().splitlines()[-1])
    assert out["lib"] == lib
    assert out["status_before"] == fathom.OK
    assert all(c > 0 for c in out["ref_counts"])
    # every group of the step reports the timeout in union_count
    assert out["withheld_counts"] == [fathom.ERR_TIMEOUT] * len(out["ref_counts"])
    assert out["status_withheld"] == fathom.ERR_TIMEOUT
    assert out["repair"] == fathom.ERR_TIMEOUT   # Step.repair raises instead of rerunning
    assert out["status_clear"] == fathom.ERR_TIMEOUT and out["status_after"] == fathom.OK
    # the next normal step on the same context is exact again
    assert out["normal_again_equal"] and out["status_end"] == fathom.OK
