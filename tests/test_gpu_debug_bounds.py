"""The debug build's device-side bounds checks (a sanitizer stand-in: a failed
check writes the device fault word instead of trapping, and the access is
skipped).  Built into the test-hook library (``build(test_hooks=True)``);
run in a child process so that the product library of the other tests is
untouched.

Every check passes on decode steps at several shapes, and those steps give
the product library's results bit for bit.  A failed check reaches the host
as FATHOM_ERR_BOUNDS in union_count and from fathom_device_status, which
clears it, and the next step is exact again."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from long_context_decode_bit_b200 import build, fathom

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_debug_bounds_checks_pass_and_report(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = build.build(test_hooks=True)
    npz = str(tmp_path / "debug_steps.npz")
    env = dict(os.environ, FATHOM_LIB=lib)
    env.pop("FATHOM_TEST_SHRINK_CAP", None)
    env.pop("FATHOM_TEST_WITHHOLD_ARRIVAL", None)
    r = subprocess.run([sys.executable, os.path.join(HERE, "_bounds_child.py"), npz], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-4000:]
    out = json.loads(r.stdout.strip().splitlines()[-1])
    assert out["lib"] == lib
    assert all(st == fathom.OK for st in out["status"].values()), out["status"]
    # The checked build gives the product library's results.
    sys.path.insert(0, HERE)
    import _bounds_child as child
    fathom.load()
    saved = np.load(npz)
    for name, w in child.SHAPES.items():
        st, q = child.step(w)
        idx, uni, cnt = st.run(q)
        torch.cuda.synchronize()
        for key, t in (("idx", idx), ("uni", uni), ("cnt", cnt)):
            assert np.array_equal(saved[f"{name}/{key}"], t.cpu().numpy()), (name, key)
    # A failed check: every group reports it, the status reads and clears.
    assert out["shrunk_counts"] == [fathom.ERR_BOUNDS] * len(out["shrunk_counts"])
    assert out["status_shrunk"] == fathom.ERR_BOUNDS
    assert out["status_clear"] == fathom.ERR_BOUNDS and out["status_after"] == fathom.OK
    assert out["normal_again_equal"]
