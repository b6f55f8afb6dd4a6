"""Child process of test_gpu_debug_bounds.py, run on the test-hook build of
the library (``FATHOM_LIB`` names it), whose device-side bounds checks are
on.  Runs decode steps at a few shapes (every check must pass), saves their
outputs for the parent to compare with the product library, then makes the
checks fail on purpose (``FATHOM_TEST_SHRINK_CAP=1``: the checks allow half
of the candidate entries; the skipped writes are never out of bounds) and
reports what the host sees.  Prints one JSON line."""
import dataclasses
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from long_context_decode_bit_b200 import fathom, inputs  # noqa: E402

SHAPES = {
    "sampled-8x32768": dataclasses.replace(inputs.LAYER_32K, H=8),
    "ragged-3x9001": dataclasses.replace(inputs.LAYER_32K, H=3, n=9001, seed=17),
    "direct-2x2000": dataclasses.replace(inputs.TINY, H=2, n=2000, seed=91),
}


def step(w):
    k = inputs.keys(w, 0, w.H, device="cuda")
    q = inputs.queries(w, 0, w.H, device="cuda").float().contiguous()
    s2 = inputs.calibration_sigma2(k, w.n_cal).contiguous()
    planes, scales = fathom.pack(k)
    st = fathom.Step(planes, scales, w.n, s2, w.G, w.k, budget=48)
    return st, q


def main(out_path):
    lib_path = fathom.load()._name
    out = {"lib": lib_path, "status": {}}
    saved = {}
    for name, w in SHAPES.items():
        st, q = step(w)
        idx, uni, cnt = st.run(q)
        torch.cuda.synchronize()
        out["status"][name] = fathom.device_status()
        saved[name + "/idx"], saved[name + "/uni"], saved[name + "/cnt"] = (t.cpu().numpy() for t in (idx, uni, cnt))
    np.savez(out_path, **saved)

    st, q = step(SHAPES["direct-2x2000"])
    os.environ["FATHOM_TEST_SHRINK_CAP"] = "1"
    try:
        _, _, cnt = st.run(q, check_overflow=False)
        torch.cuda.synchronize()
    finally:
        del os.environ["FATHOM_TEST_SHRINK_CAP"]
    out["shrunk_counts"] = cnt.tolist()
    out["status_shrunk"] = fathom.device_status()
    out["status_clear"] = fathom.device_status(clear=True)
    out["status_after"] = fathom.device_status()
    idx, uni, cnt = st.run(q)
    torch.cuda.synchronize()
    out["normal_again_equal"] = bool(np.array_equal(idx.cpu().numpy(), saved["direct-2x2000/idx"]) and
                                     np.array_equal(cnt.cpu().numpy(), saved["direct-2x2000/cnt"]))
    print(json.dumps(out))


if __name__ == "__main__":
    main(sys.argv[1])
