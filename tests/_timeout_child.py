"""Child process of test_gpu_timeout.py, run on the test-hook build of the
library (``FATHOM_LIB`` names it).  Prints one JSON line with what it saw.

One decode step runs normally, then again with one ring arrival withheld
(``FATHOM_TEST_WITHHOLD_ARRIVAL=1``): the scan's bounded waits run out, the
kernels return, and the error must reach the host through every route the
header promises -- union_count, fathom_device_status, Step.repair -- after
which a normal step on the same context is again exact."""
import dataclasses
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from long_context_decode_bit_b200 import fathom, inputs  # noqa: E402

WITHHOLD = "FATHOM_TEST_WITHHOLD_ARRIVAL"


def main():
    lib_path = fathom.load()._name
    w = dataclasses.replace(inputs.LAYER_32K, name="timeout-2x32768", H=2)
    k = inputs.keys(w, 0, w.H, device="cuda")
    q = inputs.queries(w, 0, w.H, device="cuda").float().contiguous()
    s2 = inputs.calibration_sigma2(k, w.n_cal).contiguous()
    planes, scales = fathom.pack(k)
    del k
    st = fathom.Step(planes, scales, w.n, s2, w.G, w.k, budget=48)
    ref = [t.clone() for t in st.run(q)]
    torch.cuda.synchronize()
    out = {"lib": lib_path, "status_before": fathom.device_status(),
           "ref_counts": ref[2].tolist()}

    os.environ[WITHHOLD] = "1"
    try:
        _, _, cnt = st.run(q, check_overflow=False)
        torch.cuda.synchronize()
    finally:
        del os.environ[WITHHOLD]
    out["withheld_counts"] = cnt.tolist()
    out["status_withheld"] = fathom.device_status()
    try:
        st.repair(q)
        out["repair"] = "returned"
    except fathom.FathomError as e:
        out["repair"] = e.status
    out["status_clear"] = fathom.device_status(clear=True)
    out["status_after"] = fathom.device_status()

    got = st.run(q)
    torch.cuda.synchronize()
    out["normal_again_equal"] = all(torch.equal(a, b) for a, b in zip(got, ref))
    out["status_end"] = fathom.device_status()
    print(json.dumps(out))


if __name__ == "__main__":
    main()
