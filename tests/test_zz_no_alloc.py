"""The allocation-free entry point, fathom_scan_topk_noalloc, for callers
that cannot allocate device memory (an operator inside another runtime
that owns all free device memory, or a decode loop that must not call
cudaMalloc).  It keeps its candidate buffer in the library's own fixed
device array instead of a caller buffer.

Its results must equal those of the allocating path, fathom_scan in
CANDIDATE mode followed by fathom_topk, on two calls in a row (the second
call reuses the array the first one left behind).  This file is collected
last so a stop-at-first-failure run has already run every other test."""
import ctypes
import dataclasses

import pytest
import torch

from long_context_decode_bit_b200 import inputs

pytestmark = pytest.mark.gpu


def _setup(fathom, w, budget):
    k = inputs.keys(w, 0, w.H, device="cuda")
    q = inputs.queries(w, 0, w.H, device="cuda").float().contiguous()
    s2 = inputs.calibration_sigma2(k, w.n_cal).contiguous()
    planes, scales = fathom.pack(k)
    del k
    _, active, na, _ = fathom.plan(s2, q, budget)
    return planes, scales, active, na, q


@pytest.mark.parametrize("w", [
    dataclasses.replace(inputs.LAYER_32K, name="one-layer-8x32768"),
    dataclasses.replace(inputs.STEP_1M, name="one-layer-8x1048576", H=8),
    dataclasses.replace(inputs.TINY, name="tiny-no-sample", H=3),
], ids=lambda w: w.name)
def test_noalloc_equals_scan_then_topk_twice(fathom_gpu, w):
    fathom = fathom_gpu
    assert fathom.scan_cand_bytes(w.H, w.G, w.n, w.k) <= fathom.NOALLOC_SCRATCH_BYTES
    planes, scales, active, na, q = _setup(fathom, w, 48)
    cand = fathom.scan(planes, scales, w.n, active, na, q, fathom.SCAN_CANDIDATE, w.k)
    ref = fathom.topk(w.H, w.G, w.n, w.k, cand=cand)
    for call in range(2):
        out = tuple(torch.full_like(t, -7) for t in ref)
        got = fathom.scan_topk_noalloc(planes, scales, w.n, active, na, q, w.k, out=out)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b), f"call {call}"
    assert torch.all(ref[2] >= 0)


def test_noalloc_rejects_sizes_beyond_its_array(fathom_gpu):
    fathom = fathom_gpu
    w = dataclasses.replace(inputs.STEP_1M, H=2)
    planes, scales, active, na, q = _setup(fathom, w, 48)
    H_big = 288   # a whole 288-group step needs more than the fixed array
    assert fathom.scan_cand_bytes(H_big, w.G, w.n, w.k) > fathom.NOALLOC_SCRATCH_BYTES
    idx = torch.empty((H_big, w.G, w.k), dtype=torch.int32, device="cuda")
    uni = torch.empty((H_big, w.G * w.k), dtype=torch.int32, device="cuda")
    cnt = torch.empty(H_big, dtype=torch.int32, device="cuda")
    lib = fathom.lib()
    st = lib.fathom_scan_topk_noalloc(fathom._p(planes), fathom._p(scales), H_big, w.D, w.n, planes.shape[-1],
                                      fathom._p(active), fathom._p(na), fathom._p(q), w.G, w.k, fathom._p(idx),
                                      fathom._p(uni), fathom._p(cnt), fathom._stream(None))
    assert st == fathom.ERR_WORKSPACE


def test_noalloc_takes_no_device_memory_and_checks_outputs_first(fathom_gpu):
    """A call after the first on a device takes no device memory: the free
    memory the driver reports is the same before and after it.  Bad output
    pointers are rejected before any work is enqueued."""
    fathom = fathom_gpu
    w = dataclasses.replace(inputs.LAYER_32K, name="noalloc-mem", H=4)
    planes, scales, active, na, q = _setup(fathom, w, 48)
    out = (torch.empty((w.H, w.G, w.k), dtype=torch.int32, device="cuda"),
           torch.empty((w.H, w.G * w.k), dtype=torch.int32, device="cuda"),
           torch.empty(w.H, dtype=torch.int32, device="cuda"))
    fathom.scan_topk_noalloc(planes, scales, w.n, active, na, q, w.k, out=out)   # first call: one-time set-up
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    fathom.scan_topk_noalloc(planes, scales, w.n, active, na, q, w.k, out=out)
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    assert free0 == free1
    assert torch.all(out[2] >= 0)
    # The call also captures into a CUDA graph (no allocation, no implicit
    # synchronisation) and the replay gives the same result.
    ref = tuple(t.clone() for t in out)
    for t in out:
        t.fill_(-7)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side), torch.cuda.graph(graph, stream=side):
        fathom.scan_topk_noalloc(planes, scales, w.n, active, na, q, w.k, out=out, stream=side)
    graph.replay()
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(out, ref))
    del graph
    lib = fathom.lib()
    misaligned = ctypes.c_void_p(out[0].data_ptr() + 2)
    st = lib.fathom_scan_topk_noalloc(fathom._p(planes), fathom._p(scales), w.H, w.D, w.n, planes.shape[-1],
                                      fathom._p(active), fathom._p(na), fathom._p(q), w.G, w.k, misaligned,
                                      fathom._p(out[1]), fathom._p(out[2]), fathom._stream(None))
    assert st == fathom.ERR_UNSUPPORTED
