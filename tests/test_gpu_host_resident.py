"""Host-resident index: planes and scales in page-locked host memory, read
by the scan kernel over the host link through its device mapping (zero
copy).  Results must be bit-identical to the device-resident run, and
ordinary pageable host memory must be rejected before any launch."""
import dataclasses

import pytest
import torch

from long_context_decode_bit_b200 import inputs

pytestmark = pytest.mark.gpu


def test_host_resident_index_matches_device_resident(fathom_gpu):
    fathom = fathom_gpu
    w = dataclasses.replace(inputs.LAYER_32K, H=4, n=70000, seed=51)
    k = inputs.keys(w, 0, w.H, device="cuda")
    q = inputs.queries(w, 0, w.H, device="cuda").float().contiguous()
    s2 = inputs.calibration_sigma2(k, w.n_cal).contiguous()
    planes, scales = fathom.pack(k)
    hp = torch.empty(planes.shape, dtype=planes.dtype, pin_memory=True)
    hs = torch.empty(scales.shape, dtype=scales.dtype, pin_memory=True)
    hp.copy_(planes)
    hs.copy_(scales)
    dev_step = fathom.Step(planes, scales, w.n, s2, w.G, w.k, budget=48)
    host_step = fathom.Step(hp, hs, w.n, s2, w.G, w.k, budget=48)
    a = dev_step.run(q)
    b = host_step.run(q)
    _, active, na, _ = dev_step.plan_out
    dense_dev = fathom.scan(planes, scales, w.n, active, na, q)
    dense_host = fathom.scan(hp, hs, w.n, active, na, q)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert torch.equal(dense_dev, dense_host)


def test_pageable_host_index_is_rejected(fathom_gpu):
    fathom = fathom_gpu
    w = dataclasses.replace(inputs.TINY, H=1, n=1024, n_cal=1024)
    k = inputs.keys(w, 0, 1, device="cuda")
    q = inputs.queries(w, 0, 1, device="cuda").float().contiguous()
    s2 = inputs.calibration_sigma2(k, w.n_cal).contiguous()
    planes, scales = fathom.pack(k)
    _, active, na, _ = fathom.plan(s2, q, 48)
    with pytest.raises(fathom.FathomError) as e:
        fathom.scan(planes.cpu(), scales.cpu(), w.n, active, na, q)   # pageable: not device-visible
    assert e.value.status == fathom.ERR_INVALID_ARG
