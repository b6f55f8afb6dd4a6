"""The seeded input generators (CPU): every group is drawn from its own seed,
so any subset of groups regenerates identically on its own; the recipes
have the shapes, dtypes and structure the workloads state."""
import dataclasses

import torch

from long_context_decode_bit_b200 import inputs


def test_groups_regenerate_alone():
    w = dataclasses.replace(inputs.LAYER_32K, n=256, H=4)
    allk = inputs.keys(w, 0, 4)
    assert torch.equal(inputs.keys(w, 2, 3), allk[2:3])
    assert torch.equal(inputs.queries(w, 1, 3), inputs.queries(w, 0, 4)[1:3])
    assert torch.equal(inputs.values(w, 3, 4), inputs.values(w, 0, 4)[3:4])
    assert not torch.equal(inputs.values(w, 0, 1).float(), allk[0:1].float())   # its own seed stream


def test_recipes_match_their_description():
    w = dataclasses.replace(inputs.LAYER_32K, n=512, H=2)
    k = inputs.keys(w, 0, 2)
    assert k.dtype == torch.bfloat16 and k.shape == (2, 512, 128)
    rms = k.float().pow(2).mean(-1).sqrt()
    assert torch.allclose(rms, torch.ones_like(rms), atol=1e-2)   # unit RMS per token (QK-norm-like)
    q = inputs.queries(w, 0, 2).float()
    big = (q.abs() > 0).float()
    assert q.shape == (2, 4, 128) and big.all()
    t = dataclasses.replace(inputs.TINY, n=4096)
    kt = inputs.keys(t, 0, 1)
    assert kt.dtype == torch.float32
    std = kt[0].std(0)
    assert (std.max() / std.median()) > 4.0          # outlier channels at 8x, log-normal spread
    v = inputs.values(t, 0, 1)
    assert v.dtype == torch.float32 and abs(v.mean().item()) < 0.05 and abs(v.std().item() - 1.0) < 0.05
    c = dataclasses.replace(inputs.STEP_1M_LLAMA, n=2048, H=1)
    kc = inputs.keys(c, 0, 1)[0].float()
    var = kc.var(0)
    assert var.max() / var.min() > 1.5               # uneven channel variances (no QK-norm)
    ev = torch.linalg.eigvalsh(torch.cov(kc.T.double()))
    assert ev.max() / ev.min() > 50.0                # ... and correlated: a decaying spectrum that a rotation concentrates
    assert inputs.calibration_sigma2(inputs.keys(t, 0, 1), 1024).shape == (1, 128)
