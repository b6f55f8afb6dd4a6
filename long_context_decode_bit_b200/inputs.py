"""Seeded synthetic inputs for the Fathom key scan.

This module draws random numbers and nothing else: keys, queries, the
calibration statistic sigma^2, budgets and session lengths.  It holds none
of the scan's arithmetic, so both the CUDA path and the CPU oracle can take
their inputs from it.

Every tensor is generated per group (one group = one layer x KV head) from
its own seed, so any subset of groups can be regenerated on its own, on
the CPU or on the GPU (torch's CPU and CUDA generators give different
streams; callers compare the two implementations on the same tensor, never
across devices).

Workload shapes follow the paper's Qwen3-8B setting (36 layers x 8 KV heads,
4 query heads per KV head, 128 channels; yeyulingfeng.com article, section
"先算一笔字节账").  No model weights or text exist here: keys and queries are
random with the structure described below.
"""
from __future__ import annotations

import dataclasses

import torch

HEAD_DIM = 128
GQA = 4


@dataclasses.dataclass(frozen=True)
class Workload:
    """One scan workload.  ``kind`` selects the key/query recipe:

    ``"gauss"``  fp32 keys N(0, std_j^2), std_j ~ logN(0, 1), plus
                 ``n_outlier`` channels at 8x std; fp32 queries N(0, 1).
    ``"qknorm"`` bf16 keys z ~ N(0, I), each token rescaled to unit RMS
                 (flat channel scales, as under QK-norm); bf16 queries
                 N(0, 1) with 8..12 dominant channels per group at 5x,
                 shared by the group's query heads.
    ``"corr"``   bf16 keys without QK-norm: z ~ N(0, I) mixed by a random
                 rotation and a decaying spectrum (per group), so channel
                 variances are uneven and channels correlated; queries as
                 for ``qknorm``.
    """
    name: str
    H: int
    n: int
    D: int = HEAD_DIM
    G: int = GQA
    kind: str = "qknorm"
    n_cal: int = 4096
    budgets: tuple = (48,)
    k: int = 512
    seed: int = 0
    n_outlier: int = 4

    @property
    def nb(self) -> int:
        return (self.n + 63) // 64


TINY = Workload("tiny-1x4096-gauss", H=1, n=4096, kind="gauss", n_cal=1024, budgets=(48,), k=64, seed=0)
LAYER_32K = Workload("qwen3-8b-layer-8x32768", H=8, n=32768, budgets=(48, 68, 92, 136), k=512, seed=1)
STEP_128K = Workload("qwen3-8b-step-288x131072", H=288, n=131072, budgets=(48,), k=512, seed=2)
STEP_1M = Workload("qwen3-8b-step-288x1048576", H=288, n=1048576, budgets=(48, 92, 136), k=512, seed=3)
STEP_1M_LLAMA = Workload("llama3.1-8b-step-256x1048576", H=256, n=1048576, kind="corr", budgets=(48, 92, 136),
                         k=512, seed=4)

WORKLOADS = {w.name: w for w in (TINY, LAYER_32K, STEP_128K, STEP_1M, STEP_1M_LLAMA)}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def _group_seed(w: Workload, h: int, stream: int) -> int:
    return (w.seed * 1_000_003 + h) * 16 + stream


def keys(w: Workload, h0: int, h1: int, device="cpu") -> torch.Tensor:
    """Keys of groups [h0, h1) as a [h1-h0][n][D] tensor (fp32 for
    ``gauss``, bf16 for ``qknorm``)."""
    n = w.n
    out = []
    for h in range(h0, h1):
        if w.kind == "gauss":
            g = _gen(device, _group_seed(w, h, 0))
            std = torch.exp(torch.randn(w.D, generator=g, device=device))
            outl = torch.randperm(w.D, generator=g, device=device)[: w.n_outlier]
            std[outl] *= 8.0
            z = torch.randn(n, w.D, generator=g, device=device)
            out.append((z * std).to(torch.float32))
        elif w.kind == "qknorm":
            g = _gen(device, _group_seed(w, h, 0))
            z = torch.randn(n, w.D, generator=g, device=device)
            rms = torch.sqrt(torch.mean(z * z, dim=1, keepdim=True))
            out.append((z / rms).to(torch.bfloat16))
        elif w.kind == "corr":
            g = _gen(device, _group_seed(w, h, 0))
            rot, _ = torch.linalg.qr(torch.randn(w.D, w.D, generator=g, device=device))
            spectrum = torch.exp(-torch.arange(w.D, device=device, dtype=torch.float32) / 24.0)
            mix = rot * torch.sqrt(spectrum)[None, :]
            z = torch.randn(n, w.D, generator=g, device=device)
            out.append((z @ mix.T).to(torch.bfloat16))
        else:
            raise ValueError(w.kind)
    return torch.stack(out, 0)


def queries(w: Workload, h0: int, h1: int, device="cpu") -> torch.Tensor:
    """Queries of groups [h0, h1) as [h1-h0][G][D] (fp32 for ``gauss``;
    bf16 values for ``qknorm``, returned as bf16)."""
    out = []
    for h in range(h0, h1):
        g = _gen(device, _group_seed(w, h, 1))
        q = torch.randn(w.G, w.D, generator=g, device=device)
        if w.kind in ("qknorm", "corr"):
            m = int(torch.randint(8, 13, (1,), generator=g, device=device).item())
            dom = torch.randperm(w.D, generator=g, device=device)[:m]
            q[:, dom] *= 5.0
            out.append(q.to(torch.bfloat16))
        else:
            out.append(q.to(torch.float32))
    return torch.stack(out, 0)


def values(w: Workload, h0: int, h1: int, device="cpu") -> torch.Tensor:
    """Value rows of groups [h0, h1) as [h1-h0][n][D], N(0, 1), in the keys'
    dtype: the synthetic V cache that attention over the winners reads."""
    out = []
    for h in range(h0, h1):
        g = _gen(device, _group_seed(w, h, 2))
        z = torch.randn(w.n, w.D, generator=g, device=device)
        out.append(z.to(torch.float32 if w.kind == "gauss" else torch.bfloat16))
    return torch.stack(out, 0)


def calibration_sigma2(k: torch.Tensor, n_cal: int) -> torch.Tensor:
    """sigma_j^2 per group: the population variance over the first ``n_cal``
    keys of each channel, accumulated in fp64 and rounded to fp32.  This is
    the calibration statistic the plan takes as input; the paper measures
    it once, on calibration keys, outside the per-step path."""
    x = k[:, :n_cal, :].to(torch.float64)
    return x.var(dim=1, unbiased=False).to(torch.float32)


def sigma2(w: Workload, h0: int, h1: int, device="cpu") -> torch.Tensor:
    """sigma^2 [h1-h0][D] from the first ``n_cal`` keys of each group."""
    return calibration_sigma2(keys(w, h0, h1, device=device), w.n_cal)


def session_lengths(n_sessions: int, lo: int, hi: int, seed: int) -> list[int]:
    """Lengths drawn uniformly from [lo, hi] (multi-session host-resident case)."""
    g = _gen("cpu", seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (n_sessions,), generator=g)]


def bf16_bits(t: torch.Tensor):
    """Raw uint16 bit patterns of a bf16 tensor, as a numpy array."""
    return t.contiguous().view(torch.int16).cpu().numpy().view("uint16")
