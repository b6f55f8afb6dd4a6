"""Shared helpers for the parity tests (host side only)."""
import numpy as np
import torch

SCORE_RTOL = 1e-5   # |gpu - oracle| <= 1e-5 * sum_j |q_j khat_j| (the score's L1 scale)


def np_u64(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint64)


def np_u16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def keys_for_oracle(k: torch.Tensor) -> np.ndarray:
    """fp32 values, or bf16 bit patterns, exactly as the GPU saw them."""
    if k.dtype == torch.bfloat16:
        return k.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return k.float().cpu().numpy()


def depth_to_active(depth: np.ndarray):
    H, D = depth.shape
    act = np.zeros((H, D), np.uint16)
    na = np.zeros(H, np.int32)
    for h in range(H):
        js = np.nonzero(depth[h])[0]
        na[h] = len(js)
        act[h, :len(js)] = js | (depth[h, js].astype(np.int64) << 8)
    return act, na


def assert_scores_close(gpu: np.ndarray, ref: np.ndarray, l1: np.ndarray, rtol: float = SCORE_RTOL):
    gpu = gpu.astype(np.float64)
    err = np.abs(gpu - ref)
    bound = rtol * l1
    bad = err > bound
    if np.any(bad):
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{int(bad.sum())} scores out of tolerance; first at {tuple(i)}: "
                             f"gpu={gpu[tuple(i)]!r} ref={ref[tuple(i)]!r} l1={l1[tuple(i)]!r}")


def lexsort_topk(scores: np.ndarray, k: int) -> np.ndarray:
    """Top-k of one row by (score desc, index asc), exactly."""
    n = scores.shape[-1]
    return np.lexsort((np.arange(n), -scores.astype(np.float64)))[:k]


def assert_topk_sets_match(gpu_idx, ref_idx, ref_scores, l1, k: int, rtol: float = SCORE_RTOL):
    """Sets equal except for keys whose oracle score is within the score
    tolerance of the oracle's k-th score (either side may hold those)."""
    H, G, _ = gpu_idx.shape
    for h in range(H):
        for g in range(G):
            a, b = set(gpu_idx[h, g].tolist()), set(ref_idx[h, g].tolist())
            if a == b:
                continue
            kth = ref_idx[h, g, k - 1]
            s_k = ref_scores[h, g, kth]
            for i in a ^ b:
                gap = abs(ref_scores[h, g, i] - s_k)
                assert gap <= rtol * (l1[h, g, i] + l1[h, g, kth]), (h, g, i, gap)
