"""Fathom key-scan oracle: TEST INFRASTRUCTURE ONLY.

numpy front end over ``liboracle.so`` (plain C, fp64; see
``fathom_oracle.c``).  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the product path
never does.

Functions follow the paper "Fathom: Per-Query Read Depth for Sparse
Decoding over Offloaded KV Caches" (arXiv 2609.17652) as retold on the
yeyulingfeng.com article, sections "方法一" (4-bit codes stored as bit
planes) and "方法二" (per-group reverse water-filling).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        lib.orc_fp16_bits.restype = ctypes.c_uint16
        lib.orc_fp16_bits.argtypes = [ctypes.c_double]
        lib.orc_fp16_value.restype = ctypes.c_double
        lib.orc_fp16_value.argtypes = [ctypes.c_uint16]
        lib.orc_code4.restype = I
        lib.orc_code4.argtypes = [ctypes.c_double, ctypes.c_double]
        lib.orc_dequant.restype = ctypes.c_double
        lib.orc_dequant.argtypes = [I, I, ctypes.c_double]
        lib.orc_pack.restype = I
        lib.orc_pack.argtypes = [P, I, I64, I64, I, I64, I64, P, P, I64]
        lib.orc_importance.restype = ctypes.c_float
        lib.orc_importance.argtypes = [P, P, I, I64]
        lib.orc_plan.restype = I
        lib.orc_plan.argtypes = [P, P, I64, I, I, P, P, P, P, P, P]
        lib.orc_plan_fixed.restype = I
        lib.orc_plan_fixed.argtypes = [P, I64, I, I, I, I, P, P, P]
        lib.orc_scan.restype = I
        lib.orc_scan.argtypes = [P, P, I64, I, I64, I64, P, P, I, P, P]
        lib.orc_topk.restype = I
        lib.orc_topk.argtypes = [P, I64, I, I64, I, P, P, P]
        lib.orc_dequant_rows.restype = I
        lib.orc_dequant_rows.argtypes = [P, P, I64, I, I64, I64, P, I64, P, I, P]
        lib.orc_calibrate.restype = I
        lib.orc_calibrate.argtypes = [P, I, I64, I64, I, I64, I64, P, P, P]
        lib.orc_layer_budgets.restype = I
        lib.orc_layer_budgets.argtypes = [P, P, I64, I, I, I, I64, P]
        lib.orc_pack_nibbles.restype = I
        lib.orc_pack_nibbles.argtypes = [P, I, I64, I64, I, I64, I64, P, I64]
        lib.orc_rotate_keys.restype = I
        lib.orc_rotate_keys.argtypes = [P, I, I64, I64, I, I64, I64, P, P]
        lib.orc_union_attention.restype = I
        lib.orc_union_attention.argtypes = [P, P, I, I64, I64, I, I64, I64, P, I, P, P, I64, ctypes.c_double, P]
        _LIB = lib
    return _LIB


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with status {rc}")


def fp16_bits(x: float) -> int:
    """IEEE binary16 round-to-nearest-even of ``x`` (bit pattern)."""
    return int(_lib().orc_fp16_bits(float(x)))


def fp16_value(bits: int) -> float:
    return float(_lib().orc_fp16_value(int(bits)))


def code4(k: float, s: float) -> int:
    """4-bit uniform symmetric code of value ``k`` under block scale ``s``."""
    return int(_lib().orc_code4(float(k), float(s)))


def dequant(c4: int, t: int, s: float) -> float:
    """Value of the first ``t`` planes of code ``c4`` under scale ``s``."""
    return float(_lib().orc_dequant(int(c4), int(t), float(s)))


def pack(keys: np.ndarray, nb_stride: int | None = None):
    """Quantise keys [H][n][D] (float32 values, or uint16 bf16 bit patterns)
    into planes uint64 [H][D][4][nb_stride] and fp16 scale bits
    uint16 [H][D][nb_stride]."""
    keys = np.ascontiguousarray(keys)
    if keys.dtype == np.float32:
        dt = 0
    elif keys.dtype == np.uint16:
        dt = 1
    else:
        raise TypeError("keys must be float32 or uint16 (bf16 bits)")
    H, n, D = keys.shape
    nb = (n + 63) // 64
    nbs = nb if nb_stride is None else int(nb_stride)
    planes = np.zeros((H, D, 4, nbs), dtype=np.uint64)
    scales = np.zeros((H, D, nbs), dtype=np.uint16)
    _check(_lib().orc_pack(_ptr(keys), dt, H, n, D, n * D, D, _ptr(planes), _ptr(scales), nbs), "pack")
    return planes, scales


def rotate_keys(keys: np.ndarray, U: np.ndarray) -> np.ndarray:
    """Coordinates y [H][n][D] (float32) of keys [H][n][D] (float32, or uint16
    bf16 bit patterns) in the basis U [H][D][D] (float32, U[h][d][i] =
    component d of direction i): y_i = sum_d k_d U[d][i] summed over
    d = 0..D-1 in order, one fp32 fused multiply-add per step."""
    keys = np.ascontiguousarray(keys)
    if keys.dtype == np.float32:
        dt = 0
    elif keys.dtype == np.uint16:
        dt = 1
    else:
        raise TypeError("keys must be float32 or uint16 (bf16 bits)")
    H, n, D = keys.shape
    U = np.ascontiguousarray(U, dtype=np.float32)
    if U.shape != (H, D, D):
        raise ValueError("U must be [H][D][D]")
    out = np.zeros((H, n, D), dtype=np.float32)
    _check(_lib().orc_rotate_keys(_ptr(keys), dt, H, n, D, n * D, D, _ptr(U), _ptr(out)), "rotate_keys")
    return out


def pack_rotated(keys: np.ndarray, U: np.ndarray, nb_stride: int | None = None):
    """The index of the keys' coordinates in the basis U: pack(rotate_keys)."""
    return pack(rotate_keys(keys, U), nb_stride=nb_stride)


def importance(sigma2: np.ndarray, q: np.ndarray) -> np.ndarray:
    """w [H][D] in the plan's single-precision order."""
    sigma2 = np.ascontiguousarray(sigma2, dtype=np.float32)
    q = np.ascontiguousarray(q, dtype=np.float32)
    H, G, D = q.shape
    depth = np.zeros((H, D), dtype=np.uint8)
    w = np.zeros((H, D), dtype=np.float32)
    budget = np.zeros(H, dtype=np.int32)
    _check(_lib().orc_plan(_ptr(sigma2), _ptr(q), H, G, D, _ptr(budget), _ptr(depth),
                           None, None, None, _ptr(w)), "importance")
    return w


def plan(sigma2: np.ndarray, q: np.ndarray, budget):
    """Reverse water-filling plan.  Returns (depth uint8 [H][D],
    active uint16 [H][D] (j | t<<8, ascending j, zero padded),
    n_active int32 [H], theta float64 [H])."""
    sigma2 = np.ascontiguousarray(sigma2, dtype=np.float32)
    q = np.ascontiguousarray(q, dtype=np.float32)
    H, G, D = q.shape
    budget = np.broadcast_to(np.asarray(budget, dtype=np.int32), (H,)).copy()
    depth = np.zeros((H, D), dtype=np.uint8)
    active = np.zeros((H, D), dtype=np.uint16)
    n_active = np.zeros(H, dtype=np.int32)
    theta = np.zeros(H, dtype=np.float64)
    _check(_lib().orc_plan(_ptr(sigma2), _ptr(q), H, G, D, _ptr(budget), _ptr(depth),
                           _ptr(active), _ptr(n_active), _ptr(theta), None), "plan")
    return depth, active, n_active, theta


def plan_fixed(q: np.ndarray, r: int, bits: int = 4):
    """Fixed-depth plan: the r channels with the largest sum_g |q| at ``bits`` planes."""
    q = np.ascontiguousarray(q, dtype=np.float32)
    H, G, D = q.shape
    depth = np.zeros((H, D), dtype=np.uint8)
    active = np.zeros((H, D), dtype=np.uint16)
    n_active = np.zeros(H, dtype=np.int32)
    _check(_lib().orc_plan_fixed(_ptr(q), H, G, D, int(r), int(bits), _ptr(depth), _ptr(active),
                                 _ptr(n_active)), "plan_fixed")
    return depth, active, n_active


def scan(planes: np.ndarray, scales: np.ndarray, depth: np.ndarray, q: np.ndarray, n: int,
         with_l1: bool = True):
    """fp64 scores [H][G][n] (and the per-score sum of |terms| if asked)."""
    planes = np.ascontiguousarray(planes, dtype=np.uint64)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    depth = np.ascontiguousarray(depth, dtype=np.uint8)
    q = np.ascontiguousarray(q, dtype=np.float32)
    H, G, D = q.shape
    nbs = planes.shape[-1]
    scores = np.zeros((H, G, n), dtype=np.float64)
    l1 = np.zeros((H, G, n), dtype=np.float64) if with_l1 else None
    _check(_lib().orc_scan(_ptr(planes), _ptr(scales), H, D, n, nbs, _ptr(depth), _ptr(q), G,
                           _ptr(scores), _ptr(l1) if with_l1 else None), "scan")
    return (scores, l1) if with_l1 else scores


def topk(scores: np.ndarray, k: int):
    """Per-head top-k by (score desc, index asc) and the per-group union.
    Returns (idx int32 [H][G][k], union int32 [H][G*k] (-1 padded), count int32 [H])."""
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    H, G, n = scores.shape
    idx = np.zeros((H, G, k), dtype=np.int32)
    uni = np.zeros((H, G * k), dtype=np.int32)
    cnt = np.zeros(H, dtype=np.int32)
    _check(_lib().orc_topk(_ptr(scores), H, G, n, int(k), _ptr(idx), _ptr(uni), _ptr(cnt)), "topk")
    return idx, uni, cnt


def dequant_rows(planes: np.ndarray, scales: np.ndarray, n: int, rows: np.ndarray, row_count=None, bits: int = 4):
    """fp64 key rows [H][M][D] rebuilt from the planes at ``bits`` planes."""
    planes = np.ascontiguousarray(planes, dtype=np.uint64)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    H, D = planes.shape[0], planes.shape[1]
    M = rows.shape[1]
    rc = None if row_count is None else np.ascontiguousarray(row_count, dtype=np.int32)
    out = np.zeros((H, M, D), dtype=np.float64)
    _check(_lib().orc_dequant_rows(_ptr(planes), _ptr(scales), H, D, n, planes.shape[-1], _ptr(rows), M,
                                   None if rc is None else _ptr(rc), int(bits), _ptr(out)), "dequant_rows")
    return out


def calibrate(keys: np.ndarray, n: int | None = None, with_cov: bool = True):
    """fp64 (mean [H][D], population variance [H][D], covariance [H][D][D] or
    None) of each group's first n keys; keys [H][n_total][D] float32 or
    uint16 bf16 bit patterns."""
    keys = np.ascontiguousarray(keys)
    if keys.dtype == np.float32:
        dt = 0
    elif keys.dtype == np.uint16:
        dt = 1
    else:
        raise TypeError("keys must be float32 or uint16 (bf16 bits)")
    H, nt, D = keys.shape
    n = nt if n is None else int(n)
    mean = np.zeros((H, D), dtype=np.float64)
    var = np.zeros((H, D), dtype=np.float64)
    cov = np.zeros((H, D, D), dtype=np.float64) if with_cov else None
    _check(_lib().orc_calibrate(_ptr(keys), dt, H, n, D, nt * D, D, _ptr(mean), _ptr(var),
                                _ptr(cov) if with_cov else None), "calibrate")
    return mean, var, cov


def union_attention(k: np.ndarray, v: np.ndarray, q: np.ndarray, uni: np.ndarray, count: np.ndarray,
                    scale: float | None = None):
    """fp64 softmax attention [H][G][D] of each query head over its group's
    union rows; k, v [H][n][D] float32 or uint16 bf16 bits (same dtype)."""
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    if k.dtype != v.dtype or k.shape != v.shape:
        raise TypeError("k and v must share dtype and shape")
    dt = {np.dtype(np.float32): 0, np.dtype(np.uint16): 1}[k.dtype]
    q = np.ascontiguousarray(q, dtype=np.float32)
    uni = np.ascontiguousarray(uni, dtype=np.int32)
    count = np.ascontiguousarray(count, dtype=np.int32)
    H, n, D = k.shape
    G = q.shape[1]
    M = uni.shape[1]
    sc = 1.0 / np.sqrt(D) if scale is None else float(scale)
    out = np.zeros((H, G, D), dtype=np.float64)
    _check(_lib().orc_union_attention(_ptr(k), _ptr(v), dt, H, n, D, n * D, D, _ptr(q), G, _ptr(uni), _ptr(count),
                                      M, sc, _ptr(out)), "union_attention")
    return out


def pack_nibbles(keys: np.ndarray, nb_stride: int | None = None) -> np.ndarray:
    """The 4-bit codes of ``pack`` stored whole: uint64 [H][D][4][nb_stride],
    word w of a block holding its tokens 16w..16w+15, 4 bits each."""
    keys = np.ascontiguousarray(keys)
    dt = {np.dtype(np.float32): 0, np.dtype(np.uint16): 1}[keys.dtype]
    H, n, D = keys.shape
    nb = (n + 63) // 64
    nbs = nb if nb_stride is None else int(nb_stride)
    nib = np.zeros((H, D, 4, nbs), dtype=np.uint64)
    _check(_lib().orc_pack_nibbles(_ptr(keys), dt, H, n, D, n * D, D, _ptr(nib), nbs), "pack_nibbles")
    return nib


def layer_budgets(sigma2: np.ndarray, q: np.ndarray, layers: int, total_bits: int) -> np.ndarray:
    """Greedy per-layer split of ``total_bits`` plane bits: int32 [H], the
    budget of each group (equal within a layer of H/layers groups)."""
    sigma2 = np.ascontiguousarray(sigma2, dtype=np.float32)
    q = np.ascontiguousarray(q, dtype=np.float32)
    H, G, D = q.shape
    out = np.zeros(H, dtype=np.int32)
    _check(_lib().orc_layer_budgets(_ptr(sigma2), _ptr(q), H, G, D, int(layers), int(total_bits), _ptr(out)),
           "layer_budgets")
    return out
