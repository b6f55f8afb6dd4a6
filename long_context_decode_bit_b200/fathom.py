"""ctypes binding of ``libfathom.so`` (C ABI in ``include/fathom.h``).

Argument marshalling only: every step of the scan runs in the library's
CUDA kernels.  torch tensors supply device memory and the current stream;
outputs are allocated here with torch when the caller does not pass them.
If the library is missing or cannot be loaded, every call raises -- there
is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfathom.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_CUDA = -3
ERR_WORKSPACE = -4
ERR_TIMEOUT = -5
ERR_OVERFLOW = -6
ERR_BOUNDS = -7   # debug build: a device-side bounds check failed

KEYS_F32 = 0
KEYS_BF16 = 1
SCAN_DENSE = 0
SCAN_CANDIDATE = 1
SCAN_PREPARE = 2
SCAN_FILTER = 3

# Every symbol include/fathom.h declares.
EXPORTS = (
    "fathom_version", "fathom_status_string", "fathom_last_cuda_error", "fathom_nb_stride",
    "fathom_pack", "fathom_plan", "fathom_plan_fixed", "fathom_scan_cand_bytes", "fathom_scan",
    "fathom_topk_workspace_bytes", "fathom_topk", "fathom_dequant_rows", "fathom_scan_topk_noalloc",
    "fathom_device_status", "fathom_calibrate_workspace_bytes", "fathom_calibrate",
    "fathom_union_attention_workspace_bytes", "fathom_union_attention",
    "fathom_nibbles_from_planes", "fathom_scan_nibbles", "fathom_layer_budgets_workspace_bytes",
    "fathom_layer_budgets", "fathom_pack_rotated", "fathom_nibbles_tm_from_planes", "fathom_scan_nibbles_tm",
)

NOALLOC_SCRATCH_BYTES = 16 << 20

_lib = None


class FathomError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {_lib.fathom_status_string(status).decode() if _lib else status}"
        if status == ERR_CUDA and _lib is not None:
            msg += f" (cudaError {_lib.fathom_last_cuda_error()})"
        super().__init__(msg)


def load(path: str | None = None):
    """Load the shared library (raises if it is missing).  ``FATHOM_LIB``
    may name another build of it."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or os.environ.get("FATHOM_LIB") or LIB_PATH
    if not os.path.exists(path):
        raise FileNotFoundError(
            f"{path} is missing: build it with `python -m long_context_decode_bit_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "fathom_version": (I, []),
        "fathom_status_string": (ctypes.c_char_p, [I]),
        "fathom_last_cuda_error": (I, []),
        "fathom_nb_stride": (I64, [I64]),
        "fathom_pack": (I, [P, I, I64, I64, I, I64, I64, P, P, I64, P]),
        "fathom_plan": (I, [P, P, I64, I, I, P, ctypes.c_int32, P, P, P, P, P]),
        "fathom_plan_fixed": (I, [P, I64, I, I, I, I, P, P, P, P]),
        "fathom_scan_cand_bytes": (SZ, [I64, I, I64, I]),
        "fathom_scan": (I, [P, P, I64, I, I64, I64, P, P, P, I, I, P, P, SZ, I, P]),
        "fathom_topk_workspace_bytes": (SZ, [I64, I, I64, I]),
        "fathom_topk": (I, [P, P, I64, I, I64, I, P, P, P, P, SZ, P]),
        "fathom_dequant_rows": (I, [P, P, I64, I, I64, I64, P, I64, P, I, P, P]),
        "fathom_scan_topk_noalloc": (I, [P, P, I64, I, I64, I64, P, P, P, I, I, P, P, P, P]),
        "fathom_device_status": (I, [I, P]),
        "fathom_pack_rotated": (I, [P, I, I64, I64, I, I64, I64, P, P, P, I64, P]),
        "fathom_nibbles_tm_from_planes": (I, [P, I64, I, I64, I64, P, P]),
        "fathom_scan_nibbles_tm": (I, [P, P, I64, I, I64, I64, P, P, P, I, I, P, P, SZ, I, P]),
        "fathom_calibrate_workspace_bytes": (SZ, [I64, I, I]),
        "fathom_calibrate": (I, [P, I, I64, I64, I, I64, I64, P, P, P, P, SZ, P]),
        "fathom_union_attention_workspace_bytes": (SZ, [I64, I, I, I64]),
        "fathom_nibbles_from_planes": (I, [P, I64, I, I64, I64, P, P]),
        "fathom_layer_budgets_workspace_bytes": (SZ, [I64, I]),
        "fathom_layer_budgets": (I, [P, P, I64, I, I, I, I64, P, P, SZ, P]),
        "fathom_scan_nibbles": (I, [P, P, I64, I, I64, I64, P, P, P, I, I, P, P, SZ, I, P]),
        "fathom_union_attention": (I, [P, P, I, I64, I64, I, I64, I64, P, I, P, P, I64, ctypes.c_float, P, P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def lib():
    return load()


def _check(st: int, what: str):
    if st != OK:
        raise FathomError(st, what)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def nb_stride(n: int) -> int:
    return int(lib().fathom_nb_stride(int(n)))


def scan_cand_bytes(H: int, G: int, n: int, k: int) -> int:
    return int(lib().fathom_scan_cand_bytes(H, G, n, k))


def topk_workspace_bytes(H: int, G: int, n: int, k: int) -> int:
    return int(lib().fathom_topk_workspace_bytes(H, G, n, k))


def pack(keys: torch.Tensor, nb_stride_words: int | None = None, planes=None, scales=None, stream=None):
    """Bit-plane index of keys [H][n][D] (fp32 or bf16, channels contiguous).
    Returns (planes uint64-as-int64 [H][D][4][nb_stride], scales int16 [H][D][nb_stride])."""
    H, n, D = keys.shape
    if keys.stride(2) != 1:
        raise ValueError("keys must be contiguous along channels")
    dt = {torch.float32: KEYS_F32, torch.bfloat16: KEYS_BF16}[keys.dtype]
    nbs = nb_stride(n) if nb_stride_words is None else int(nb_stride_words)
    dev = keys.device
    if planes is None:
        planes = torch.zeros((H, D, 4, nbs), dtype=torch.int64, device=dev)
    if scales is None:
        scales = torch.zeros((H, D, nbs), dtype=torch.int16, device=dev)
    _check(lib().fathom_pack(_p(keys), dt, H, n, D, keys.stride(0), keys.stride(1), _p(planes), _p(scales),
                             nbs, _stream(stream)), "fathom_pack")
    return planes, scales


def pack_rotated(keys: torch.Tensor, U: torch.Tensor, nb_stride_words: int | None = None, planes=None, scales=None,
                 stream=None):
    """Bit-plane index of the keys' coordinates in the basis U [H][D][D]
    (fp32, columns = directions), rotated inside the kernel in a fixed fp32
    fused multiply-add order (see fathom_pack_rotated in include/fathom.h)."""
    H, n, D = keys.shape
    if keys.stride(2) != 1:
        raise ValueError("keys must be contiguous along channels")
    if U.dtype != torch.float32 or tuple(U.shape) != (H, D, D) or not U.is_contiguous():
        raise ValueError("U must be a contiguous fp32 [H][D][D] tensor")
    dt = {torch.float32: KEYS_F32, torch.bfloat16: KEYS_BF16}[keys.dtype]
    nbs = nb_stride(n) if nb_stride_words is None else int(nb_stride_words)
    dev = keys.device
    if planes is None:
        planes = torch.zeros((H, D, 4, nbs), dtype=torch.int64, device=dev)
    if scales is None:
        scales = torch.zeros((H, D, nbs), dtype=torch.int16, device=dev)
    _check(lib().fathom_pack_rotated(_p(keys), dt, H, n, D, keys.stride(0), keys.stride(1), _p(U), _p(planes),
                                     _p(scales), nbs, _stream(stream)), "fathom_pack_rotated")
    return planes, scales


def pack_range(keys: torch.Tensor, planes: torch.Tensor, scales: torch.Tensor, block0: int, stream=None):
    """(Re)pack blocks block0.. of an existing index from ``keys`` [H][m][D],
    the keys of tokens 64*block0 .. 64*block0 + m - 1 (appending to the tail
    block during decode).  ``planes``/``scales`` are the whole index."""
    H, m, D = keys.shape
    if keys.stride(2) != 1:
        raise ValueError("keys must be contiguous along channels")
    dt = {torch.float32: KEYS_F32, torch.bfloat16: KEYS_BF16}[keys.dtype]
    nbs = planes.shape[-1]
    if block0 < 0 or block0 + (m + 63) // 64 > nbs:
        raise ValueError("block range outside the index")
    pp = ctypes.c_void_p(planes.data_ptr() + 8 * block0)
    sp = ctypes.c_void_p(scales.data_ptr() + 2 * block0)
    _check(lib().fathom_pack(_p(keys), dt, H, m, D, keys.stride(0), keys.stride(1), pp, sp, nbs, _stream(stream)),
           "fathom_pack")
    return planes, scales


def plan(sigma2: torch.Tensor, q: torch.Tensor, budget, out=None, stream=None):
    """Reverse water-filling plan.  ``budget`` is an int (flat) or an int32
    device tensor [H].  Returns (depth uint8 [H][D], active int16 [H][D],
    n_active int32 [H], theta fp32 [H])."""
    H, G, D = q.shape
    dev = q.device
    if out is None:
        out = (torch.empty((H, D), dtype=torch.uint8, device=dev), torch.empty((H, D), dtype=torch.int16, device=dev),
               torch.empty(H, dtype=torch.int32, device=dev), torch.empty(H, dtype=torch.float32, device=dev))
    depth, active, n_active, theta = out
    if isinstance(budget, torch.Tensor):
        bptr, flat = _p(budget), 0
    else:
        bptr, flat = None, int(budget)
    _check(lib().fathom_plan(_p(sigma2), _p(q), H, G, D, bptr, flat, _p(depth), _p(active), _p(n_active),
                             _p(theta), _stream(stream)), "fathom_plan")
    return depth, active, n_active, theta


def layer_budgets(sigma2: torch.Tensor, q: torch.Tensor, layers: int, total_bits: int, out=None, stream=None):
    """Greedy per-layer split of ``total_bits`` plane bits from calibration
    queries q [H][G][D]: int32 [H] budgets for ``plan``."""
    H, G, D = q.shape
    dev = q.device
    if out is None:
        out = torch.empty(H, dtype=torch.int32, device=dev)
    ws = torch.empty(max(int(lib().fathom_layer_budgets_workspace_bytes(H, D)), 1), dtype=torch.uint8, device=dev)
    _check(lib().fathom_layer_budgets(_p(sigma2), _p(q), H, G, D, int(layers), int(total_bits), _p(out), _p(ws),
                                      ws.numel(), _stream(stream)), "fathom_layer_budgets")
    return out


def plan_fixed(q: torch.Tensor, r: int, out=None, stream=None, bits: int = 4):
    """Fixed-depth comparator plan: the r channels with the largest
    sum_g |q| read at ``bits`` planes."""
    H, G, D = q.shape
    dev = q.device
    if out is None:
        out = (torch.empty((H, D), dtype=torch.uint8, device=dev), torch.empty((H, D), dtype=torch.int16, device=dev),
               torch.empty(H, dtype=torch.int32, device=dev))
    depth, active, n_active = out
    _check(lib().fathom_plan_fixed(_p(q), H, G, D, int(r), int(bits), _p(depth), _p(active), _p(n_active),
                                   _stream(stream)),
           "fathom_plan_fixed")
    return depth, active, n_active


def scan(planes, scales, n: int, active, n_active, q, mode: int = SCAN_DENSE, k: int = 0,
         scores=None, cand=None, stream=None, nibbles: bool = False, token_major: bool = False):
    """Scores [H][G][n] (DENSE) or the candidate buffer (CANDIDATE).  With
    ``nibbles`` the first argument is the nibble store (every active channel
    read at 4 bits); with ``token_major`` it is the token-major store of
    ``nibbles_tm_from_planes`` (the same scores)."""
    H, G, D = q.shape
    nbs = scales.shape[-1]
    if token_major:
        fn, name = lib().fathom_scan_nibbles_tm, "fathom_scan_nibbles_tm"
    elif nibbles:
        fn, name = lib().fathom_scan_nibbles, "fathom_scan_nibbles"
    else:
        fn, name = lib().fathom_scan, "fathom_scan"
    if mode == SCAN_DENSE:
        if scores is None:
            scores = torch.empty((H, G, n), dtype=torch.float32, device=q.device)
        _check(fn(_p(planes), _p(scales), H, D, n, nbs, _p(active), _p(n_active), _p(q), G,
                  SCAN_DENSE, _p(scores), None, 0, int(k), _stream(stream)), name)
        return scores
    nbytes = scan_cand_bytes(H, G, n, k)
    if cand is None:
        cand = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    _check(fn(_p(planes), _p(scales), H, D, n, nbs, _p(active), _p(n_active), _p(q), G,
              int(mode), None, _p(cand), cand.numel() * cand.element_size(), int(k), _stream(stream)), name)
    return cand


def nibbles_from_planes(planes, n: int, out=None, stream=None):
    """The nibble store [H][D][4][nb_stride] of the codes the planes hold."""
    H, D, _, nbs = planes.shape
    if out is None:
        out = torch.empty_like(planes)
    _check(lib().fathom_nibbles_from_planes(_p(planes), H, D, n, nbs, _p(out), _stream(stream)),
           "fathom_nibbles_from_planes")
    return out


def nibbles_tm_from_planes(planes, n: int, out=None, stream=None):
    """The token-major 4-bit store uint8 [H][64*nb_stride][D/2] of the codes
    the planes hold (two channels per byte, channel 2c in the low nibble)."""
    H, D, _, nbs = planes.shape
    if out is None:
        out = torch.zeros((H, 64 * nbs, D // 2), dtype=torch.uint8, device=planes.device)
    _check(lib().fathom_nibbles_tm_from_planes(_p(planes), H, D, n, nbs, _p(out), _stream(stream)),
           "fathom_nibbles_tm_from_planes")
    return out


def topk(H: int, G: int, n: int, k: int, scores=None, cand=None, out=None, workspace=None, stream=None):
    """Per-head top-k and per-group union.  Returns (idx int32 [H][G][k],
    union int32 [H][G*k], union_count int32 [H])."""
    dev = (scores if scores is not None else cand).device
    if out is None:
        out = (torch.empty((H, G, k), dtype=torch.int32, device=dev),
               torch.empty((H, G * k), dtype=torch.int32, device=dev),
               torch.empty(H, dtype=torch.int32, device=dev))
    idx, uni, cnt = out
    ws_need = topk_workspace_bytes(H, G, n, k)
    if workspace is None and ws_need:
        workspace = torch.empty(ws_need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().fathom_topk(_p(scores), _p(cand), H, G, n, int(k), _p(idx), _p(uni), _p(cnt), _p(workspace),
                             ws_bytes, _stream(stream)), "fathom_topk")
    return idx, uni, cnt


def dequant_rows(planes, scales, n: int, rows, row_count=None, bits: int = 4, out=None, stream=None):
    """Key rows rebuilt from the index: fp32 [H][M][D] for rows int32 [H][M]
    (e.g. the union of ``topk``), at ``bits`` planes."""
    H, D = planes.shape[0], planes.shape[1]
    M = rows.shape[1]
    if out is None:
        out = torch.empty((H, M, D), dtype=torch.float32, device=rows.device)
    _check(lib().fathom_dequant_rows(_p(planes), _p(scales), H, D, n, planes.shape[-1], _p(rows), M,
                                     _p(row_count), int(bits), _p(out), _stream(stream)), "fathom_dequant_rows")
    return out


def scan_topk_noalloc(planes, scales, n: int, active, n_active, q, k: int, out=None, stream=None):
    """Candidate scan + top-k + union using the library's own fixed device
    scratch instead of a caller buffer, for callers that cannot allocate
    device memory (see fathom_scan_topk_noalloc in include/fathom.h).  The
    output tensors may be preallocated and passed as ``out``."""
    H, G, D = q.shape
    if out is None:
        dev = q.device
        out = (torch.empty((H, G, k), dtype=torch.int32, device=dev),
               torch.empty((H, G * k), dtype=torch.int32, device=dev),
               torch.empty(H, dtype=torch.int32, device=dev))
    idx, uni, cnt = out
    _check(lib().fathom_scan_topk_noalloc(_p(planes), _p(scales), H, D, n, planes.shape[-1], _p(active),
                                          _p(n_active), _p(q), G, int(k), _p(idx), _p(uni), _p(cnt),
                                          _stream(stream)), "fathom_scan_topk_noalloc")
    return idx, uni, cnt


def calibrate_workspace_bytes(H: int, D: int, with_cov: bool) -> int:
    return int(lib().fathom_calibrate_workspace_bytes(H, D, 1 if with_cov else 0))


def calibrate(keys: torch.Tensor, n: int | None = None, with_mean: bool = True, with_cov: bool = False,
              workspace=None, stream=None):
    """Per-group key statistics over the first ``n`` keys of keys [H][n_total][D]
    (fp32 or bf16): (mean [H][D] or None, sigma2 [H][D], cov [H][D][D] or None),
    all fp32."""
    H, nt, D = keys.shape
    n = nt if n is None else int(n)
    if keys.dtype == torch.float32:
        dt = KEYS_F32
    elif keys.dtype == torch.bfloat16:
        dt = KEYS_BF16
    else:
        raise TypeError("keys must be float32 or bfloat16")
    if keys.stride(2) != 1:
        raise ValueError("keys must be contiguous along D")
    dev = keys.device
    sigma2 = torch.empty((H, D), dtype=torch.float32, device=dev)
    mean = torch.empty((H, D), dtype=torch.float32, device=dev) if with_mean else None
    cov = torch.empty((H, D, D), dtype=torch.float32, device=dev) if with_cov else None
    need = calibrate_workspace_bytes(H, D, with_cov)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _check(lib().fathom_calibrate(_p(keys), dt, H, n, D, keys.stride(0), keys.stride(1), _p(mean), _p(sigma2),
                                  _p(cov), _p(workspace), workspace.numel(), _stream(stream)), "fathom_calibrate")
    return mean, sigma2, cov


def union_attention_workspace_bytes(H: int, G: int, D: int, M: int) -> int:
    return int(lib().fathom_union_attention_workspace_bytes(H, G, D, M))


def union_attention(k_cache: torch.Tensor, v_cache: torch.Tensor, q: torch.Tensor, union_idx: torch.Tensor,
                    union_count: torch.Tensor, scale: float | None = None, out=None, workspace=None, stream=None):
    """Softmax attention [H][G][D] (fp32) of each query head over its group's
    union rows of the K/V cache [H][n][D] (fp32 or bf16)."""
    H, n, D = k_cache.shape
    G = q.shape[1]
    M = union_idx.shape[1]
    if k_cache.dtype != v_cache.dtype or k_cache.shape != v_cache.shape or k_cache.stride() != v_cache.stride():
        raise ValueError("k_cache and v_cache must share dtype, shape and strides")
    dt = {torch.float32: KEYS_F32, torch.bfloat16: KEYS_BF16}[k_cache.dtype]
    if k_cache.stride(2) != 1:
        raise ValueError("the cache must be contiguous along D")
    if out is None:
        out = torch.empty((H, G, D), dtype=torch.float32, device=q.device)
    need = int(lib().fathom_union_attention_workspace_bytes(H, G, D, M))
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    sc = 1.0 / math.sqrt(D) if scale is None else float(scale)
    _check(lib().fathom_union_attention(_p(k_cache), _p(v_cache), dt, H, n, D, k_cache.stride(0), k_cache.stride(1),
                                        _p(q), G, _p(union_idx), _p(union_count), M, sc, _p(out), _p(workspace),
                                        workspace.numel(), _stream(stream)), "fathom_union_attention")
    return out


def device_status(clear: bool = False, stream=None) -> int:
    """OK, or ERR_TIMEOUT if a library kernel on the current device gave up
    a bounded wait since the fault word was last cleared (synchronises the
    stream)."""
    st = int(lib().fathom_device_status(1 if clear else 0, _stream(stream)))
    if st not in (OK, ERR_TIMEOUT, ERR_BOUNDS):
        _check(st, "fathom_device_status")
    return st


class Step:
    """One decode step of the scan over a resident index: plan -> candidate
    scan -> top-k + union, with the dense rerun for any group whose
    candidate pass could not prove its top-k exact.  Buffers are allocated
    once; ``run`` launches only library kernels.  With ``nibbles`` the scans
    read that nibble store (every active channel whole) instead of the
    planes; with ``token_major`` too, it is the token-major store."""

    def __init__(self, planes, scales, n: int, sigma2, G: int, k: int, budget=48, fixed_r: int | None = None,
                 fixed_bits: int = 4, nibbles=None, token_major: bool = False):
        self.planes, self.scales, self.n, self.sigma2, self.k = planes, scales, n, sigma2, k
        self.nibbles = nibbles
        self.token_major = token_major   # ``nibbles`` is the token-major store
        self.store = planes if nibbles is None else nibbles
        self.H, self.D = sigma2.shape
        self.G = G
        self.budget = budget
        self.fixed_r = fixed_r
        self.fixed_bits = fixed_bits
        dev = sigma2.device
        H, D = self.H, self.D
        self.plan_out = (torch.empty((H, D), dtype=torch.uint8, device=dev),
                         torch.empty((H, D), dtype=torch.int16, device=dev),
                         torch.empty(H, dtype=torch.int32, device=dev),
                         torch.empty(H, dtype=torch.float32, device=dev))
        self.cand = torch.empty(scan_cand_bytes(H, G, n, k), dtype=torch.uint8, device=dev)
        self.topk_out = (torch.empty((H, G, k), dtype=torch.int32, device=dev),
                         torch.empty((H, G * k), dtype=torch.int32, device=dev),
                         torch.empty(H, dtype=torch.int32, device=dev))

    def run_plan(self, q):
        if self.fixed_r is None:
            plan(self.sigma2, q, self.budget, out=self.plan_out)
        else:
            plan_fixed(q, self.fixed_r, out=self.plan_out[:3], bits=self.fixed_bits)
        return self.plan_out

    def run_prepare(self, q):
        _, active, n_active, _ = self.plan_out
        return scan(self.store, self.scales, self.n, active, n_active, q, SCAN_PREPARE, self.k, cand=self.cand,
                    nibbles=self.nibbles is not None, token_major=self.token_major)

    def run_filter(self, q):
        _, active, n_active, _ = self.plan_out
        return scan(self.store, self.scales, self.n, active, n_active, q, SCAN_FILTER, self.k, cand=self.cand,
                    nibbles=self.nibbles is not None, token_major=self.token_major)

    def run_scan(self, q):
        self.run_prepare(q)
        return self.run_filter(q)

    def run_topk(self):
        return topk(self.H, self.G, self.n, self.k, cand=self.cand, out=self.topk_out)

    def run(self, q, check_overflow: bool = True):
        self.run_plan(q)
        self.run_scan(q)
        idx, uni, cnt = self.run_topk()
        if check_overflow:
            self.repair(q)
        return idx, uni, cnt

    def repair(self, q) -> int:
        """Dense rerun of groups whose candidate pass overflowed (host check)."""
        idx, uni, cnt = self.topk_out
        bad = torch.nonzero(cnt < 0).flatten().tolist()
        if not bad:
            return 0
        if int(cnt[bad[0]]) in (ERR_TIMEOUT, ERR_BOUNDS):
            raise FathomError(int(cnt[bad[0]]), "candidate scan (device fault word set)")
        _, active, n_active, _ = self.plan_out
        for h in bad:
            sl = slice(h, h + 1)
            sc = scan(self.store[sl], self.scales[sl], self.n, active[sl], n_active[sl], q[sl], SCAN_DENSE,
                      nibbles=self.nibbles is not None, token_major=self.token_major)
            topk(1, self.G, self.n, self.k, scores=sc, out=(idx[sl], uni[sl], cnt[sl]))
        return len(bad)
