"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs.  Planes, scales and plans must be bit-exact; scores
within 1e-5 of their L1 scale; top-k sets equal up to ties at the k-th
score; top-k of the GPU's own scores identical to a full sort of them."""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

from long_context_decode_bit_b200 import inputs
from _util import (assert_scores_close, assert_topk_sets_match, depth_to_active, keys_for_oracle,
                   lexsort_topk, np_u16, np_u64)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def make(w, dev=DEV):
    k = inputs.keys(w, 0, w.H, device=dev)
    q = inputs.queries(w, 0, w.H, device=dev).float().contiguous()
    s2 = inputs.calibration_sigma2(k, w.n_cal).contiguous()
    return k, q, s2


def oracle_pack(orc, k, nbs):
    return orc.pack(keys_for_oracle(k), nb_stride=nbs)


CASES = [
    inputs.TINY,
    dataclasses.replace(inputs.TINY, name="ragged", H=3, n=5037, seed=7),
    dataclasses.replace(inputs.TINY, name="one-block", H=2, n=64, seed=8, n_cal=64),
    dataclasses.replace(inputs.TINY, name="sub-block", H=2, n=37, seed=9, n_cal=37),
    dataclasses.replace(inputs.LAYER_32K, name="qk-ragged", H=2, n=9000, seed=10),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_pack_bit_exact(fathom_gpu, orc, w):
    k, _, _ = make(w)
    planes, scales = fathom_gpu.pack(k)
    torch.cuda.synchronize()
    p_ref, s_ref = oracle_pack(orc, k, planes.shape[-1])
    assert np.array_equal(np_u64(planes), p_ref)
    assert np.array_equal(np_u16(scales), s_ref)


@pytest.mark.parametrize("D,G", [(32, 1), (64, 3), (256, 8)])
def test_pack_plan_scan_other_shapes(fathom_gpu, orc, D, G):
    w = dataclasses.replace(inputs.TINY, name=f"d{D}g{G}", H=2, n=3000, D=D, G=G, seed=11 + D)
    k, q, s2 = make(w)
    planes, scales = fathom_gpu.pack(k)
    depth, active, na, _ = fathom_gpu.plan(s2, q, min(4 * D, 3 * D // 2))
    sc = fathom_gpu.scan(planes, scales, w.n, active, na, q)
    torch.cuda.synchronize()
    p_ref, s_ref = oracle_pack(orc, k, planes.shape[-1])
    assert np.array_equal(np_u64(planes), p_ref) and np.array_equal(np_u16(scales), s_ref)
    d_ref, a_ref, na_ref, _ = orc.plan(s2.cpu().numpy(), q.cpu().numpy(), min(4 * D, 3 * D // 2))
    assert np.array_equal(depth.cpu().numpy(), d_ref)
    ref, l1 = orc.scan(p_ref, s_ref, d_ref, q.cpu().numpy(), w.n)
    assert_scores_close(sc.cpu().numpy(), ref, l1)


@pytest.mark.parametrize("budget", [0, 1, 7, 48, 68, 92, 136, 300, 512])
def test_plan_bit_exact(fathom_gpu, orc, budget):
    w = dataclasses.replace(inputs.LAYER_32K, H=16, n=4096, seed=21)
    k, q, s2 = make(w)
    depth, active, na, theta = fathom_gpu.plan(s2, q, budget)
    torch.cuda.synchronize()
    d_ref, a_ref, na_ref, th_ref = orc.plan(s2.cpu().numpy(), q.cpu().numpy(), budget)
    assert np.array_equal(depth.cpu().numpy(), d_ref)
    assert np.array_equal(np_u16(active), a_ref)
    assert np.array_equal(na.cpu().numpy(), na_ref)
    assert np.array_equal(theta.cpu().numpy(), th_ref.astype(np.float32))


def test_plan_per_group_budgets_and_edge_importances(fathom_gpu, orc):
    rng = np.random.default_rng(0)
    H, G, D = 12, 4, 128
    q = rng.standard_normal((H, G, D)).astype(np.float32)
    s2 = np.abs(rng.standard_normal((H, D))).astype(np.float32)
    s2[0, :] = 1.0; q[0] = 1.0                        # all importances tied
    s2[1, :64] = 0.0                                  # half the channels worthless
    s2[2] = np.float32(1e-42) * (1 + np.arange(D))    # subnormal importances
    q[3, :, ::2] = 0.0
    s2[4] = np.exp(rng.uniform(-80, 80, D)).astype(np.float32)   # wide dynamic range
    budgets = np.array([5, 48, 100, 48, 136, 0, 512, 1, 47, 49, 255, 256], np.int32)
    depth, active, na, theta = fathom_gpu.plan(torch.tensor(s2, device=DEV), torch.tensor(q, device=DEV),
                                               torch.tensor(budgets, device=DEV))
    torch.cuda.synchronize()
    d_ref, a_ref, na_ref, th_ref = orc.plan(s2, q, budgets)
    assert np.array_equal(depth.cpu().numpy(), d_ref)
    assert np.array_equal(np_u16(active), a_ref)
    assert np.array_equal(na.cpu().numpy(), na_ref)


@pytest.mark.parametrize("r,bits", [(0, 4), (1, 4), (16, 4), (32, 4), (128, 4), (128, 2), (40, 1), (32, 3)])
def test_plan_fixed_bit_exact(fathom_gpu, orc, r, bits):
    w = dataclasses.replace(inputs.LAYER_32K, H=16, n=4096, seed=22)
    _, q, _ = make(w)
    q[3, :, 7] = q[3, :, 9]  # a tie, broken towards the lower channel
    depth, active, na = fathom_gpu.plan_fixed(q, r, bits=bits)
    torch.cuda.synchronize()
    d_ref, a_ref, na_ref = orc.plan_fixed(q.cpu().numpy(), r, bits)
    assert np.array_equal(depth.cpu().numpy(), d_ref)
    assert np.array_equal(np_u16(active), a_ref)
    assert np.array_equal(na.cpu().numpy(), na_ref)


def _full_path(fathom_gpu, orc, w, budget, fixed_r=None, fixed_bits=4):
    k, q, s2 = make(w)
    planes, scales = fathom_gpu.pack(k)
    if fixed_r is None:
        depth, active, na, _ = fathom_gpu.plan(s2, q, budget)
    else:
        depth, active, na = fathom_gpu.plan_fixed(q, fixed_r, bits=fixed_bits)
    sc = fathom_gpu.scan(planes, scales, w.n, active, na, q)
    idx, uni, cnt = fathom_gpu.topk(w.H, w.G, w.n, w.k, scores=sc)
    torch.cuda.synchronize()
    p_ref, s_ref = oracle_pack(orc, k, planes.shape[-1])
    assert np.array_equal(np_u64(planes), p_ref) and np.array_equal(np_u16(scales), s_ref)
    qn = q.cpu().numpy()
    if fixed_r is None:
        d_ref = orc.plan(s2.cpu().numpy(), qn, budget)[0]
    else:
        d_ref = orc.plan_fixed(qn, fixed_r, fixed_bits)[0]
    assert np.array_equal(depth.cpu().numpy(), d_ref)
    ref, l1 = orc.scan(p_ref, s_ref, d_ref, qn, w.n)
    gsc = sc.cpu().numpy()
    assert_scores_close(gsc, ref, l1)
    gidx = idx.cpu().numpy()
    # exact against a full sort of the GPU's own fp32 scores
    for h in range(w.H):
        for g in range(w.G):
            assert np.array_equal(gidx[h, g], lexsort_topk(gsc[h, g], w.k))
    # up to ties against the oracle's fp64 top-k
    r_idx, r_uni, r_cnt = orc.topk(ref, w.k)
    assert_topk_sets_match(gidx, r_idx, ref, l1, w.k)
    # union = sorted unique of the GPU's own lists
    guni, gcnt = uni.cpu().numpy(), cnt.cpu().numpy()
    for h in range(w.H):
        u = np.unique(gidx[h].reshape(-1))
        assert gcnt[h] == len(u)
        assert np.array_equal(guni[h, :gcnt[h]], u) and np.all(guni[h, gcnt[h]:] == -1)
    return planes, scales, active, na, q, sc, idx, uni, cnt


def test_tiny_full_path(fathom_gpu, orc):
    _full_path(fathom_gpu, orc, inputs.TINY, 48)


@pytest.mark.parametrize("budget", [48, 68, 92, 136])
def test_layer_32k_full_path(fathom_gpu, orc, budget):
    _full_path(fathom_gpu, orc, inputs.LAYER_32K, budget)


@pytest.mark.parametrize("r,bits", [(32, 4), (16, 4), (128, 2)], ids=["136-bit", "sparq-r16", "thumbnail"])
def test_layer_32k_fixed_depth_comparators(fathom_gpu, orc, r, bits):
    _full_path(fathom_gpu, orc, inputs.LAYER_32K, None, fixed_r=r, fixed_bits=bits)


@pytest.mark.parametrize("n,k", [(1, 1), (37, 37), (64, 5), (5037, 1), (5037, 100)])
def test_ragged_and_degenerate_sizes(fathom_gpu, orc, n, k):
    w = dataclasses.replace(inputs.TINY, name=f"n{n}", H=2, n=n, k=k, n_cal=n, seed=30 + n)
    _full_path(fathom_gpu, orc, w, 48)


def test_zero_budget_all_scores_zero_topk_takes_lowest_indices(fathom_gpu, orc):
    w = dataclasses.replace(inputs.TINY, H=2, n=3000, k=50, seed=40)
    *_, sc, idx, uni, cnt = _full_path(fathom_gpu, orc, w, 0)
    assert torch.all(sc == 0)
    assert np.array_equal(idx.cpu().numpy()[0, 0], np.arange(50))


@pytest.mark.parametrize("budget", [48, 136])
def test_candidate_path_equals_dense(fathom_gpu, orc, budget):
    w = inputs.LAYER_32K
    k, q, s2 = make(w)
    planes, scales = fathom_gpu.pack(k)
    depth, active, na, _ = fathom_gpu.plan(s2, q, budget)
    dense = fathom_gpu.scan(planes, scales, w.n, active, na, q)
    d_idx, d_uni, d_cnt = fathom_gpu.topk(w.H, w.G, w.n, w.k, scores=dense)
    step = fathom_gpu.Step(planes, scales, w.n, s2, w.G, w.k, budget=budget)
    c_idx, c_uni, c_cnt = step.run(q, check_overflow=False)
    torch.cuda.synchronize()
    assert torch.all(c_cnt >= 0)   # every group proved exact without a rerun
    assert torch.equal(c_idx, d_idx) and torch.equal(c_uni, d_uni) and torch.equal(c_cnt, d_cnt)
    # No ring wait of either scan gave up: the device fault word is clear.
    assert fathom_gpu.device_status() == fathom_gpu.OK


@pytest.mark.parametrize("n", [2000, 20000], ids=["direct", "sampled"])
def test_nan_query_channel_candidate_equals_dense(fathom_gpu, orc, n):
    """A non-finite query channel (device memory: no host check sees it)
    makes one head's scores NaN.  NaN ranks above every number in the
    top-k's order, so the candidate path must keep such keys: without a
    threshold sample every key sits at its own slot, and with one a NaN
    score counts as reaching tau (a head of NaN scores then overflows and is
    the dense rerun's business).  Every group the candidate path proves
    exact equals the dense path's top-k and union."""
    w = dataclasses.replace(inputs.TINY, name=f"nan-{n}", H=2, n=n, k=64, seed=91)
    k, q, s2 = make(w)
    planes, scales = fathom_gpu.pack(k)
    depth = np.zeros((w.H, w.D), np.uint8)
    depth[:, :40] = 1
    depth[:, 5] = 3
    act, na = depth_to_active(depth)
    active = torch.from_numpy(act.view(np.int16)).to(DEV)
    n_active = torch.from_numpy(na).to(DEV)
    q[0, 1, 5] = float("nan")
    dense = fathom_gpu.scan(planes, scales, w.n, active, n_active, q)
    d_idx, d_uni, d_cnt = fathom_gpu.topk(w.H, w.G, w.n, w.k, scores=dense)
    cand = fathom_gpu.scan(planes, scales, w.n, active, n_active, q, fathom_gpu.SCAN_CANDIDATE, w.k)
    c_idx, c_uni, c_cnt = fathom_gpu.topk(w.H, w.G, w.n, w.k, cand=cand)
    torch.cuda.synchronize()
    assert torch.isnan(dense[0, 1]).all() and not torch.isnan(dense[0, 0]).any() and not torch.isnan(dense[1]).any()
    assert np.array_equal(d_idx[0, 1].cpu().numpy(), np.arange(w.k))   # equal NaN keys: lowest indices
    proved = (c_cnt >= 0).cpu().numpy()
    assert proved[1]
    if n <= 2048:   # one scan tile: no threshold sample
        assert proved.all()
    for h in range(w.H):
        if proved[h]:
            assert torch.equal(c_idx[h], d_idx[h]) and torch.equal(c_uni[h], d_uni[h]) and c_cnt[h] == d_cnt[h]


def test_candidate_overflow_is_flagged_and_repaired(fathom_gpu, orc):
    # Budget 0: every score is 0, so every key reaches the sampled threshold
    # and the candidate buffer overflows; the group must be flagged, and the
    # dense rerun must give the dense answer.
    w = dataclasses.replace(inputs.LAYER_32K, H=2, seed=41)
    k, q, s2 = make(w)
    planes, scales = fathom_gpu.pack(k)
    step = fathom_gpu.Step(planes, scales, w.n, s2, w.G, w.k, budget=0)
    step.run_plan(q)
    step.run_scan(q)
    idx, uni, cnt = step.run_topk()
    torch.cuda.synchronize()
    assert torch.all(cnt == fathom_gpu.ERR_OVERFLOW)
    assert step.repair(q) == 2
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy()[1, 3], np.arange(w.k))
    assert torch.all(cnt == w.k)


def test_rotated_basis_full_path(fathom_gpu, orc):
    """Llama-shaped keys (no QK-norm) stored in the rotated basis: the scan
    sees fp32 rotated keys and queries; parity holds as for any input."""
    from long_context_decode_bit_b200 import basis
    w = dataclasses.replace(inputs.STEP_1M_LLAMA, H=3, n=20000, seed=61)
    k = inputs.keys(w, 0, w.H, device=DEV)
    q = inputs.queries(w, 0, w.H, device=DEV).float().contiguous()
    U = basis.klt_basis(k[:, :w.n_cal], q)
    kr, qr = basis.rotate(k, U), basis.rotate(q, U)
    s2 = inputs.calibration_sigma2(kr, w.n_cal).contiguous()
    planes, scales = fathom_gpu.pack(kr)
    depth, active, na, _ = fathom_gpu.plan(s2, qr, 48)
    sc = fathom_gpu.scan(planes, scales, w.n, active, na, qr)
    idx, uni, cnt = fathom_gpu.Step(planes, scales, w.n, s2, w.G, w.k, budget=48).run(qr)
    torch.cuda.synchronize()
    p_ref, s_ref = oracle_pack(orc, kr, planes.shape[-1])
    assert np.array_equal(np_u64(planes), p_ref) and np.array_equal(np_u16(scales), s_ref)
    d_ref = orc.plan(s2.cpu().numpy(), qr.cpu().numpy(), 48)[0]
    assert np.array_equal(depth.cpu().numpy(), d_ref)
    ref, l1 = orc.scan(p_ref, s_ref, d_ref, qr.cpu().numpy(), w.n)
    assert_scores_close(sc.cpu().numpy(), ref, l1)
    assert_topk_sets_match(idx.cpu().numpy(), orc.topk(ref, w.k)[0], ref, l1, w.k)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_dequant_rows_bit_exact(fathom_gpu, orc, bits):
    w = dataclasses.replace(inputs.LAYER_32K, H=3, n=9000, seed=71)
    k, q, s2 = make(w)
    planes, scales = fathom_gpu.pack(k)
    rng = np.random.default_rng(bits)
    M = 300
    rows = np.sort(rng.integers(-5, w.n + 5, (w.H, M)), axis=1).astype(np.int32)
    count = np.array([M, 123, -6], np.int32)          # full, partial, flagged group
    out = fathom_gpu.dequant_rows(planes, scales, w.n, torch.tensor(rows, device=DEV),
                                  torch.tensor(count, device=DEV), bits=bits)
    torch.cuda.synchronize()
    p_ref, s_ref = oracle_pack(orc, k, planes.shape[-1])
    ref = orc.dequant_rows(p_ref, s_ref, w.n, rows, count, bits)
    assert np.array_equal(out.cpu().numpy().astype(np.float64), ref)


def test_dequant_rows_of_the_union(fathom_gpu, orc):
    """The winners' keys, rebuilt from the planes for the union a step returns."""
    w = inputs.LAYER_32K
    k, q, s2 = make(w)
    planes, scales = fathom_gpu.pack(k)
    idx, uni, cnt = fathom_gpu.Step(planes, scales, w.n, s2, w.G, w.k, budget=48).run(q)
    out = fathom_gpu.dequant_rows(planes, scales, w.n, uni, cnt)
    torch.cuda.synchronize()
    p_ref, s_ref = oracle_pack(orc, k, planes.shape[-1])
    ref = orc.dequant_rows(p_ref, s_ref, w.n, uni.cpu().numpy(), cnt.cpu().numpy(), 4)
    assert np.array_equal(out.cpu().numpy().astype(np.float64), ref)
    # the 4-plane rows are the keys' 4-bit values: within half a cell of the key
    kk = k.float().cpu().numpy()
    for h in range(w.H):
        u = uni[h, :cnt[h]].cpu().numpy()
        err = np.abs(out[h, :len(u)].cpu().numpy() - kk[h, u])
        s = np.array([[orc.fp16_value(int(x)) for x in row] for row in s_ref[h][:, u // 64].T])
        assert np.all(err <= s / 16 + 1e-7)


def test_append_repacks_the_tail_block(fathom_gpu, orc):
    """Decode-time append: tokens arrive one small batch at a time; each time
    the tail block is packed again from its raw keys.  The index must equal
    packing every token at once (and so the oracle's)."""
    w = dataclasses.replace(inputs.LAYER_32K, H=3, n=5200, seed=81)
    k, _, _ = make(w)
    n_max = w.n
    nbs = fathom_gpu.nb_stride(n_max)
    planes = torch.zeros((w.H, w.D, 4, nbs), dtype=torch.int64, device=DEV)
    scales = torch.zeros((w.H, w.D, nbs), dtype=torch.int16, device=DEV)
    n = 4990
    fathom_gpu.pack_range(k[:, :n].contiguous(), planes, scales, 0)
    for step in (1, 5, 64, 70, 3, 67):            # crosses several block boundaries
        n_new = min(n_max, n + step)
        b0 = n // 64                              # the block holding token n (the old tail)
        fathom_gpu.pack_range(k[:, b0 * 64:n_new].contiguous(), planes, scales, b0)
        n = n_new
    torch.cuda.synchronize()
    full_p, full_s = fathom_gpu.pack(k[:, :n].contiguous(), nb_stride_words=nbs)
    torch.cuda.synchronize()
    assert torch.equal(planes, full_p) and torch.equal(scales, full_s)
    p_ref, s_ref = orc.pack(keys_for_oracle(k[:, :n]), nb_stride=nbs)
    assert np.array_equal(np_u64(planes), p_ref) and np.array_equal(np_u16(scales), s_ref)


# --------------------------------------------------------------------------
# Session calibration statistics (方法二 sigma^2; experiments section: one
# covariance per KV head from the session's own prefill keys)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("w,n", [(inputs.TINY, None), (inputs.TINY, 1024),
                                 (dataclasses.replace(inputs.LAYER_32K, name="cal", H=3, n=9000, seed=12), None),
                                 (dataclasses.replace(inputs.TINY, name="cal-d64", H=2, D=64, n=777, seed=13), None),
                                 (dataclasses.replace(inputs.STEP_1M_LLAMA, name="cal-corr", H=2, n=5000, seed=14), None),
                                 (dataclasses.replace(inputs.TINY, name="cal-d256", H=1, D=256, n=1500, seed=18), None)],
                         ids=["tiny", "tiny-first-1024", "qk-bf16-9000", "d64-ragged", "corr-bf16-5000", "d256"])
def test_calibrate_matches_oracle(fathom_gpu, orc, w, n):
    """Mean and sigma^2 equal the oracle's fp64 values rounded to fp32 (a
    one-ulp allowance covers the fp64 summation order); the covariance is
    within fp32 rounding of the oracle's plus 1e-12 of sqrt(var_a var_b)."""
    k = inputs.keys(w, 0, w.H, device=DEV)
    mean, s2, cov = fathom_gpu.calibrate(k, n=n, with_cov=True)
    torch.cuda.synchronize()
    om, ov, oc = orc.calibrate(keys_for_oracle(k), n=n)
    ulp = lambda x: np.spacing(np.abs(x).astype(np.float32)).astype(np.float64)
    for got, ref in ((mean, om), (s2, ov)):
        g = got.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(g - ref) <= ulp(ref) + 1e-30), np.abs(g - ref).max()
    g = cov.cpu().numpy().astype(np.float64)
    scale = np.sqrt(np.einsum("ha,hb->hab", ov, ov))
    assert np.all(np.abs(g - oc) <= ulp(oc) + 1e-12 * scale + 1e-30)


def test_calibrate_sigma2_feeds_the_plan(fathom_gpu, orc):
    """sigma^2 from the calibration call over the first n_cal keys gives the
    same plan as the harness statistic, bit for bit, on every group whose
    sigma^2 row came out identical; a group whose row differs (a one-ulp fp64
    summation-order case) still gets the oracle's plan of its own sigma^2."""
    w = inputs.LAYER_32K
    k, q, s2 = make(w)
    _, s2_gpu, _ = fathom_gpu.calibrate(k, n=w.n_cal, with_mean=False)
    d_ref, a_ref, n_ref, _ = fathom_gpu.plan(s2, q, 48)
    d_cal, a_cal, n_cal, _ = fathom_gpu.plan(s2_gpu, q, 48)
    torch.cuda.synchronize()
    same = torch.all(s2_gpu == s2, dim=1).cpu().numpy()
    assert (s2_gpu != s2).sum().item() <= 2   # one-ulp fp64 summation-order cases at most
    for h in range(w.H):
        if same[h]:
            assert torch.equal(d_ref[h], d_cal[h]) and torch.equal(a_ref[h], a_cal[h]) and n_ref[h] == n_cal[h]
        else:
            d_o, a_o, n_o, _ = orc.plan(s2_gpu[h:h + 1].cpu().numpy(), q[h:h + 1].cpu().numpy(), 48)
            assert np.array_equal(d_cal[h:h + 1].cpu().numpy(), d_o)
            assert np.array_equal(np_u16(a_cal[h:h + 1]), a_o) and n_cal[h].item() == n_o[0]


# --------------------------------------------------------------------------
# Attention over the union of winners (byte-accounting section: the KV rows
# of the union of the G heads' top-k are what a step fetches)
# --------------------------------------------------------------------------
def _attention_tolerance(k, v, q, uni, cnt):
    """Per-element bound for the fp32 kernel against the fp64 oracle.  A
    score is a D-term fp32 dot product (per-lane sums of D/32 terms, a
    5-level shuffle tree, a scaled query), so |ds| <= (D/32 + 7) u S with
    S = scale sum_j |q_j k_j| and u = 2^-24; a weight exp(s - m) then has
    relative error <= 2 max|ds| + 4u (expf, the max, the combine), and the
    output, a ratio of weighted sums over the c rows, adds (c + 8) u.  So
    |out - ref| <= (4 max|ds| + 8u + (c + 8) u) sum_i p_i |v_i| / sum_i p_i."""
    H, n, D = k.shape
    G = q.shape[1]
    u = 2.0 ** -24
    tol = np.zeros((H, G, D))
    for h in range(H):
        c = max(0, min(int(cnt[h]), uni.shape[1]))
        if c == 0:
            continue
        rows = uni[h, :c]
        kk = k[h, rows].astype(np.float64)
        vv = np.abs(v[h, rows].astype(np.float64))
        s = q[h].astype(np.float64) @ kk.T / np.sqrt(D)
        S = np.abs(q[h].astype(np.float64)) @ np.abs(kk).T / np.sqrt(D)
        p = np.exp(s - s.max(1, keepdims=True))
        w = (p @ vv) / p.sum(1, keepdims=True)
        ds = (D / 32 + 7) * u * S.max(1, keepdims=True)
        tol[h] = (4 * ds + 8 * u + (c + 8) * u) * w
    return tol


def _as_np(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


def test_union_attention_random_unions(fathom_gpu, orc):
    """Ragged counts over several 256-row chunks, -1 padding, an empty and an
    error count, and out-of-range indices (skipped) on fp32 keys."""
    w = dataclasses.replace(inputs.TINY, name="att", H=5, n=3000, seed=15)
    k = inputs.keys(w, 0, w.H, device=DEV)
    v = inputs.values(w, 0, w.H, device=DEV)
    q = inputs.queries(w, 0, w.H, device=DEV).float().contiguous()
    M = 700
    g = np.random.default_rng(15)
    uni = np.full((w.H, M), -1, np.int32)
    cnt = np.array([700, 513, 1, 0, -6], np.int32)
    for h in range(w.H):
        c = max(cnt[h], 0)
        uni[h, :c] = np.sort(g.choice(w.n, c, replace=False))
    bad = uni.copy()
    bad[1, 5] = w.n + 3          # outside the cache: skipped by the kernel
    out = fathom_gpu.union_attention(k, v, q, torch.from_numpy(bad).to(DEV), torch.from_numpy(cnt).to(DEV))
    torch.cuda.synchronize()
    ref_uni = uni.copy()
    ref_cnt = cnt.copy()
    ref_uni[1, 5:512] = ref_uni[1, 6:513]   # the same rows without the skipped entry
    ref_uni[1, 512] = -1
    ref_cnt[1] = 512
    ref = orc.union_attention(_as_np(k), _as_np(v), _as_np(q), ref_uni, ref_cnt)
    got = out.cpu().numpy().astype(np.float64)
    tol = _attention_tolerance(_as_np(k), _as_np(v), _as_np(q), ref_uni, ref_cnt)
    assert np.all(np.abs(got - ref) <= tol + 1e-30), np.max(np.abs(got - ref) - tol)
    assert not np.any(got[3]) and not np.any(got[4])
    # Rows 130 floats apart (not 16-byte multiples): the general kernel, same answer.
    kp = torch.zeros((w.H, w.n, w.D + 2), dtype=k.dtype, device=DEV)
    vp = torch.zeros_like(kp)
    kp[:, :, :w.D] = k
    vp[:, :, :w.D] = v
    out2 = fathom_gpu.union_attention(kp[:, :, :w.D], vp[:, :, :w.D], q, torch.from_numpy(bad).to(DEV),
                                      torch.from_numpy(cnt).to(DEV))
    torch.cuda.synchronize()
    got2 = out2.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got2 - ref) <= tol + 1e-30), np.max(np.abs(got2 - ref) - tol)


def test_union_attention_after_a_step(fathom_gpu, orc):
    """The union a 48-bit candidate step selects on a Qwen3-8B-shaped layer
    (bf16 K/V, up to 2048 rows per group), attended over and checked against
    the oracle on the same rows."""
    w = dataclasses.replace(inputs.LAYER_32K, H=3, seed=16)
    k, q, s2 = make(w)
    v = inputs.values(w, 0, w.H, device=DEV)
    planes, scales = fathom_gpu.pack(k)
    step = fathom_gpu.Step(planes, scales, w.n, s2, w.G, w.k, budget=48)
    _, uni, cnt = step.run(q)
    out = fathom_gpu.union_attention(k, v, q, uni, cnt)
    torch.cuda.synchronize()
    un, cn = uni.cpu().numpy(), cnt.cpu().numpy()
    assert np.all(cn > w.k)
    ref = orc.union_attention(keys_for_oracle(k), keys_for_oracle(v), _as_np(q), un, cn)
    tol = _attention_tolerance(_as_np(k), _as_np(v), _as_np(q), un, cn)
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= tol + 1e-30), np.max(np.abs(got - ref) - tol)


# --------------------------------------------------------------------------
# Nibble store comparator (byte-accounting section: the fixed-depth scans
# read 32 coordinates' whole 4-bit codes)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("w", [inputs.TINY, dataclasses.replace(inputs.LAYER_32K, name="nib-ragged", H=3, n=9001,
                                                                seed=17)], ids=["tiny", "qk-ragged"])
def test_nibbles_bit_exact_and_scan_equals_full_depth(fathom_gpu, orc, w):
    """The nibble store built from the GPU planes equals the oracle's nibble
    pack of the keys; its dense scan equals the plane scan at full depth
    bit for bit (same coefficients, same odd integers, same FMA order) and
    the oracle within tolerance; its candidate step picks the same top-k."""
    k, q, s2 = make(w)
    planes, scales = fathom_gpu.pack(k)
    nib = fathom_gpu.nibbles_from_planes(planes, w.n)
    torch.cuda.synchronize()
    ref = orc.pack_nibbles(keys_for_oracle(k), nb_stride=planes.shape[-1])
    nb = w.nb
    assert np.array_equal(np_u64(nib)[..., :nb], ref[..., :nb])
    depth, active, na = fathom_gpu.plan_fixed(q, 32)
    s_nib = fathom_gpu.scan(nib, scales, w.n, active, na, q, nibbles=True)
    s_pl = fathom_gpu.scan(planes, scales, w.n, active, na, q)
    torch.cuda.synchronize()
    assert torch.equal(s_nib, s_pl)
    o_scores, o_l1 = orc.scan(np_u64(planes), np_u16(scales), depth.cpu().numpy(), q.cpu().numpy(), w.n)
    assert_scores_close(s_nib.cpu().numpy(), o_scores, o_l1)
    st_n = fathom_gpu.Step(planes, scales, w.n, s2, w.G, w.k, fixed_r=32, nibbles=nib)
    st_p = fathom_gpu.Step(planes, scales, w.n, s2, w.G, w.k, fixed_r=32)
    a = st_n.run(q)
    b = st_p.run(q)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(a, b))


# --------------------------------------------------------------------------
# Per-layer budgets (方法二, per-layer plan paragraph)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("w,layers,mean_bits", [
    (dataclasses.replace(inputs.STEP_128K, name="lb-qwen", n=4096, n_cal=4096), 36, 48),
    (dataclasses.replace(inputs.STEP_1M_LLAMA, name="lb-llama", H=64, n=4096, n_cal=4096), 8, 48),
    (dataclasses.replace(inputs.TINY, name="lb-gauss", H=6, n=1024, n_cal=1024), 3, 200)],
    ids=["qwen-36-layers", "llama-8-layers", "gauss-3-layers-capped"])
def test_layer_budgets_match_oracle(fathom_gpu, orc, w, layers, mean_bits):
    """The greedy split equals the oracle's integer for integer, spends the
    whole total (capped at 4D per layer), and the plans it feeds respect it."""
    k, q, s2 = make(w)
    b = fathom_gpu.layer_budgets(s2, q, layers, layers * mean_bits)
    torch.cuda.synchronize()
    ref = orc.layer_budgets(s2.cpu().numpy(), q.cpu().numpy(), layers, layers * mean_bits)
    got = b.cpu().numpy()
    assert np.array_equal(got, ref)
    per = got.reshape(layers, -1)
    assert np.all(per == per[:, :1]) and per[:, 0].sum() == min(layers * mean_bits, layers * 4 * w.D)
    depth, _, _, _ = fathom_gpu.plan(s2, q, b)
    assert np.all(depth.int().sum(1).cpu().numpy() <= got)


@pytest.mark.parametrize("D,G", [(64, 3), (256, 8), (32, 1)])
def test_union_attention_other_shapes(fathom_gpu, orc, D, G):
    """Odd and extreme head counts and head dims (fp32 cache), one chunk and
    several, against the oracle with the same per-element bound."""
    w = dataclasses.replace(inputs.TINY, name=f"att-{D}-{G}", H=2, n=2000, D=D, G=G, seed=19 + D + G)
    k = inputs.keys(w, 0, w.H, device=DEV)
    v = inputs.values(w, 0, w.H, device=DEV)
    q = inputs.queries(w, 0, w.H, device=DEV).float().contiguous()
    g = np.random.default_rng(D + G)
    cnt = np.array([300, 1], np.int32)
    uni = np.full((w.H, 300), -1, np.int32)
    for h in range(w.H):
        uni[h, :cnt[h]] = np.sort(g.choice(w.n, cnt[h], replace=False))
    out = fathom_gpu.union_attention(k, v, q, torch.from_numpy(uni).to(DEV), torch.from_numpy(cnt).to(DEV))
    torch.cuda.synchronize()
    ref = orc.union_attention(_as_np(k), _as_np(v), _as_np(q), uni, cnt)
    tol = _attention_tolerance(_as_np(k), _as_np(v), _as_np(q), uni, cnt)
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= tol + 1e-30), np.max(np.abs(got - ref) - tol)


@pytest.mark.parametrize("D,G", [(64, 3), (256, 8)])
def test_nibble_scan_other_shapes(fathom_gpu, orc, D, G):
    """The nibble-store scan equals the full-depth plane scan bit for bit for
    odd G (padded coefficient records) and the largest D and G."""
    w = dataclasses.replace(inputs.TINY, name=f"nib-{D}-{G}", H=2, n=3001, D=D, G=G, seed=23 + D)
    k, q, s2 = make(w)
    planes, scales = fathom_gpu.pack(k)
    nib = fathom_gpu.nibbles_from_planes(planes, w.n)
    depth, active, na = fathom_gpu.plan_fixed(q, D // 4)
    s_nib = fathom_gpu.scan(nib, scales, w.n, active, na, q, nibbles=True)
    s_pl = fathom_gpu.scan(planes, scales, w.n, active, na, q)
    torch.cuda.synchronize()
    assert torch.equal(s_nib, s_pl)


# --------------------------------------------------------------------------
# Fused KLT rotation inside pack (section 基座选择): bit-exact planes and
# scales against the oracle's fixed-order fp32 fused multiply-add chain.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("D,n,dtype", [(128, 3000, torch.bfloat16), (128, 64 * 37, torch.float32),
                                       (64, 1000, torch.bfloat16), (96, 777, torch.float32),
                                       (256, 700, torch.bfloat16)],
                         ids=["d128-bf16-ragged", "d128-f32", "d64-bf16", "d96-f32", "d256-bf16"])
def test_pack_rotated_matches_oracle(fathom_gpu, orc, D, n, dtype):
    from long_context_decode_bit_b200 import basis
    w = dataclasses.replace(inputs.LAYER_32K, name=f"rot-{D}-{n}", H=3, n=n, D=D, kind="corr", n_cal=min(n, 512), seed=77 + D)
    k = inputs.keys(w, 0, w.H, device=DEV).to(dtype).contiguous()
    q = inputs.queries(w, 0, w.H, device=DEV).float().contiguous()
    U = basis.klt_basis(k[:, :w.n_cal], q).contiguous()
    planes, scales = fathom_gpu.pack_rotated(k, U)
    torch.cuda.synchronize()
    p_ref, s_ref = orc.pack_rotated(keys_for_oracle(k), U.cpu().numpy(), nb_stride=planes.shape[-1])
    assert np.array_equal(np_u64(planes), p_ref)
    assert np.array_equal(np_u16(scales), s_ref)


def test_pack_rotated_identity_is_pack_and_appends(fathom_gpu):
    w = dataclasses.replace(inputs.LAYER_32K, name="rot-eye", H=2, n=5000, seed=78)
    k = inputs.keys(w, 0, w.H, device=DEV)
    eye = torch.eye(w.D, device=DEV).expand(w.H, w.D, w.D).contiguous()
    p0, s0 = fathom_gpu.pack(k)
    p1, s1 = fathom_gpu.pack_rotated(k, eye)
    torch.cuda.synchronize()
    assert torch.equal(p0, p1) and torch.equal(s0, s1)
    # Rewriting from block b0 on (the decode-time append) equals packing at once.
    U = torch.linalg.qr(torch.randn(w.H, w.D, w.D, device=DEV, dtype=torch.float64))[0].float().contiguous()
    pa, sa = fathom_gpu.pack_rotated(k, U)
    b0 = 40
    pb = torch.zeros_like(pa)
    sb = torch.zeros_like(sa)
    fathom_gpu.pack_rotated(k[:, :64 * b0 + 10].contiguous(), U, nb_stride_words=pa.shape[-1], planes=pb, scales=sb)
    lib = fathom_gpu.lib()
    tail = k[:, 64 * b0:].contiguous()
    st = lib.fathom_pack_rotated(fathom_gpu._p(tail), fathom_gpu.KEYS_BF16, w.H, tail.shape[1], w.D, tail.stride(0),
                                 tail.stride(1), fathom_gpu._p(U), ctypes.c_void_p(pb.data_ptr() + 8 * b0),
                                 ctypes.c_void_p(sb.data_ptr() + 2 * b0), pa.shape[-1], fathom_gpu._stream(None))
    assert st == fathom_gpu.OK
    torch.cuda.synchronize()
    assert torch.equal(pa, pb) and torch.equal(sa, sb)


# --------------------------------------------------------------------------
# Token-major 4-bit comparator (byte-accounting section: a serving stack's
# 4-bit K copy, one row of D/2 bytes per token, read for r chosen channels).
# --------------------------------------------------------------------------
def _tm_codes(store: np.ndarray, n: int) -> np.ndarray:
    """Codes [H][D][n] from the token-major rows (low nibble = even channel)."""
    lo, hi = store & 15, store >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(store.shape[0], store.shape[1], -1)   # [H][tokens][D]
    return codes[:, :n].transpose(0, 2, 1)


def _cm_codes(nib_words: np.ndarray, n: int) -> np.ndarray:
    """Codes [H][D][n] from the oracle's channel-major nibble words [H][D][4][nbs]."""
    H, D, _, nbs = nib_words.shape
    sh = (np.arange(16, dtype=np.uint64) * np.uint64(4))
    c = (nib_words[..., None] >> sh) & np.uint64(15)             # [H][D][4 words][nbs][16]
    c = c.transpose(0, 1, 3, 2, 4).reshape(H, D, nbs * 64)      # token 64b + 16w + e
    return c[:, :, :n].astype(np.uint8)


@pytest.mark.parametrize("w", [
    dataclasses.replace(inputs.LAYER_32K, name="tm-8x32768", H=8),
    dataclasses.replace(inputs.TINY, name="tm-g3-d64", H=3, n=5001, D=64, G=3, seed=31),
    dataclasses.replace(inputs.TINY, name="tm-g8-d256", H=2, n=2500, D=256, G=8, seed=32),
    dataclasses.replace(inputs.TINY, name="tm-direct", H=2, n=1500, seed=33),
], ids=lambda w: w.name)
def test_token_major_store_and_scan(fathom_gpu, orc, w):
    """The token-major rows hold the oracle's 4-bit codes; the scan over them
    gives the oracle's full-depth scores of the chosen channels within
    tolerance and the channel-major nibble scan's to fp32 rounding, and its
    candidate step picks exactly the top-k of its own dense scores."""
    k, q, s2 = make(w)
    planes, scales = fathom_gpu.pack(k)
    tm = fathom_gpu.nibbles_tm_from_planes(planes, w.n)
    torch.cuda.synchronize()
    assert tm.shape == (w.H, 64 * planes.shape[-1], w.D // 2)
    ref = orc.pack_nibbles(keys_for_oracle(k), nb_stride=planes.shape[-1])
    assert np.array_equal(_tm_codes(tm.cpu().numpy(), w.n), _cm_codes(ref, w.n))
    r = min(32, w.D // 4)
    depth, active, na = fathom_gpu.plan_fixed(q, r)
    s_tm = fathom_gpu.scan(tm, scales, w.n, active, na, q, token_major=True)
    nib = fathom_gpu.nibbles_from_planes(planes, w.n)
    s_cm = fathom_gpu.scan(nib, scales, w.n, active, na, q, nibbles=True)
    torch.cuda.synchronize()
    o_scores, o_l1 = orc.scan(np_u64(planes), np_u16(scales), depth.cpu().numpy(), q.cpu().numpy(), w.n)
    assert_scores_close(s_tm.cpu().numpy(), o_scores, o_l1)
    assert_scores_close(s_tm.cpu().numpy(), s_cm.cpu().numpy().astype(np.float64), o_l1)
    st = fathom_gpu.Step(planes, scales, w.n, s2, w.G, w.k, fixed_r=r, nibbles=tm, token_major=True)
    idx, uni, cnt = st.run(q)
    d_idx, d_uni, d_cnt = fathom_gpu.topk(w.H, w.G, w.n, w.k, scores=s_tm)
    torch.cuda.synchronize()
    assert torch.equal(idx, d_idx) and torch.equal(uni, d_uni) and torch.equal(cnt, d_cnt)
    assert_topk_sets_match(idx.cpu().numpy(), orc.topk(o_scores, w.k)[0], o_scores, o_l1, w.k)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_pack_of_unaligned_rows_equals_contiguous(fathom_gpu, dtype):
    """Key rows 130 elements apart (not 16-byte multiples) take the element-wise
    staging; the index equals that of the same keys stored contiguously."""
    w = dataclasses.replace(inputs.LAYER_32K, name="pack-unaligned", H=2, n=3001, seed=79)
    k = inputs.keys(w, 0, w.H, device=DEV).to(dtype).contiguous()
    kp = torch.zeros((w.H, w.n, w.D + 2), dtype=dtype, device=DEV)
    kp[:, :, :w.D] = k
    p0, s0 = fathom_gpu.pack(k)
    p1, s1 = fathom_gpu.pack(kp[:, :, :w.D])
    torch.cuda.synchronize()
    assert torch.equal(p0, p1) and torch.equal(s0, s1)
