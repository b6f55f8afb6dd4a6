"""Pins for the CPU oracle (no GPU).

Each test checks the oracle against something other than itself: a library
routine (numpy's binary16 conversion, sorts, matmul), exact rational
arithmetic on the pages' geometric definitions, brute force over all
allocations for tiny inputs, an independent greedy algorithm, or a figure
the pages print (``tests/golden``).  The paper is "Fathom: Per-Query Read
Depth for Sparse Decoding over Offloaded KV Caches" (arXiv 2609.17652); the
sections cited are those of the yeyulingfeng.com article unless noted.
"""
import heapq
import itertools
import os
from fractions import Fraction

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f16_bits_np(x):
    return int(np.array([x], dtype=np.float64).astype(np.float16).view(np.uint16)[0])


# --------------------------------------------------------------------------
# binary16 rounding of the block scale (section 方法一: one fp16 scale per
# 64-token block per channel)
# --------------------------------------------------------------------------
def test_fp16_rounding_matches_numpy(orc):
    rng = np.random.default_rng(0)
    xs = list(np.exp2(rng.uniform(-30, 17, 4000)))
    # exact halfway points between consecutive binary16 values, both parities
    for b in list(range(1, 0x7BFF, 97)) + [0x3BFF, 0x3C00, 0x0001, 0x03FF, 0x0400]:
        lo = float(np.array([b], np.uint16).view(np.float16)[0])
        hi = float(np.array([b + 1], np.uint16).view(np.float16)[0])
        xs += [(lo + hi) / 2, np.nextafter((lo + hi) / 2, 0), np.nextafter((lo + hi) / 2, 1e9)]
    xs += [0.0, 65504.0, 65519.99, 65520.0, 1e6, 2.0 ** -25, 2.0 ** -26, 3 * 2.0 ** -26]
    for x in xs:
        assert orc.fp16_bits(float(x)) == f16_bits_np(float(x)), x
    for b in range(0, 0x7C00, 37):
        v = float(np.array([b], np.uint16).view(np.float16)[0])
        assert orc.fp16_value(b) == v


# --------------------------------------------------------------------------
# The 4-bit code (section 方法一): uniform, symmetric, code 8 = zero, MSB =
# sign; a prefix of t planes is the t-bit mid-rise quantiser on [-s, s].
# --------------------------------------------------------------------------
SCALES = [1.0, 0.7998046875, 3.0, 2.0 ** -10, 1234.0, 6.103515625e-05]


def test_code_sign_bit_and_zero(orc):
    rng = np.random.default_rng(1)
    for s in SCALES:
        for k in rng.uniform(-s, s, 500):
            c = orc.code4(float(k), s)
            assert (c >> 3) == (1 if k >= 0 else 0)
        assert orc.code4(0.0, s) == 8
        assert orc.code4(s * 1e-9, s) == 8
        assert orc.code4(-s * 1e-9, s) == 7


def test_code_cells_uniform_and_symmetric(orc):
    for s in SCALES:
        S = Fraction(s)
        for c in range(16):
            lo = -S + c * S / 8           # lower edge belongs to the cell
            centre = -S + (2 * c + 1) * S / 16
            assert orc.code4(float(lo), s) == c
            assert orc.code4(float(centre), s) == c
            # mirror image of a cell centre lands in the mirrored cell
            assert orc.code4(float(-centre), s) == 15 - c
        assert orc.code4(s, s) == 15          # top edge clamps into the last cell
        assert orc.code4(2 * s, s) == 15
        assert orc.code4(-2 * s, s) == 0


def midrise(k: Fraction, t: int, s: Fraction) -> Fraction:
    """t-bit mid-rise quantiser on [-s, s]: 2^t equal cells, value at the
    cell centre, inputs beyond the range clamped into the end cells."""
    cells = 2 ** t
    width = 2 * s / cells
    idx = (k + s) // width
    idx = max(0, min(cells - 1, int(idx)))
    return -s + (idx + Fraction(1, 2)) * width


def test_prefix_is_t_bit_midrise_quantiser(orc):
    rng = np.random.default_rng(2)
    for s in SCALES:
        ks = list(rng.uniform(-1.2 * s, 1.2 * s, 300).astype(np.float32))
        ks += [np.float32(e * s / 8) for e in range(-8, 9)]
        for k in ks:
            c = orc.code4(float(k), s)
            for t in range(1, 5):
                want = midrise(Fraction(float(k)), t, Fraction(s))
                assert Fraction(orc.dequant(c, t, s)) == want, (k, s, t)
        assert orc.dequant(11, 0, s) == 0.0


def test_four_planes_give_the_4bit_form_and_nearest_centre(orc):
    rng = np.random.default_rng(3)
    for s in SCALES:
        centres = np.array([(c - 7.5) * s / 8 for c in range(16)])
        for c in range(16):
            assert orc.dequant(c, 4, s) == centres[c]
        for k in rng.uniform(-s, s, 300):
            c = orc.code4(float(k), s)
            d = np.abs(centres - k)
            assert d[c] <= d.min() + 1e-12 * s


def test_error_bound_and_variance_quarter_per_plane(orc):
    # Each extra plane halves the cell and divides the error variance by 4
    # (section 方法二, second paragraph).  Uniform k over [-s, s).
    s = 1.5
    ks = (np.arange(32768) + 0.5) / 32768 * 2 * s - s
    mse = []
    for t in range(1, 5):
        err = np.array([k - orc.dequant(orc.code4(float(k), s), t, s) for k in ks])
        assert np.max(np.abs(err)) <= s / 2 ** t + 1e-15
        mse.append(np.mean(err ** 2))
        assert mse[-1] == pytest.approx((2 * s / 2 ** t) ** 2 / 12, rel=1e-3)
    for a, b in zip(mse, mse[1:]):
        assert a / b == pytest.approx(4.0, rel=1e-3)


def test_code_floor_is_exact_next_to_cell_edges(orc):
    # fp32 and bf16 keys one ulp either side of every cell edge
    for s in SCALES:
        for e in range(-8, 9):
            edge = np.float32(e * s / 8)
            for k in (np.nextafter(edge, np.float32(-np.inf)), edge, np.nextafter(edge, np.float32(np.inf))):
                exact = int((Fraction(float(k)) * 8) // Fraction(s)) + 8
                assert orc.code4(float(k), s) == max(0, min(15, exact))


# --------------------------------------------------------------------------
# Pack: channel-major planes + fp16 block scales, 68 B/token/KV head
# --------------------------------------------------------------------------
def unpack_codes(planes, n):
    """[H][D][4][nb] uint64 -> codes [H][n][D] (bit i of word b = token 64b+i;
    plane 0 is the most significant bit)."""
    H, D, _, nb = planes.shape
    bits = np.zeros((H, D, 4, nb * 64), dtype=np.int64)
    for i in range(64):
        bits[..., i::64] = ((planes >> np.uint64(i)) & np.uint64(1)).astype(np.int64)
    codes = bits[:, :, 0] * 8 + bits[:, :, 1] * 4 + bits[:, :, 2] * 2 + bits[:, :, 3]
    return codes[:, :, :n].transpose(0, 2, 1), bits


def test_pack_scales_codes_padding(orc):
    rng = np.random.default_rng(4)
    H, n, D = 2, 200, 8
    keys = (rng.standard_normal((H, n, D)) * np.exp(rng.standard_normal(D))).astype(np.float32)
    planes, scales = orc.pack(keys)
    nb = 4
    assert planes.shape == (H, D, 4, nb) and scales.shape == (H, D, nb)
    for h in range(H):
        for j in range(D):
            for b in range(nb):
                blk = keys[h, b * 64:min(n, b * 64 + 64), j]
                assert scales[h, j, b] == f16_bits_np(float(np.max(np.abs(blk))))
    codes, bits = unpack_codes(planes, n)
    for h in range(H):
        for i in range(n):
            for j in range(D):
                s = orc.fp16_value(int(scales[h, j, i // 64]))
                assert codes[h, i, j] == orc.code4(float(keys[h, i, j]), s)
    assert np.all(bits[..., n:] == 0)  # padded tail tokens carry no bits


def test_pack_bf16_equals_fp32_of_same_values(orc):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, 130, 32)).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)        # bf16 truncation of x
    vals = (bits.astype(np.uint32) << 16).view(np.float32)    # exact bf16 values
    p1, s1 = orc.pack(bits)
    p2, s2 = orc.pack(vals)
    assert np.array_equal(p1, p2) and np.array_equal(s1, s2)


def test_storage_is_68_bytes_per_token_per_kv_head(orc):
    H, n, D = 1, 256, 128
    planes, scales = orc.pack(np.ones((H, n, D), np.float32))
    assert (planes.nbytes + scales.nbytes) / (H * n) == 68


def test_pack_matches_printed_bitplane_figure(orc):
    # tests/golden/bitplane_figure.txt: three keys' bits, plane3..plane0.
    rows = [list(map(int, ln.split())) for ln in open(os.path.join(GOLDEN, "bitplane_figure.txt"))
            if ln.strip() and not ln.startswith("#")]
    s = 2.0
    ks = [s]  # token 0 sets the block maximum
    for _, p3, p2, p1, p0 in rows:
        c = p3 * 8 + p2 * 4 + p1 * 2 + p0
        ks.append((c - 7.5) * s / 8)  # centre of cell c
    keys = np.zeros((1, 64, 1), np.float32)
    keys[0, :len(ks), 0] = ks
    planes, scales = orc.pack(keys)
    assert orc.fp16_value(int(scales[0, 0, 0])) == s
    for tok, (_, p3, p2, p1, p0) in enumerate(rows, start=1):
        got = [int(planes[0, 0, p, 0] >> np.uint64(tok)) & 1 for p in range(4)]
        assert got == [p3, p2, p1, p0]  # our plane 0 is the figure's plane3 (the sign)


# --------------------------------------------------------------------------
# Plan: importance and reverse water-filling (section 方法二)
# --------------------------------------------------------------------------
def test_importance_single_precision_order(orc):
    rng = np.random.default_rng(6)
    H, G, D = 3, 4, 128
    q = rng.standard_normal((H, G, D)).astype(np.float32) * 3
    s2 = np.abs(rng.standard_normal((H, D))).astype(np.float32)
    w = orc.importance(s2, q)
    acc = q[:, 0] * q[:, 0]
    for g in range(1, G):
        acc = (acc + q[:, g] * q[:, g]).astype(np.float32)
    want = (s2 * acc).astype(np.float32)
    assert np.array_equal(w.view(np.uint32), want.view(np.uint32))


def test_importance_is_each_channels_measured_score_error(orc):
    """The importance w_j = sigma_j^2 sum_g q_{g,j}^2 is what a channel's
    unread or partly read planes cost in expected squared score error
    (section 方法二: reading a plane divides the channel's error variance by 4,
    and the error enters every head's score through q_{g,j}).

    Keys k_ij = sigma_j z_i share one standard-normal column z and the
    sigma_j are powers of two, so every channel has the same codes and block
    scales up to its power of two: the squared score error of channel j read
    alone at depth t, measured against the full-precision keys through
    orc_pack and orc_scan, is exactly sigma_j^2 sum_g q_{g,j}^2 MSE_z(t).
    Its ratio to orc_importance must therefore be one constant over the
    channels at every depth; sigma in place of sigma^2, or (sum_g q)^2 in
    place of sum_g q^2, breaks that.  From depth 2 on each further plane
    divides the error by about 4."""
    rng = np.random.default_rng(11)
    D, G, n, n_cal = 8, 4, 64 * 256, 4096
    sig = 2.0 ** np.array([-2, -1, 0, 1, 2, 3, -3, 1], dtype=np.float64)
    z = rng.standard_normal(n).astype(np.float32)
    keys = (z[:, None].astype(np.float64) * sig[None, :]).astype(np.float32)[None]
    q = rng.standard_normal((1, G, D)).astype(np.float32)
    q[0, 1] = -0.5 * q[0, 0]        # mixed signs: sum_g q^2 and (sum_g q)^2 disagree
    s2 = keys[:, :n_cal].astype(np.float64).var(axis=1).astype(np.float32)
    w = orc.importance(s2, q)[0].astype(np.float64)
    planes, scales = orc.pack(keys)
    exact = q[0].astype(np.float64)[:, None, :] * keys[0].astype(np.float64)[None, :, :]   # [G][n][D]
    err = {}
    for t in (0, 1, 2, 3, 4):
        e = np.zeros(D)
        for j in range(D):
            depth = np.zeros((1, D), np.uint8)
            depth[0, j] = t
            sc = orc.scan(planes, scales, depth, q, n, with_l1=False)[0]   # [G][n]
            e[j] = np.mean(np.sum((exact[:, :, j] - sc) ** 2, axis=0))
        ratio = e / w
        assert np.allclose(ratio, ratio[0], rtol=1e-5), (t, ratio)
        err[t] = e
        for alt in (np.sqrt(s2[0]) * np.sum(q[0].astype(np.float64) ** 2, axis=0),
                    s2[0] * np.sum(q[0].astype(np.float64), axis=0) ** 2):
            r = e / alt
            assert not np.allclose(r, r[0], rtol=1e-2)
    for t in (2, 3):
        assert np.all((err[t] / err[t + 1] > 3.0) & (err[t] / err[t + 1] < 6.0)), err[t] / err[t + 1]


def plan_from_w(orc, w, B):
    """Plan with G = 1, q = 1 so that the importance is exactly w."""
    w = np.asarray(w, np.float32)
    D = w.shape[-1]
    q = np.ones((1, 1, D), np.float32)
    return orc.plan(w.reshape(1, D), q, B)


def objective(w, t):
    return sum(float(wj) * 4.0 ** (-int(tj)) for wj, tj in zip(w, t))


def test_plan_is_optimal_by_brute_force(orc):
    rng = np.random.default_rng(7)
    for trial in range(60):
        D = int(rng.integers(1, 7))
        w = np.exp(rng.uniform(-6, 6, D)).astype(np.float32)
        if trial % 5 == 0:
            w[rng.integers(0, D)] = 0.0  # a channel with no importance
        npos = int(np.sum(w > 0))
        for B in range(0, 4 * D + 2):
            depth, active, na, theta = plan_from_w(orc, w, B)
            t = depth[0]
            best = min(objective(w, a) for a in itertools.product(range(5), repeat=D) if sum(a) <= B)
            assert objective(w, t) == pytest.approx(best, rel=1e-12, abs=0)
            assert int(t.sum()) == min(B, 4 * npos)
            assert np.all(t[w == 0] == 0)


def test_plan_with_ties_is_optimal_for_its_own_bit_count(orc):
    rng = np.random.default_rng(8)
    for _ in range(40):
        D = int(rng.integers(2, 7))
        w = rng.choice(np.array([1.0, 4.0, 0.25, 16.0, 2.0], np.float32), D)
        for B in range(0, 4 * D + 1):
            t = plan_from_w(orc, w, B)[0][0]
            used = int(t.sum())
            assert used <= B
            best = min(objective(w, a) for a in itertools.product(range(5), repeat=D) if sum(a) == used)
            assert objective(w, t) == pytest.approx(best, rel=1e-12)


def test_plan_equals_greedy_marginal_allocation(orc):
    # Hand bits one at a time to the largest marginal gain w_j 4^-t_j * 3/4.
    rng = np.random.default_rng(9)
    for _ in range(10):
        D = 128
        w = np.exp(rng.uniform(-8, 8, D)).astype(np.float32)
        for B in (0, 1, 17, 48, 92, 136, 300, 511, 512):
            t = np.zeros(D, int)
            heap = [(-float(w[j]), j) for j in range(D)]
            heapq.heapify(heap)
            for _ in range(B):
                negv, j = heapq.heappop(heap)
                t[j] += 1
                if t[j] < 4:
                    heapq.heappush(heap, (negv / 4.0, j))
            assert np.array_equal(plan_from_w(orc, w, B)[0][0], t)


def test_plan_invariants(orc):
    rng = np.random.default_rng(10)
    H, G, D = 5, 4, 128
    q = rng.standard_normal((H, G, D)).astype(np.float32)
    q[:, :, rng.integers(0, D, 10)] *= 5
    s2 = np.abs(rng.standard_normal((H, D))).astype(np.float32)
    w = orc.importance(s2, q)
    for B in (0, 1, 48, 68, 92, 136, 512, 600, -3):
        depth, active, na, theta = orc.plan(s2, q, B)
        Bc = min(max(B, 0), 4 * D)
        for h in range(H):
            t = depth[h].astype(int)
            assert t.sum() <= Bc
            order = np.argsort(-w[h], kind="stable")
            assert np.all(np.diff(t[order]) <= 0)            # more important, at least as deep
            js = np.nonzero(t)[0]
            assert na[h] == len(js)
            assert np.array_equal(active[h, :na[h]], (js | (t[js] << 8)).astype(np.uint16))
            assert np.all(active[h, na[h]:] == 0)
        # scaling every importance by 4 leaves depths unchanged
        d4 = orc.plan(s2 * 4, q, B)[0]
        assert np.array_equal(d4, depth)
    assert np.all(orc.plan(s2, q, 0)[0] == 0)
    assert np.all(orc.plan(s2, q, 4 * D)[0] == 4)


def test_plan_fixed_reduces_to_a_sort(orc):
    rng = np.random.default_rng(11)
    H, G, D = 4, 4, 128
    q = rng.standard_normal((H, G, D)).astype(np.float32)
    q[1, :, 5] = q[1, :, 9]  # a tie, broken towards the lower channel
    for r, bits in ((0, 4), (1, 4), (16, 4), (32, 4), (128, 4), (128, 2), (40, 1), (32, 3)):
        depth, active, na = orc.plan_fixed(q, r, bits)
        for h in range(H):
            a = np.abs(q[h, 0])
            for g in range(1, G):
                a = (a + np.abs(q[h, g])).astype(np.float32)
            top = np.lexsort((np.arange(D), -a.astype(np.float64)))[:r]
            want = np.zeros(D, np.uint8)
            want[top] = bits
            assert np.array_equal(depth[h], want)
            assert na[h] == r
            js = np.sort(top)
            assert np.array_equal(active[h, :r], (js | (bits << 8)).astype(np.uint16))


# --------------------------------------------------------------------------
# Scan (section 方法二, last paragraph: the G heads share the plan)
# --------------------------------------------------------------------------
def _dequant_all(orc, keys):
    planes, scales = orc.pack(keys)
    H, n, D = keys.shape
    codes, _ = unpack_codes(planes, n)
    s = np.array([[[orc.fp16_value(int(x)) for x in row] for row in sc] for sc in scales])  # [H][D][nb]
    sk = np.repeat(s, 64, axis=2)[:, :, :n].transpose(0, 2, 1)                        # [H][n][D]
    return planes, scales, (codes - 7.5) * sk / 8


def test_scan_full_depth_is_a_matvec(orc):
    rng = np.random.default_rng(12)
    H, G, n, D = 2, 4, 300, 32
    keys = rng.standard_normal((H, n, D)).astype(np.float32)
    q = rng.standard_normal((H, G, D)).astype(np.float32)
    planes, scales, K4 = _dequant_all(orc, keys)
    depth = np.full((H, D), 4, np.uint8)
    sc, l1 = orc.scan(planes, scales, depth, q, n)
    want = np.einsum("hgd,hnd->hgn", q.astype(np.float64), K4)
    assert np.all(np.abs(sc - want) <= 1e-13 * l1)
    assert np.allclose(l1, np.einsum("hgd,hnd->hgn", np.abs(q.astype(np.float64)), np.abs(K4)), rtol=1e-13)
    zero = orc.scan(planes, scales, np.zeros((H, D), np.uint8), q, n)[0]
    assert np.all(zero == 0)


def test_scan_one_channel_prefix_matches_midrise(orc):
    rng = np.random.default_rng(13)
    H, G, n, D = 1, 2, 150, 6
    keys = (rng.standard_normal((H, n, D)) * 2).astype(np.float32)
    planes, scales = orc.pack(keys)
    for j in range(D):
        for t in range(1, 5):
            depth = np.zeros((H, D), np.uint8)
            depth[0, j] = t
            q = np.zeros((H, G, D), np.float32)
            q[0, 0, j] = 1.0
            q[0, 1, j] = -0.5
            sc = orc.scan(planes, scales, depth, q, n, with_l1=False)
            for i in range(n):
                s = Fraction(orc.fp16_value(int(scales[0, j, i // 64])))
                want = midrise(Fraction(float(keys[0, i, j])), t, s)
                assert Fraction(sc[0, 0, i]) == want
                assert Fraction(sc[0, 1, i]) == -want / 2


def test_scan_is_linear_in_the_query(orc):
    rng = np.random.default_rng(14)
    H, G, n, D = 2, 4, 257, 64
    keys = rng.standard_normal((H, n, D)).astype(np.float32)
    planes, scales = orc.pack(keys)
    depth = rng.integers(0, 5, (H, D)).astype(np.uint8)
    q1 = rng.standard_normal((H, G, D)).astype(np.float32)
    q2 = rng.standard_normal((H, G, D)).astype(np.float32)
    s1, l1a = orc.scan(planes, scales, depth, q1, n)
    s2, l1b = orc.scan(planes, scales, depth, q2, n)
    s12 = orc.scan(planes, scales, depth, (q1 + q2).astype(np.float32), n, with_l1=False)
    # (q1+q2) is rounded to fp32, so compare against that rounding's size
    assert np.all(np.abs(s12 - (s1 + s2)) <= 1e-6 * (l1a + l1b))
    # head g only sees query row g: swapping two rows swaps two score rows
    qs = q1.copy()
    qs[:, [0, 3]] = qs[:, [3, 0]]
    ss = orc.scan(planes, scales, depth, qs, n, with_l1=False)
    assert np.array_equal(ss[:, [3, 0]], s1[:, [0, 3]])


# --------------------------------------------------------------------------
# Top-k and union (section 先算一笔字节账, top-k bullet)
# --------------------------------------------------------------------------
def test_topk_reduces_to_lexsort_and_union_to_unique(orc):
    rng = np.random.default_rng(15)
    H, G, n, k = 3, 4, 1000, 64
    sc = rng.standard_normal((H, G, n))
    sc[0, 0, 10:20] = sc[0, 0, 5]          # ties: lower index first
    sc[1] = np.round(sc[1], 1)             # many ties
    idx, uni, cnt = orc.topk(sc, k)
    for h in range(H):
        allw = []
        for g in range(G):
            want = np.lexsort((np.arange(n), -sc[h, g]))[:k]
            assert np.array_equal(idx[h, g], want)
            allw.append(want)
        u = np.unique(np.concatenate(allw))
        assert cnt[h] == len(u)
        assert np.array_equal(uni[h, :cnt[h]], u)
        assert np.all(uni[h, cnt[h]:] == -1)


# --------------------------------------------------------------------------
# Printed byte accounting (tests/golden/byte_accounting.txt)
# --------------------------------------------------------------------------
def _golden_accounting():
    out = {}
    for ln in open(os.path.join(GOLDEN, "byte_accounting.txt")):
        if ln.startswith("#") or not ln.strip():
            continue
        name, val, unit, tol, _ = [x.strip() for x in ln.split("|")]
        out[name] = (float(val), unit, float(tol))
    return out


def test_byte_accounting_matches_printed_figures():
    from long_context_decode_bit_b200 import accounting as acc
    g = _golden_accounting()

    def check(name, got):
        want, _, tol = g[name]
        assert got == pytest.approx(want, rel=tol, abs=0 if tol else 1e-9), name

    check("index_bytes_per_token_kv_head", acc.index_bytes_per_token(128))
    check("fixed_scan_bits_r32", acc.fixed_scan_bits(32))
    check("fixed_scan_step_traffic_32k", acc.per_token_index_bytes(288, 32768, acc.fixed_scan_bits(32) / 8) / 1e6)
    check("fixed_scan_step_traffic_1m", acc.per_token_index_bytes(288, 2 ** 20, acc.fixed_scan_bits(32) / 8) / 1e9)
    check("dense_bf16_kv_32k", acc.dense_kv_bytes(36, 8, 128, 32768) / 1e9)
    check("sparq_r16_bits", acc.fixed_scan_bits(16))
    check("fathom_read_bits_mean48", acc.read_bits_per_token(48, 32))
    check("fewer_bytes_56_vs_68", 100 * (1 - acc.read_bits_per_token(48, 32) / acc.fixed_scan_bits(16)))
    check("fathom_read_bits_mean40", acc.read_bits_per_token(40, 28))
    check("fewer_bytes_47_vs_68", 100 * (1 - acc.read_bits_per_token(40, 28) / acc.fixed_scan_bits(16)))
    check("label_cache_1m", acc.per_token_index_bytes(288, 2 ** 20, 17) / 1e9)
    check("landmark_index_1m", acc.per_token_index_bytes(288, 2 ** 20, 32) / 1e9)
    check("a100_int_ops_per_hbm_byte", 108 * 64 * 1.41e9 / 2.0e12)
    # the scan-byte helper agrees with the per-token figure
    assert acc.scan_bytes(2 ** 20, 48, 32, query_bytes=False) * 8 / 2 ** 20 == acc.read_bits_per_token(48, 32)


# --------------------------------------------------------------------------
# Key rows rebuilt from the planes (section 边界, storage-overhead paragraph)
# --------------------------------------------------------------------------
def test_dequant_rows_is_the_midrise_value_of_each_key(orc):
    rng = np.random.default_rng(16)
    H, n, D = 2, 300, 16
    keys = (rng.standard_normal((H, n, D)) * 3).astype(np.float32)
    planes, scales = orc.pack(keys)
    M = 40
    rows = rng.integers(-3, n + 3, (H, M)).astype(np.int32)   # includes out-of-range entries
    count = np.array([M, 25], np.int32)
    for bits in range(1, 5):
        out = orc.dequant_rows(planes, scales, n, rows, count, bits)
        for h in range(H):
            for r in range(M):
                i = rows[h, r]
                for j in range(D):
                    if r >= count[h] or not 0 <= i < n:
                        assert out[h, r, j] == 0.0
                        continue
                    s = Fraction(orc.fp16_value(int(scales[h, j, i // 64])))
                    assert Fraction(out[h, r, j]) == midrise(Fraction(float(keys[h, i, j])), bits, s)


# --------------------------------------------------------------------------
# Session calibration statistics (section 方法二: sigma^2 measured on
# calibration keys; experiments section: one covariance per KV head from
# the session's own prefill keys)
# --------------------------------------------------------------------------
def test_calibrate_closed_forms(orc):
    """Values the definitions fix: a constant channel has variance 0 and
    its own value as mean; a +-a two-point channel has mean 0 and variance
    a^2; two channels equal up to sign have covariance -+var."""
    n = 512
    k = np.zeros((1, n, 4), dtype=np.float32)
    k[0, :, 0] = 3.25
    k[0, ::2, 1], k[0, 1::2, 1] = 1.5, -1.5
    k[0, :, 2] = (2 * np.arange(n) - (n - 1)) / 512.0        # evenly spaced, exact in fp32
    k[0, :, 3] = -k[0, :, 2]
    mean, var, cov = orc.calibrate(k)
    assert mean[0, 0] == 3.25 and var[0, 0] == 0.0 and not np.any(cov[0, 0]) and not np.any(cov[0, :, 0])
    assert mean[0, 1] == 0.0 and var[0, 1] == 2.25
    v2 = var[0, 2]
    # variance of i = 0..n-1 is (n^2 - 1)/12; the channel is (2i - (n-1))/512
    assert v2 == pytest.approx(4.0 * (n * n - 1) / 12.0 / 512.0 ** 2, rel=1e-12)
    assert cov[0, 2, 3] == pytest.approx(-v2, rel=1e-12) and cov[0, 3, 3] == pytest.approx(v2, rel=1e-12)


def test_calibrate_matches_library_moments_and_invariances(orc):
    """Against numpy's population variance and biased covariance (the
    special case of library routines); shift leaves the centred moments
    unchanged, scaling by a multiplies them by a^2; the covariance is
    symmetric, positive semi-definite, with the variances on its diagonal;
    bf16 keys give the statistics of their fp32 values; n selects a prefix."""
    rng = np.random.default_rng(7)
    H, nt, D = 3, 700, 16
    std = np.exp(rng.normal(0, 1, D))
    k = (rng.standard_normal((H, nt, D)) * std + rng.normal(0, 2, D)).astype(np.float32)
    n = 600
    mean, var, cov = orc.calibrate(k, n=n)
    x = k[:, :n].astype(np.float64)
    assert np.allclose(mean, x.mean(1), rtol=1e-12, atol=1e-12)
    assert np.allclose(var, x.var(1), rtol=1e-10)
    for h in range(H):
        assert np.allclose(cov[h], np.cov(x[h].T, bias=True), rtol=1e-9, atol=1e-12)
        assert np.array_equal(cov[h], cov[h].T)
        assert np.linalg.eigvalsh(cov[h]).min() > -1e-9 * np.trace(cov[h])
        assert np.allclose(np.diag(cov[h]), var[h], rtol=1e-12)
    m2, v2, c2 = orc.calibrate((k + np.float32(4.0)).astype(np.float32), n=n)   # shift (exact in fp32 here? not always)
    assert np.allclose(v2, var, rtol=1e-5) and np.allclose(m2, mean + 4.0, rtol=1e-6)
    m3, v3, c3 = orc.calibrate((k * np.float32(2.0)).astype(np.float32), n=n)   # exact scaling by 2
    assert np.allclose(v3, 4.0 * var, rtol=1e-12) and np.allclose(c3, 4.0 * cov, rtol=1e-12, atol=1e-12)
    kb = (k.view(np.uint32) >> 16).astype(np.uint16)              # bf16 truncation of k
    kf = (kb.astype(np.uint32) << 16).view(np.float32)            # ... and its exact fp32 value
    mb, vb, cb = orc.calibrate(kb, n=n)
    mf, vf, cf = orc.calibrate(np.ascontiguousarray(kf), n=n)
    assert np.array_equal(mb, mf) and np.array_equal(vb, vf) and np.array_equal(cb, cf)
    m0, v0, c0 = orc.calibrate(k, n=0)
    assert not np.any(m0) and not np.any(v0) and not np.any(c0)


# --------------------------------------------------------------------------
# Attention over the union of winners (byte-accounting section: the rows a
# step fetches are the union of the G heads' top-k)
# --------------------------------------------------------------------------
def test_union_attention_special_cases(orc):
    """With every row in the union it is dense softmax attention (numpy
    matmul + exp); one row returns that value row; a zero query averages the
    union's value rows; the order of the union list does not matter; an
    empty or error count gives zeros; bf16 K/V give the result of their
    fp32 values."""
    rng = np.random.default_rng(11)
    H, n, D, G = 2, 300, 32, 4
    k = rng.standard_normal((H, n, D)).astype(np.float32)
    v = rng.standard_normal((H, n, D)).astype(np.float32)
    q = rng.standard_normal((H, G, D)).astype(np.float32)
    full = np.tile(np.arange(n, dtype=np.int32), (H, 1))
    out = orc.union_attention(k, v, q, full, np.full(H, n, np.int32))
    s = np.einsum("hgd,hnd->hgn", q.astype(np.float64), k.astype(np.float64)) / np.sqrt(D)
    p = np.exp(s - s.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    assert np.allclose(out, np.einsum("hgn,hnd->hgd", p, v.astype(np.float64)), rtol=1e-12, atol=1e-13)
    one = orc.union_attention(k, v, q, np.array([[17], [250]], np.int32), np.array([1, 1], np.int32))
    assert np.array_equal(one[0], np.tile(v[0, 17].astype(np.float64), (G, 1)))
    assert np.array_equal(one[1], np.tile(v[1, 250].astype(np.float64), (G, 1)))
    rows = np.stack([rng.choice(n, 40, replace=False) for _ in range(H)]).astype(np.int32)
    zq = np.zeros_like(q)
    avg = orc.union_attention(k, v, zq, rows, np.full(H, 40, np.int32))
    for h in range(H):
        assert np.allclose(avg[h], np.tile(v[h, rows[h]].astype(np.float64).mean(0), (G, 1)), rtol=1e-12, atol=1e-14)
    a = orc.union_attention(k, v, q, rows, np.full(H, 40, np.int32))
    b = orc.union_attention(k, v, q, rows[:, ::-1].copy(), np.full(H, 40, np.int32))
    assert np.allclose(a, b, rtol=1e-12, atol=1e-14)
    # a very sharp query: the softmax collapses onto the best row of the
    # union (its score exceeds the next by far more than 1), with no overflow
    big = (q * np.float32(1e4)).astype(np.float32)
    sharp = orc.union_attention(k, v, big, rows, np.full(H, 40, np.int32))
    for h in range(H):
        s_h = big[h].astype(np.float64) @ k[h, rows[h]].astype(np.float64).T
        best = rows[h][np.argmax(s_h, axis=1)]
        assert np.all(np.isfinite(sharp[h]))
        assert np.allclose(sharp[h], v[h, best].astype(np.float64), rtol=1e-9, atol=1e-9)
    pad = np.concatenate([rows, np.full((H, 10), -1, np.int32)], axis=1)   # -1 padded past the count
    assert np.array_equal(orc.union_attention(k, v, q, pad, np.full(H, 40, np.int32)), a)
    assert not np.any(orc.union_attention(k, v, q, pad, np.array([0, -6], np.int32)))
    kb = (k.view(np.uint32) >> 16).astype(np.uint16)
    vb = (v.view(np.uint32) >> 16).astype(np.uint16)
    kf = (kb.astype(np.uint32) << 16).view(np.float32)
    vf = (vb.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(orc.union_attention(kb, vb, q, rows, np.full(H, 40, np.int32)),
                          orc.union_attention(np.ascontiguousarray(kf), np.ascontiguousarray(vf), q, rows,
                                              np.full(H, 40, np.int32)))


# --------------------------------------------------------------------------
# Nibble store (byte-accounting section: the fixed-depth scans' whole 4-bit
# coordinates)
# --------------------------------------------------------------------------
def test_nibbles_hold_the_plane_codes(orc):
    """Token i's nibble is the 4-bit code whose bits the four planes hold
    (plane p = bit 3 - p), for every token, with zero past n; and with all
    four planes read the scan equals the nibble code's mid-rise value times
    the query (decoded here straight from the nibbles)."""
    rng = np.random.default_rng(21)
    H, n, D = 2, 300, 8
    k = (rng.standard_normal((H, n, D)) * np.exp(rng.normal(0, 1, D))).astype(np.float32)
    planes, scales = orc.pack(k)
    nib = orc.pack_nibbles(k)
    nb = (n + 63) // 64
    for h in range(H):
        for j in range(D):
            for b in range(nb):
                for i in range(64):
                    code_p = sum(((int(planes[h, j, p, b]) >> i) & 1) << (3 - p) for p in range(4))
                    code_n = (int(nib[h, j, i // 16, b]) >> (4 * (i % 16))) & 15
                    assert code_n == code_p
                    if b * 64 + i >= n:
                        assert code_n == 0
    q = rng.standard_normal((H, 4, D)).astype(np.float32)
    depth = np.full((H, D), 4, np.uint8)
    sc = orc.scan(planes, scales, depth, q, n, with_l1=False)
    s = np.array([[orc.fp16_value(int(x)) for x in row] for row in scales.reshape(H * D, nb)]).reshape(H, D, nb)
    for h in range(H):
        for i in range(n):
            b = i // 64
            codes = np.array([(int(nib[h, j, (i % 64) // 16, b]) >> (4 * (i % 16))) & 15 for j in range(D)])
            khat = (codes - 7.5) * s[h, :, b] / 8.0
            assert np.allclose(sc[h, :, i], q[h].astype(np.float64) @ khat, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# Per-layer budgets (section 方法二, per-layer plan paragraph)
# --------------------------------------------------------------------------
def _layer_cost(orc, s2, q, layers, budgets):
    """sum over layers of the layer's expected squared score error relative
    to its unread error, from the oracle's own plans (fp64 over fp32 w)."""
    H, G, D = q.shape
    w = orc.importance(s2, q).astype(np.float64)
    depth, _, _, _ = orc.plan(s2, q, np.asarray(budgets, np.int32))
    E = (w * 4.0 ** (-depth.astype(np.float64))).sum(1)
    P = H // layers
    return sum(E[l * P:(l + 1) * P].sum() / w[l * P:(l + 1) * P].sum() for l in range(layers))


def test_layer_budgets_are_optimal_by_brute_force(orc):
    """On tiny layers (D = 2, 2 groups each) the greedy split reaches the
    least total relative error over every split of the total, and it always
    spends the whole total (capped at 4D per layer)."""
    rng = np.random.default_rng(31)
    for trial in range(12):
        L, P, D, G = 3, 2, 2, 2
        H = L * P
        s2 = np.exp(rng.normal(0, 1.5, (H, D))).astype(np.float32)
        q = rng.standard_normal((H, G, D)).astype(np.float32)
        T = int(rng.integers(0, 4 * D * L + 3))
        b = orc.layer_budgets(s2, q, L, T)
        per_layer = b[::P]
        assert np.array_equal(b, np.repeat(per_layer, P))
        assert per_layer.sum() == min(T, 4 * D * L) and per_layer.max() <= 4 * D
        best = min(_layer_cost(orc, s2, q, L, np.repeat(np.array(split), P))
                   for split in itertools.product(range(4 * D + 1), repeat=L) if sum(split) == min(T, 4 * D * L))
        assert _layer_cost(orc, s2, q, L, b) <= best * (1 + 1e-12)


def test_layer_budgets_invariances(orc):
    """Identical layers share the total evenly (the remainder to the lower
    layers); scaling one layer's sigma^2 by a power of 4 leaves its relative
    curve, so the split, unchanged; one layer gets the flat budget."""
    rng = np.random.default_rng(32)
    P, D, G = 2, 16, 4
    s2 = np.exp(rng.normal(0, 1, (P, D))).astype(np.float32)
    q = rng.standard_normal((P, G, D)).astype(np.float32)
    s2_3, q_3 = np.tile(s2, (3, 1)), np.tile(q, (3, 1, 1))
    assert list(orc.layer_budgets(s2_3, q_3, 3, 3 * 40 + 2)[::P]) == [41, 41, 40]
    s2_a = np.exp(rng.normal(0, 1, (3 * P, D))).astype(np.float32)
    q_a = rng.standard_normal((3 * P, G, D)).astype(np.float32)
    base = orc.layer_budgets(s2_a, q_a, 3, 150)
    s2_b = s2_a.copy()
    s2_b[P:2 * P] *= np.float32(16.0)
    assert np.array_equal(orc.layer_budgets(s2_b, q_a, 3, 150), base)
    assert np.all(orc.layer_budgets(s2_a, q_a, 1, 50) == 50)


# --------------------------------------------------------------------------
# Rotated basis (section 基座选择: keys stored as their coordinates in an
# orthonormal KLT basis, queries rotated to match).  The oracle's rotation
# y_i = sum_d k_d U[d][i] runs in one stated order of fp32 fused
# multiply-adds (d ascending from +0), so the codes packed from it are
# defined bit for bit.
# --------------------------------------------------------------------------
def _round_f32(x: Fraction) -> Fraction:
    """Nearest-even binary32 value of the exact rational x (normal and
    subnormal range; no overflow), by integer arithmetic."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    quantum = Fraction(2) ** (max(e, -126) - 23)
    return sign * round(a / quantum) * quantum   # round() on a Fraction is half-to-even


def _fma_chain(x, u):
    y = Fraction(0)
    for xd, ud in zip(x, u):
        y = _round_f32(Fraction(float(xd)) * Fraction(float(ud)) + y)
    return y


def test_rotation_identity_and_permutation(orc):
    rng = np.random.default_rng(11)
    H, n, D = 2, 150, 32
    k = (rng.standard_normal((H, n, D)) * np.exp2(rng.integers(-3, 4, (H, 1, D)))).astype(np.float32)
    kb = (k.view(np.uint32) >> 16).astype(np.uint16)        # bf16 bit patterns (truncated values)
    eye = np.stack([np.eye(D, dtype=np.float32)] * H)
    for keys in (k, kb):
        assert np.array_equal(orc.rotate_keys(keys, eye), orc.rotate_keys(keys, eye))
        p0, s0 = orc.pack(keys)
        p1, s1 = orc.pack_rotated(keys, eye)
        assert np.array_equal(p0, p1) and np.array_equal(s0, s1)
    assert np.array_equal(orc.rotate_keys(k, eye), k)
    # U[d][i] = 1 iff d = pi(i): coordinate i is channel pi(i), exactly, and
    # so are its planes and scales (pi is not an involution: U and U^T differ).
    pi = np.roll(np.arange(D), 5)
    P = np.zeros((H, D, D), np.float32)
    P[:, pi, np.arange(D)] = 1.0
    assert not np.array_equal(P[0], P[0].T)
    y = orc.rotate_keys(k, P)
    assert np.array_equal(y, k[:, :, pi])
    p0, s0 = orc.pack(k)
    p1, s1 = orc.pack_rotated(k, P)
    assert np.array_equal(p1, p0[:, pi]) and np.array_equal(s1, s0[:, pi])


def test_rotation_is_the_stated_fma_chain_exactly(orc):
    # Random inputs against the chain evaluated in exact rational arithmetic
    # with nearest-even rounding after every step.
    rng = np.random.default_rng(12)
    H, n, D = 1, 4, 8
    k = rng.standard_normal((H, n, D)).astype(np.float32)
    U = rng.standard_normal((H, D, D)).astype(np.float32)
    y = orc.rotate_keys(k, U)
    for t in range(n):
        for i in range(D):
            assert Fraction(float(y[0, t, i])) == _fma_chain(k[0, t], U[0, :, i]), (t, i)
    # Fused: k = (1, a), column (-(1 + 2^-11), a) with a = 1 + 2^-12.  The
    # exact a*a = 1 + 2^-11 + 2^-24 survives one rounding after the add
    # (2^-24); a separately rounded product would have given 0.
    a = 1.0 + 2.0 ** -12
    U2 = np.zeros((1, 2, 2), np.float32)
    U2[0, :, 0] = [-(1.0 + 2.0 ** -11), a]
    y2 = orc.rotate_keys(np.array([[[1.0, a]]], np.float32), U2)
    assert y2[0, 0, 0] == np.float32(2.0 ** -24)
    # Order: d ascending.  (2^-30, 1, -1) against a column of ones gives 0
    # (2^-30 is lost against 1); the reverse order would keep 2^-30.
    U3 = np.zeros((1, 3, 3), np.float32)
    U3[0, :, 0] = 1.0
    y3 = orc.rotate_keys(np.array([[[2.0 ** -30, 1.0, -1.0]]], np.float32), U3)
    assert y3[0, 0, 0] == 0.0
    assert _fma_chain([-1.0, 1.0, 2.0 ** -30], [1.0, 1.0, 1.0]) == Fraction(2) ** -30


def test_rotated_scores_preserve_q_dot_k(orc):
    # An orthonormal U keeps q.k: with the queries rotated the same way, the
    # full-depth scan of the rotated index is q.k up to the quantiser's
    # half-cell error per coordinate (s/16 in the block's scale) and U's fp32
    # rounding.  The transposed basis does not: the pin sees the orientation.
    rng = np.random.default_rng(13)
    H, n, D, G = 2, 256, 32, 2
    k = rng.standard_normal((H, n, D)).astype(np.float32)
    q = rng.standard_normal((H, G, D))
    U64 = np.stack([np.linalg.qr(rng.standard_normal((D, D)))[0] for _ in range(H)])
    U = U64.astype(np.float32)
    exact = np.einsum("hgd,hnd->hgn", q, k.astype(np.float64))
    full = np.full((H, D), 4, np.uint8)

    def err_and_bound(Uk, Uq):
        planes, scales = orc.pack_rotated(k, Uk)
        qr = np.einsum("hgd,hdi->hgi", q, Uq.astype(np.float64)).astype(np.float32)
        sc = orc.scan(planes, scales, full, qr, n, with_l1=False)
        s = np.array([[[orc.fp16_value(int(b)) for b in row] for row in sh] for sh in scales])   # [H][D][nb]
        s_tok = np.repeat(s, 64, axis=2)[:, :, :n]                                              # [H][D][n]
        bound = np.einsum("hgi,hin->hgn", np.abs(qr.astype(np.float64)), s_tok) / 16.0
        bound += 1e-5 * np.linalg.norm(q, axis=2)[:, :, None] * np.linalg.norm(k, axis=2)[:, None, :]
        return np.abs(sc - exact), bound

    err, bound = err_and_bound(U, U)
    assert np.all(err <= bound)
    # Keys rotated by U^T while the queries use U: the bound fails widely.
    err_t, bound_t = err_and_bound(np.ascontiguousarray(U.transpose(0, 2, 1)), U)
    assert np.mean(err_t > bound_t) > 0.1
