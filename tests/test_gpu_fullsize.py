"""Parity at the benchmark's full sizes, in the launch configuration the
benchmark times (all groups of the step in one batched launch, candidate
path), on outputs the oracle can compute one by one:

- the plan of every group, bit-exact;
- planes and scales of sampled groups, bit-exact;
- the scores of sampled keys of sampled groups, within 1e-5 of their L1 scale;
- the top-k and union of sampled groups against the oracle's full sort.
"""
import numpy as np
import pytest
import torch

import bench
from long_context_decode_bit_b200 import fathom, inputs
from _util import SCORE_RTOL, assert_topk_sets_match, keys_for_oracle, np_u16, np_u64

pytestmark = pytest.mark.gpu

# 16 groups spread over all 36 layers of the step (first and last included)
SAMPLED_GROUPS = tuple(int(h) for h in np.linspace(0, 287, 16).round())


@pytest.fixture(scope="module")
def step_1m():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fathom.load()
    w = inputs.STEP_1M
    dev = torch.device("cuda", 0)
    planes, scales, s2, q, _ = bench.build_index(w, dev)
    st = fathom.Step(planes, scales, w.n, s2, w.G, w.k, budget=48)
    idx, uni, cnt = st.run(q)
    torch.cuda.synchronize()
    yield w, planes, scales, s2, q, st
    del planes, scales
    torch.cuda.empty_cache()


@pytest.mark.parametrize("h", SAMPLED_GROUPS)
def test_fullsize_step_matches_oracle_on_sampled_group(step_1m, orc, h):
    w, planes, scales, s2, q, st = step_1m
    # planes/scales of group h from its own keys, regenerated (same seed)
    k = inputs.keys(w, h, h + 1, device="cuda")
    p_ref, s_ref = orc.pack(keys_for_oracle(k), nb_stride=planes.shape[-1])
    del k
    assert np.array_equal(np_u64(planes[h:h + 1]), p_ref)
    assert np.array_equal(np_u16(scales[h:h + 1]), s_ref)
    qn = q[h:h + 1].cpu().numpy()
    d_ref = orc.plan(s2[h:h + 1].cpu().numpy(), qn, 48)[0]
    depth = st.plan_out[0]
    assert np.array_equal(depth[h:h + 1].cpu().numpy(), d_ref)
    # scores of sampled keys (GPU dense scan of this group vs the oracle)
    ref, l1 = orc.scan(p_ref, s_ref, d_ref, qn, w.n)
    _, active, na, _ = st.plan_out
    dense = fathom.scan(planes[h:h + 1], scales[h:h + 1], w.n, active[h:h + 1], na[h:h + 1], q[h:h + 1])
    torch.cuda.synchronize()
    rng = np.random.default_rng(h)
    sample = np.concatenate([rng.integers(0, w.n, 20000), np.arange(0, 2048), np.arange(w.n - 2048, w.n)])
    g_sc = dense.cpu().numpy()[0][:, sample].astype(np.float64)
    err = np.abs(g_sc - ref[0][:, sample])
    assert np.all(err <= SCORE_RTOL * l1[0][:, sample])
    # top-k of the batched candidate step vs the oracle's full sort
    idx, uni, cnt = st.topk_out
    r_idx, r_uni, r_cnt = orc.topk(ref, w.k)
    g_idx = idx[h:h + 1].cpu().numpy()
    assert int(cnt[h]) > 0
    assert_topk_sets_match(g_idx, r_idx, ref, l1, w.k)
    # and exactly the top-k of the GPU's own dense scores of this group
    g_all = dense.cpu().numpy()[0]
    for g in range(w.G):
        want = np.lexsort((np.arange(w.n), -g_all[g].astype(np.float64)))[:w.k]
        assert np.array_equal(g_idx[0, g], want)
    u = np.unique(g_idx.reshape(-1))
    assert int(cnt[h]) == len(u) and np.array_equal(uni[h, :len(u)].cpu().numpy(), u)


def test_fullsize_plan_every_group_bit_exact(step_1m, orc):
    w, planes, scales, s2, q, st = step_1m
    depth, active, na, theta = st.plan_out
    d_ref, a_ref, na_ref, _ = orc.plan(s2.cpu().numpy(), q.cpu().numpy(), 48)
    assert np.array_equal(depth.cpu().numpy(), d_ref)
    assert np.array_equal(np_u16(active), a_ref)
    assert np.array_equal(na.cpu().numpy(), na_ref)
    assert int(torch.min(st.topk_out[2])) > 0   # no group needed the dense rerun


def test_step_128k_sampled_groups(orc):
    """The 288 x 131072 step (a second full-size configuration)."""
    w = inputs.STEP_128K
    dev = torch.device("cuda", 0)
    planes, scales, s2, q, _ = bench.build_index(w, dev)
    st = fathom.Step(planes, scales, w.n, s2, w.G, w.k, budget=48)
    idx, uni, cnt = st.run(q)
    torch.cuda.synchronize()
    d_ref = orc.plan(s2.cpu().numpy(), q.cpu().numpy(), 48)[0]
    assert np.array_equal(st.plan_out[0].cpu().numpy(), d_ref)
    for h in (int(x) for x in np.linspace(5, 287, 16).round()):
        k = inputs.keys(w, h, h + 1, device="cuda")
        p_ref, s_ref = orc.pack(keys_for_oracle(k), nb_stride=planes.shape[-1])
        assert np.array_equal(np_u64(planes[h:h + 1]), p_ref)
        qn = q[h:h + 1].cpu().numpy()
        ref, l1 = orc.scan(p_ref, s_ref, d_ref[h:h + 1], qn, w.n)
        r_idx = orc.topk(ref, w.k)[0]
        assert_topk_sets_match(idx[h:h + 1].cpu().numpy(), r_idx, ref, l1, w.k)
        assert int(cnt[h]) > 0


def test_rotated_llama_step_full_size_sampled(orc):
    """The rotated Llama-shaped step at its full size (256 groups x 2^20 keys,
    keys rotated inside the pack kernel): the planes and scales of sampled
    groups' first 65,536 keys are bit-exact against the oracle's fp32 FMA
    chain and pack, and the candidate step proves every group exact."""
    from long_context_decode_bit_b200 import basis
    w = inputs.STEP_1M_LLAMA
    dev = torch.device("cuda", 0)
    planes, scales, s2, q, _ = bench.build_index(w, dev, rotated=True, log=lambda *a: None)
    st = fathom.Step(planes, scales, w.n, s2, w.G, w.k, budget=48)
    idx, uni, cnt = st.run(q, check_overflow=False)
    torch.cuda.synchronize()
    assert int(torch.min(cnt)) > 0
    m = 65536
    for h in (0, 100, 255):
        # The basis exactly as the index build formed it: per chunk of 8 groups.
        h0 = h - h % 8
        kc = inputs.keys(w, h0, min(w.H, h0 + 8), device="cuda")
        qc = inputs.queries(w, h0, min(w.H, h0 + 8), device="cuda").float().contiguous()
        U = basis.klt_basis(kc[:, :w.n_cal], qc)[h - h0:h - h0 + 1].contiguous()
        k = kc[h - h0:h - h0 + 1]
        del kc
        p_ref, s_ref = orc.pack_rotated(keys_for_oracle(k[:, :m]), U.cpu().numpy())
        nb = m // 64
        assert np.array_equal(np_u64(planes[h:h + 1])[..., :nb], p_ref[..., :nb])
        assert np.array_equal(np_u16(scales[h:h + 1])[..., :nb], s_ref[..., :nb])
    del planes, scales
    torch.cuda.empty_cache()


def test_token_major_store_full_size_sampled(step_1m, orc):
    """The token-major 4-bit copy of the 288 x 2^20 index holds the oracle's
    codes for sampled groups (every token)."""
    w, planes, scales, s2, q, st = step_1m
    for h in (3, 200):
        tm = fathom.nibbles_tm_from_planes(planes[h:h + 1], w.n)
        k = inputs.keys(w, h, h + 1, device="cuda")
        ref = orc.pack_nibbles(keys_for_oracle(k), nb_stride=planes.shape[-1])
        del k
        got = tm.cpu().numpy()[:, :w.n]
        lo, hi = got & 15, got >> 4
        codes = np.stack([lo, hi], axis=-1).reshape(1, w.n, w.D).transpose(0, 2, 1)
        sh = np.arange(16, dtype=np.uint64) * np.uint64(4)
        c = ((ref[..., None] >> sh) & np.uint64(15)).transpose(0, 1, 3, 2, 4).reshape(1, w.D, -1)[:, :, :w.n]
        assert np.array_equal(codes, c.astype(np.uint8))
        del tm
