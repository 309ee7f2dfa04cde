"""GPU parity of mala_decode (split-KV decoding) against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

from oracle import mala_oracle as orc
from tile_skipping_causal_b200 import mala, synth
from tests.parity import check_decode, check_decode_group

pytestmark = pytest.mark.gpu

DEV = "cuda"
SEED = 42


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tile_skipping_causal_b200 import build
    build.build()
    mala.load_library()


def _decode(q, k, v, tau, splits=0, **kw):
    o, lse, keep, P = mala.mala_decode(q, k, v, tau, 128, splits, **kw)
    mala.check_device_error()
    return o, lse, keep, P


def _small(batch, Nk, seed=SEED, Hq=32, Hkv=8):
    w = synth.DecodeWorkload("decode_small", batch, Hq, Hkv, Nk, 128, 128, 0.05)
    q = synth.make_decode_query(w, seed)
    k, v = synth.fill_decode_cache(w, seed, q, DEV)
    return w, q.to(DEV), k, v


@pytest.mark.parametrize("Nk", [300, 1000, 4096])
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_decode_recipe_reduced_all_heads(Nk, splits):
    w, q, k, v = _small(2, Nk)
    o, lse, keep, P = _decode(q, k, v, w.tau, splits)
    if splits:
        assert P == splits
    rep = check_decode(q, k, v, o, lse, keep, w.tau, P)
    assert rep.heads == 2 * 32


@pytest.mark.parametrize("Nk", synth.DECODE_SEQLENS)
def test_decode_full_size_sampled(Nk):
    w = synth.decode_workload(Nk)
    q = synth.make_decode_query(w, SEED)
    sample_kv = [(0, 0), (17, 3), (63, 7)]
    k, v = synth.fill_decode_cache(w, SEED, q, DEV, slices=sample_kv)
    qd = q.to(DEV)
    o, lse, keep, P = _decode(qd, k, v, w.tau)
    heads = [(b, hk * 4 + g) for (b, hk) in sample_kv for g in range(4)]
    rep = check_decode(qd, k, v, o, lse, keep, w.tau, P, heads=heads)
    assert rep.heads == len(heads)
    del k, v
    torch.cuda.empty_cache()


@pytest.mark.parametrize("Nk,splits,tau", [(1000, 1, 5.0), (1000, 3, 50.0), (4096, 0, 5.0),
                                           (4096, 1, 50.0), (4096, 3, 50.0), (129, 0, 50.0)])
def test_decode_per_head_with_disagreeing_group_heads(Nk, splits, tau):
    """Per-head decisions ("Fused decoding execution"): a V tile is read when
    some head of the group retains it, and only the retaining heads
    accumulate it. At these tau the needle recipe makes heads of one group
    disagree on many tiles, so the kernel runs the path that loads V for the
    group and zeroes P for the heads that skip."""
    w, q, k, v = _small(2, Nk, seed=21)
    stats = torch.zeros(4, dtype=torch.int64, device=DEV)
    o, lse, keep, P = _decode(q, k, v, tau, splits, stats=stats)
    if splits:
        assert P == splits
    nKB = -(-Nk // 128)
    m = mala.unpack_mask(keep, nKB).reshape(2, 8, 4, nKB)
    disagree = m.any(axis=2) & ~m.all(axis=2)
    if Nk >= 1000:
        assert disagree.sum() > 0, "no tile with heads of one group deciding differently"
    tested, vread, kept_heads = (int(x) for x in stats.cpu().tolist()[:3])
    assert tested == 2 * 8 * nKB
    assert vread == int(m.any(axis=2).sum())          # V read iff some head of the group retains
    assert kept_heads == int(m.sum())
    rep = check_decode(q, k, v, o, lse, keep, tau, P)
    assert rep.heads == 2 * 32


def test_decode_tau_zero_is_dense():
    w, q, k, v = _small(1, 777)
    o, lse, keep, P = _decode(q, k, v, 0.0, 2)
    assert mala.unpack_mask(keep, 7).all()
    check_decode(q, k, v, o, lse, keep, 0.0, P)


def test_decode_tau_inf_keeps_first_tile_of_each_split():
    w, q, k, v = _small(1, 1280)
    o, lse, keep, P = _decode(q, k, v, math.inf, 3)
    m = mala.unpack_mask(keep, 10)
    expect = np.zeros(10, dtype=bool)
    for (t0, t1) in orc.split_ranges(10, 3):
        expect[t1 - 1] = True
    assert (m == expect[None, None]).all()
    check_decode(q, k, v, o, lse, keep, math.inf, P)


@pytest.mark.parametrize("Nk", [1, 127, 128, 129])
def test_decode_edge_lengths(Nk):
    w, q, k, v = _small(2, Nk)
    o, lse, keep, P = _decode(q, k, v, 0.05)
    check_decode(q, k, v, o, lse, keep, 0.05, P)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 1), (6, 2)])
def test_decode_group_sizes(Hq, Hkv):
    w, q, k, v = _small(2, 640, Hq=Hq, Hkv=Hkv)
    o, lse, keep, P = _decode(q, k, v, 0.05, 2)
    check_decode(q, k, v, o, lse, keep, 0.05, P)


def test_decode_explicit_head_map():
    w, q, k, v = _small(1, 512, Hq=4, Hkv=2)
    hmap = [1, 0, 0, 1]
    o, lse, keep, P = _decode(q, k, v, 0.05, 2, q_to_kv=hmap)
    kp = k[:, :, hmap].contiguous()
    vp = v[:, :, hmap].contiguous()
    # the oracle reads the same map through per-head copies (group of 1)
    check_decode(q, kp, vp, o, lse, keep, 0.05, P)


def test_decode_stats():
    w, q, k, v = _small(1, 2048)
    stats = torch.zeros(4, dtype=torch.int64, device=DEV)
    o, lse, keep, P = _decode(q, k, v, 0.05, 4, stats=stats)
    m = mala.unpack_mask(keep, 16)
    s = stats.cpu().tolist()
    assert s[0] == 8 * 16                     # (b, kv head) x tiles
    assert s[2] == m.sum()                    # head-tiles retained
    grp = m.reshape(1, 8, 4, 16).any(axis=2)  # V read iff some head of the group retains
    assert s[1] == grp.sum()


# ------------------------------------------------------------ e4m3 KV cache
# The decode recipe's cache quantised to OCP e4m3 codes with a scale per
# tensor; the oracle runs on the dequantised values (code * scale), which
# are exactly what the kernel computes with.

def _quantise(x, scale):
    codes = (x.float() / scale).to(torch.float8_e4m3fn)
    return codes, codes.float() * scale


@pytest.mark.parametrize("Nk,splits,scales", [(1000, 1, (1.0, 1.0)), (1000, 3, (0.5, 2.0)),
                                               (4096, 0, (0.25, 0.75)), (129, 0, (1.0, 0.5))])
def test_decode_e4m3_cache(Nk, splits, scales):
    w, q, k, v = _small(2, Nk, seed=7)
    sk, sv = scales
    kc, kd = _quantise(k, sk)
    vc, vd = _quantise(v, sv)
    stats = torch.zeros(4, dtype=torch.int64, device=DEV)
    o, lse, keep, P = _decode(q, kc, vc, w.tau, splits, k_scale=sk, v_scale=sv, stats=stats)
    if splits:
        assert P == splits
    rep = check_decode(q, kd, vd, o, lse, keep, w.tau, P)
    assert rep.heads == 2 * 32
    assert stats[0].item() == 2 * 8 * -(-Nk // 128)


def test_decode_e4m3_per_head_with_disagreeing_group_heads():
    """The e4m3 instantiation of the per-head path at a tau where heads of a
    group disagree (V read for the group, P zeroed for skipping heads)."""
    w, q, k, v = _small(2, 3000, seed=22)
    kc, kd = _quantise(k, 0.5)
    vc, vd = _quantise(v, 1.5)
    o, lse, keep, P = _decode(q, kc, vc, 50.0, 0, k_scale=0.5, v_scale=1.5)
    m = mala.unpack_mask(keep, 24).reshape(2, 8, 4, 24)
    assert (m.any(axis=2) & ~m.all(axis=2)).sum() > 0
    rep = check_decode(q, kd, vd, o, lse, keep, 50.0, P)
    assert rep.heads == 2 * 32


def test_decode_e4m3_large_cache_sampled():
    """Batch 64, 32 query heads, 8 KV heads, N_k = 16384 (1 GB of e4m3 codes
    per cache), sampled heads against the oracle."""
    w = synth.decode_workload(16384)
    q = synth.make_decode_query(w, SEED)
    sample_kv = [(0, 0), (40, 5)]
    k, v = synth.fill_decode_cache(w, SEED, q, DEV, slices=sample_kv)
    kc, kd = _quantise(k, 0.5)
    vc, vd = _quantise(v, 0.5)
    del k, v
    qd = q.to(DEV)
    o, lse, keep, P = _decode(qd, kc, vc, w.tau, k_scale=0.5, v_scale=0.5)
    heads = [(b, hk * 4 + g) for (b, hk) in sample_kv for g in range(4)]
    rep = check_decode(qd, kd, vd, o, lse, keep, w.tau, P, heads=heads)
    assert rep.heads == len(heads)
    del kc, vc, kd, vd


def test_decode_e4m3_rejects_bad_scales():
    w, q, k, v = _small(1, 300)
    kc, _ = _quantise(k, 1.0)
    vc, _ = _quantise(v, 1.0)
    with pytest.raises(mala.MalaError):
        mala.mala_decode(q, kc, vc, w.tau, k_scale=0.0)
    with pytest.raises(ValueError):
        mala.mala_decode(q, kc, v, w.tau)            # mixed cache types


# ------------------------------------------------------ group-joint voting

@pytest.mark.parametrize("Nk,splits,tau", [(1000, 1, 0.05), (1000, 3, 5.0), (4096, 0, 5.0),
                                           (4096, 1, 50.0), (129, 0, 50.0)])
def test_decode_group_vote_matches_oracle(Nk, splits, tau):
    w, q, k, v = _small(2, Nk, seed=11)
    stats = torch.zeros(4, dtype=torch.int64, device=DEV)
    o, lse, keep, P = _decode(q, k, v, tau, splits, group_vote=True, stats=stats)
    rep = check_decode_group(q, k, v, o, lse, keep, tau, P)
    assert rep.heads == 2 * 32
    tested, vread, kept_heads = (int(x) for x in stats.cpu().tolist()[:3])
    assert tested == 2 * 8 * -(-Nk // 128)
    assert kept_heads == 4 * vread                   # every head accumulates every V tile read
    if tau >= 50.0 and Nk > 1000:
        assert vread < tested                        # the case does skip


def test_decode_group_vote_with_single_head_groups_is_per_head():
    w, q, k, v = _small(2, 2000, seed=12, Hq=8, Hkv=8)
    a = _decode(q, k, v, 5.0, 0)
    b = _decode(q, k, v, 5.0, 0, group_vote=True)
    assert a[3] == b[3]
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)


def test_decode_group_vote_e4m3_cache():
    w, q, k, v = _small(1, 3000, seed=13)
    kc, kd = _quantise(k, 0.5)
    vc, vd = _quantise(v, 1.0)
    o, lse, keep, P = _decode(q, kc, vc, 5.0, 0, group_vote=True, k_scale=0.5, v_scale=1.0)
    rep = check_decode_group(q, kd, vd, o, lse, keep, 5.0, P)
    assert rep.heads == 32
