"""GPU parity of mala_fwd against the fp64 oracle (through the C ABI)."""
import math

import numpy as np
import pytest
import torch

from oracle import mala_oracle as orc
from tile_skipping_causal_b200 import mala, synth
from tests.parity import FwdReport, assert_close, check_decode, check_fwd, f64

pytestmark = pytest.mark.gpu

DEV = "cuda"
SEED = 42


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tile_skipping_causal_b200 import build
    build.build()
    mala.load_library()


def _run(w, seed=SEED, **kw):
    t = synth.make_prefill(w, seed, **kw)
    return {n: x.to(DEV) for n, x in t.items()}


def _fwd(t, tau, bq, bk, **kw):
    o, lse, keep = mala.mala_fwd(t["q"], t["k"], t["v"], tau, bq, bk, **kw)
    mala.check_device_error()
    return o, lse, keep


# ---------------------------------------------------------------- configs

@pytest.mark.parametrize("tau", [0.0, 0.05, 0.5])
def test_toy_fp32_512_full(tau):
    """One fp32 head, N=512, d=64, 64x64 tiles, planted previous-token keys."""
    w = synth.WORKLOADS["toy_fp32_512"]
    t = _run(w)
    o, lse, keep = _fwd(t, tau, 64, 64)
    rep = check_fwd(t["q"], t["k"], t["v"], o, lse, keep, tau, 64, 64)
    if tau == 0.0:
        assert rep.kept == rep.tiles
    else:
        assert rep.kept < rep.tiles          # the planted structure lets tiles be skipped


@pytest.mark.parametrize("tau", [0.01, 0.1, 1.0])
def test_prefill_recipe_reduced_all_blocks(tau):
    """Sharp/diffuse head recipe at N=1000 (ragged last block), every block."""
    w = synth.WORKLOADS["prefill_4k"]
    t = _run(w, batch=1, seqlen=1000)
    o, lse, keep = _fwd(t, tau, 128, 128)
    rep = check_fwd(t["q"], t["k"], t["v"], o, lse, keep, tau, 128, 128)
    assert rep.blocks == 16 * 8


def _spread_samples(B, H, nQB, n_i=3):
    out = []
    for b in range(B):
        for h in range(H):
            for i in sorted({0, nQB // 2, nQB - 1} if n_i == 3 else range(nQB)):
                out.append((b, h, i))
    return out


@pytest.mark.parametrize("tau", [0.01, 0.1, 1.0])
def test_prefill_4k_full_size_sampled(tau):
    w = synth.WORKLOADS["prefill_4k"]
    t = _run(w)
    o, lse, keep = _fwd(t, tau, 128, 128)
    samples = [(b, h, i) for b in (0, 1) for h in (0, 5, 8, 15) for i in (0, 17, 31)]
    check_fwd(t["q"], t["k"], t["v"], o, lse, keep, tau, 128, 128, samples)


@pytest.fixture(scope="module")
def gqa32k():
    return _run(synth.WORKLOADS["gqa_32k"])


@pytest.mark.parametrize("tau", [0.02, 0.2])
def test_gqa_32k_full_size_sampled(gqa32k, tau):
    t = gqa32k
    o, lse, keep = _fwd(t, tau, 128, 128)
    # heads from each third (diffuse 0-10, local 11-21, retrieval 22-31)
    samples = [(0, h, i) for h in (0, 10, 13, 21, 24, 31) for i in (0, 97, 255)]
    check_fwd(t["q"], t["k"], t["v"], o, lse, keep, tau, 128, 128, samples)


def test_gqa_recipe_reduced_all_blocks():
    t = _run(synth.WORKLOADS["gqa_32k"], seqlen=1536)
    o, lse, keep = _fwd(t, 0.2, 128, 128)
    check_fwd(t["q"], t["k"], t["v"], o, lse, keep, 0.2, 128, 128)


# ---------------------------------------------------------------- limits

def test_tau_zero_keeps_everything_and_is_dense():
    t = _run(synth.WORKLOADS["prefill_4k"], batch=1, seqlen=700)
    o, lse, keep = _fwd(t, 0.0, 128, 128)
    nQB = nKB = 6
    m = mala.unpack_mask(keep, nKB)
    assert (m == np.tril(np.ones((nQB, nKB), dtype=bool))[None, None]).all()
    check_fwd(t["q"], t["k"], t["v"], o, lse, keep, 0.0, 128, 128)


def test_tau_inf_keeps_only_diagonal():
    t = _run(synth.WORKLOADS["prefill_4k"], batch=1, seqlen=640)
    o, lse, keep = _fwd(t, math.inf, 128, 128)
    m = mala.unpack_mask(keep, 5)
    assert (m == np.eye(5, dtype=bool)[None, None]).all()
    check_fwd(t["q"], t["k"], t["v"], o, lse, keep, math.inf, 128, 128)


# ---------------------------------------------------------------- edge cases

def _random_bf16(B, N, Hq, Hkv, d, seed, sharp=3.0):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, N, Hq, d, generator=g) * sharp / math.sqrt(d)).bfloat16()
    k = torch.randn(B, N, Hkv, d, generator=g).bfloat16()
    v = torch.randn(B, N, Hkv, d, generator=g).bfloat16()
    return {"q": q.to(DEV), "k": k.to(DEV), "v": v.to(DEV)}


@pytest.mark.parametrize("N", [1, 5, 127, 128, 129, 255, 300])
@pytest.mark.parametrize("d", [64, 128])
def test_edge_lengths_gqa(N, d):
    t = _random_bf16(2, N, 4, 2, d, seed=N * 10 + d)
    o, lse, keep = _fwd(t, 0.3, 128, 128)
    check_fwd(t["q"], t["k"], t["v"], o, lse, keep, 0.3, 128, 128)


@pytest.mark.parametrize("bq,bk", [(64, 64), (32, 128), (128, 64), (16, 16)])
def test_cuda_core_path_block_sizes(bq, bk):
    t = _random_bf16(1, 333, 2, 1, 64, seed=bq + bk)
    o, lse, keep = _fwd(t, 0.2, bq, bk)
    check_fwd(t["q"], t["k"], t["v"], o, lse, keep, 0.2, bq, bk)


def test_explicit_head_map_and_packed_layout():
    B, N, H, d = 1, 400, 4, 128
    g = torch.Generator().manual_seed(7)
    qkv = torch.randn(B, N, 3, H, d, generator=g)
    qkv[:, :, 0] *= 3.0 / math.sqrt(d)
    qkv = qkv.bfloat16().to(DEV)
    q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]       # strided views
    hmap = [3, 0, 2, 1]
    o, lse, keep = mala.mala_fwd(q, k, v, 0.2, 128, 128, q_to_kv=hmap)
    mala.check_device_error()
    # the oracle reads the same head map through a permuted copy of K/V
    kp = k[:, :, hmap].contiguous()
    vp = v[:, :, hmap].contiguous()
    check_fwd(q, kp, vp, o, lse, keep, 0.2, 128, 128)


def test_stats_count_kept_tiles():
    t = _run(synth.WORKLOADS["prefill_4k"], batch=1, seqlen=1024)
    stats = torch.zeros(4, dtype=torch.int64, device=DEV)
    o, lse, keep = _fwd(t, 0.1, 128, 128, stats=stats)
    m = mala.unpack_mask(keep, 8)
    s = stats.cpu().tolist()
    assert s[0] == 16 * 8 * 9 // 2
    assert s[1] == m.sum()
    assert s[2] == m.sum() * 128 * 128


# ------------------------------------------- bottom-right causal alignment
# A chunk of N_q queries appended to a context of N_k - N_q keys: query q sits
# at position q + N_k - N_q. The chunk is the last N_q query rows of a longer
# seeded problem (a strided view, as a chunked-prefill caller would pass it).

@pytest.mark.parametrize("Nq,Nk", [(1, 700), (100, 164), (128, 384), (200, 456), (300, 301), (129, 1000)])
@pytest.mark.parametrize("d", [64, 128])
def test_bottom_right_chunk_gqa(Nq, Nk, d):
    t = _random_bf16(2, Nk, 4, 2, d, seed=Nq * 7 + Nk + d)
    q = t["q"][:, Nk - Nq:]
    o, lse, keep = mala.mala_fwd(q, t["k"], t["v"], 0.3, 128, 128)
    mala.check_device_error()
    assert keep.shape[-1] == mala.mask_words(-(-Nk // 128))
    check_fwd(q, t["k"], t["v"], o, lse, keep, 0.3, 128, 128)


@pytest.mark.parametrize("tau", [0.1, 1.0])
def test_bottom_right_chunk_recipe_skips(tau):
    t = _run(synth.WORKLOADS["prefill_4k"], batch=1, seqlen=1024)
    q = t["q"][:, 1024 - 320:]
    stats = torch.zeros(4, dtype=torch.int64, device=DEV)
    o, lse, keep = mala.mala_fwd(q, t["k"], t["v"], tau, 128, 128, stats=stats)
    mala.check_device_error()
    rep = check_fwd(q, t["k"], t["v"], o, lse, keep, tau, 128, 128)
    tested, kept = stats[0].item(), stats[1].item()
    assert tested == rep.tiles and kept == rep.kept
    if tau == 1.0:
        assert kept < tested                      # the sharp heads skip tiles


def test_bottom_right_cuda_core_path():
    g = torch.Generator().manual_seed(3)
    B, Nk, Nq, H, d = 1, 333, 90, 2, 64
    q = (torch.randn(B, Nk, H, d, generator=g) * 3 / math.sqrt(d))[:, Nk - Nq:].to(DEV)
    k = torch.randn(B, Nk, H, d, generator=g).to(DEV)
    v = torch.randn(B, Nk, H, d, generator=g).to(DEV)
    o, lse, keep = mala.mala_fwd(q, k, v, 0.2, 64, 64)
    mala.check_device_error()
    check_fwd(q, k, v, o, lse, keep, 0.2, 64, 64)


def test_bottom_right_single_query_matches_decode():
    """N_q = 1 is the decoding case (L_0 = N_k): the prefill kernel on a
    one-row chunk and the decode kernel without splits agree."""
    g = torch.Generator().manual_seed(11)
    B, Nk, Hq, Hkv, d = 2, 1000, 8, 2, 128
    q = (torch.randn(B, 1, Hq, d, generator=g) * 3 / math.sqrt(d)).bfloat16().to(DEV)
    k = torch.randn(B, Nk, Hkv, d, generator=g).bfloat16().to(DEV)
    v = torch.randn(B, Nk, Hkv, d, generator=g).bfloat16().to(DEV)
    o, lse, keep = mala.mala_fwd(q, k, v, 0.05, 128, 128)
    od, lsed, keepd, P = mala.mala_decode(q, k, v, 0.05, 128, 1)
    mala.check_device_error()
    assert P == 1
    check_fwd(q, k, v, o, lse, keep, 0.05, 128, 128)
    check_decode(q, k, v, od, lsed, keepd, 0.05, P)
    assert_close(f64(o), f64(od), "O fwd vs decode")
    assert_close(lse.cpu().numpy().reshape(B, Hq), lsed.cpu().numpy(), "LSE fwd vs decode")
