"""Packed variable-length sequences through the C ABI (GPU).

A packed call holds several independent problems back to back: sequence s
owns query rows [cu_q[s], cu_q[s+1]) and key rows [cu_k[s], cu_k[s+1]) and
is bottom-right aligned on its own. Each sequence of a packed call must give
exactly what the same sequence gives alone (the kernels compute every work
item the same way; dQ, summed with fp32 reductions from several CTAs, within
a tight bound), and must match the oracle.
"""
import math

import numpy as np
import pytest
import torch

from tile_skipping_causal_b200 import mala
from tests.parity import check_bwd_blocks, check_fwd

pytestmark = pytest.mark.gpu

DEV = "cuda"
# (N_q, N_k) per sequence: ragged, block-aligned, a single query, a long
# context behind a short chunk, and a sequence without queries
LENGTHS = [(100, 300), (256, 256), (1, 77), (130, 900), (0, 50), (300, 301)]
HQ, HKV, D = 4, 2, 128


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tile_skipping_causal_b200 import build
    build.build()
    mala.load_library()


def _packed_inputs(seed):
    g = torch.Generator().manual_seed(seed)
    tq = sum(a for a, _ in LENGTHS)
    tk = sum(b for _, b in LENGTHS)
    q = (torch.randn(1, tq, HQ, D, generator=g) * 3 / math.sqrt(D)).bfloat16().to(DEV)
    k = torch.randn(1, tk, HKV, D, generator=g).bfloat16().to(DEV)
    v = torch.randn(1, tk, HKV, D, generator=g).bfloat16().to(DEV)
    do = torch.randn(1, tq, HQ, D, generator=g).bfloat16().to(DEV)
    cq = np.concatenate([[0], np.cumsum([a for a, _ in LENGTHS])]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum([b for _, b in LENGTHS])]).astype(np.int32)
    qb = np.concatenate([[0], np.cumsum([-(-a // 128) for a, _ in LENGTHS])]).astype(np.int64)
    return q, k, v, do, cq, ck, qb


def _seq(t, c, s):
    return t[:, c[s]:c[s + 1]]


@pytest.mark.parametrize("tau", [0.3, 2.0])
def test_packed_forward_equals_each_sequence_alone(tau):
    q, k, v, do, cq, ck, qb = _packed_inputs(1)
    o, lse, keep = mala.mala_fwd(q, k, v, tau, cu_seqlens_q=cq, cu_seqlens_k=ck)
    mala.check_device_error()
    assert lse.shape == (HQ, q.shape[1]) and keep.shape[:2] == (HQ, int(qb[-1]))
    for s, (nq, nk) in enumerate(LENGTHS):
        if nq == 0:
            continue
        qs, ks, vs = _seq(q, cq, s), _seq(k, ck, s), _seq(v, ck, s)
        o1, lse1, keep1 = mala.mala_fwd(qs, ks, vs, tau)
        mala.check_device_error()
        assert torch.equal(_seq(o, cq, s), o1), f"sequence {s}: O differs from the unpacked call"
        assert torch.equal(lse[:, cq[s]:cq[s + 1]], lse1[0]), f"sequence {s}: LSE differs"
        ks_words = keep[:, qb[s]:qb[s + 1]]
        w1 = keep1.shape[-1]
        assert torch.equal(ks_words[..., :w1], keep1[0]), f"sequence {s}: keep bits differ"
        assert not ks_words[..., w1:].any(), f"sequence {s}: bits beyond its key blocks"
        if nq <= 300:
            check_fwd(qs, ks, vs, _seq(o, cq, s), lse[:, cq[s]:cq[s + 1]][None],
                      ks_words[None, ..., :w1], tau, 128, 128)


@pytest.mark.parametrize("tau", [0.3, 2.0])
def test_packed_backward_equals_each_sequence_alone(tau):
    q, k, v, do, cq, ck, qb = _packed_inputs(2)
    o, lse, keep = mala.mala_fwd(q, k, v, tau, cu_seqlens_q=cq, cu_seqlens_k=ck)
    dq, dk, dv, bkeep = mala.mala_bwd(q, k, v, o, do, lse, tau, keep, with_bwd_mask=True,
                                      cu_seqlens_q=cq, cu_seqlens_k=ck)
    mala.check_device_error()
    for s, (nq, nk) in enumerate(LENGTHS):
        ks, vs = _seq(k, ck, s), _seq(v, ck, s)
        if nq == 0:
            # no query sees these keys: their gradients are zero
            assert not _seq(dk, ck, s).any() and not _seq(dv, ck, s).any()
            continue
        qs, dos = _seq(q, cq, s), _seq(do, cq, s)
        o1, lse1, keep1 = mala.mala_fwd(qs, ks, vs, tau)
        dq1, dk1, dv1, bkeep1 = mala.mala_bwd(qs, ks, vs, o1, dos, lse1, tau, keep1, with_bwd_mask=True)
        mala.check_device_error()
        assert torch.equal(_seq(dk, ck, s), dk1) and torch.equal(_seq(dv, ck, s), dv1), f"sequence {s}: dK/dV"
        rel = (_seq(dq, cq, s).float() - dq1.float()).norm() / dq1.float().norm().clamp_min(1e-30)
        assert rel < 1e-3, f"sequence {s}: dQ differs by {rel:.2e}"
        w1 = bkeep1.shape[-1]
        assert torch.equal(bkeep[:, qb[s]:qb[s + 1], :w1], bkeep1[0]), f"sequence {s}: backward bits"
        if nq <= 130:
            check_bwd_blocks(qs, ks, vs, dos, keep[:, qb[s]:qb[s + 1], :w1][None],
                             bkeep[:, qb[s]:qb[s + 1], :w1][None], _seq(dq, cq, s), _seq(dk, ck, s),
                             _seq(dv, ck, s), tau)


def test_packed_rejects_bad_offsets():
    q, k, v, do, cq, ck, qb = _packed_inputs(3)
    bad = cq.copy()
    bad[1] = -1                                           # decreasing right at the start
    with pytest.raises(mala.MalaError) as ei:
        mala.mala_fwd(q, k, v, 0.3, cu_seqlens_q=bad, cu_seqlens_k=ck)
    assert ei.value.code == mala.MALA_ERR_INVALID_ARG
    longer = cq.copy()
    longer[1:] += 250                                    # first sequence: more queries than keys
    longer[-1] = cq[-1]
    with pytest.raises(mala.MalaError):
        mala.mala_fwd(q, k, v, 0.3, cu_seqlens_q=longer, cu_seqlens_k=ck)
