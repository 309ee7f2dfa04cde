"""The device-side timeout path, on the GPU, without a fault.

Every wait inside the kernels is bounded. A call made with a wait limit far
below the time its waits legitimately take (wait_limit_ns of 1 ns or 100 ns)
makes them run out: the kernels stop early, drain the copies and MMAs they
already issued, free their tensor memory, return, and record
MALA_ERR_TIMEOUT, which mala_check_device_error() reports (and clears).
The next call with the default limit must then run normally and match the
oracle, which shows the context stayed usable and no stale state survived.
Each case is sized so that some wait of every CTA cannot be satisfied at
its first try (the first Q / K tile is still in flight), so the timeout is
certain under a limit of 1 ns or 100 ns.
"""
import pytest
import torch

from tile_skipping_causal_b200 import mala, synth
from tests.parity import check_bwd_blocks, check_decode, check_fwd

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tile_skipping_causal_b200 import build
    build.build()
    mala.load_library()


def _expect_timeout():
    with pytest.raises(mala.MalaError) as ei:
        mala.check_device_error()
    assert ei.value.code == mala.MALA_ERR_TIMEOUT, str(ei.value)
    mala.check_device_error()                   # the record was cleared


def _prefill(seed=5):
    w = synth.WORKLOADS["prefill_4k"]
    t = synth.make_prefill(w, seed, with_do=True, batch=1, seqlen=512)
    return {n: x.to(DEV) for n, x in t.items()}


@pytest.mark.parametrize("limit", [1, 100])
def test_forward_timeout_then_normal_call(limit):
    t = _prefill()
    mala.mala_fwd(t["q"], t["k"], t["v"], 1.0, wait_limit_ns=limit)
    _expect_timeout()
    o, lse, keep = mala.mala_fwd(t["q"], t["k"], t["v"], 1.0)
    mala.check_device_error()
    check_fwd(t["q"], t["k"], t["v"], o, lse, keep, 1.0, 128, 128)


@pytest.mark.parametrize("limit", [1, 100])
def test_group_vote_forward_timeout_then_normal_call(limit):
    w = synth.WORKLOADS["gqa_32k"]
    t = {n: x.to(DEV) for n, x in synth.make_prefill(w, 6, batch=1, seqlen=384).items()}
    mala.mala_fwd(t["q"], t["k"], t["v"], 64.0, group_vote=True, wait_limit_ns=limit)
    _expect_timeout()
    o, lse, keep = mala.mala_fwd(t["q"], t["k"], t["v"], 64.0, group_vote=True)
    mala.check_device_error()
    from tests.parity import check_fwd_group
    check_fwd_group(t["q"], t["k"], t["v"], o, lse, keep, 64.0)


@pytest.mark.parametrize("limit", [1, 100])
def test_backward_timeout_then_normal_call(limit):
    t = _prefill()
    o, lse, keep = mala.mala_fwd(t["q"], t["k"], t["v"], 1.0)
    mala.check_device_error()
    mala.mala_bwd(t["q"], t["k"], t["v"], o, t["do"], lse, 1.0, keep, wait_limit_ns=limit)
    _expect_timeout()
    dq, dk, dv, bkeep = mala.mala_bwd(t["q"], t["k"], t["v"], o, t["do"], lse, 1.0, keep, with_bwd_mask=True)
    mala.check_device_error()
    rep = check_bwd_blocks(t["q"], t["k"], t["v"], t["do"], keep, bkeep, dq, dk, dv, 1.0)
    assert rep["worst_rel_fro"] < 3e-2


@pytest.mark.parametrize("limit", [1, 100])
def test_decode_timeout_then_normal_call(limit):
    # one split over 32 key tiles: the producer must wait for ring slots,
    # so some wait of every CTA outlasts the limit
    splits = 1
    w = synth.DecodeWorkload("decode_timeout", 2, 8, 2, 4000, 128, 128, 5.0)
    q = synth.make_decode_query(w, 8)
    k, v = synth.fill_decode_cache(w, 8, q, DEV)
    q = q.to(DEV)
    mala.mala_decode(q, k, v, w.tau, 128, splits, wait_limit_ns=limit)
    _expect_timeout()
    o, lse, keep, P = mala.mala_decode(q, k, v, w.tau, 128, splits)
    mala.check_device_error()
    check_decode(q, k, v, o, lse, keep, w.tau, P)
