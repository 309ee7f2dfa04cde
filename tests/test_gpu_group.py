"""Group-joint voting in prefill (GPU): the query heads of a KV head decide
together per (query block, key tile), against the oracle's group-joint
prefill; the backward replays the group's forward mask."""
import pytest
import torch

from tile_skipping_causal_b200 import mala, synth
from tests.parity import check_bwd_blocks, check_fwd_group

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tile_skipping_causal_b200 import build
    build.build()
    mala.load_library()


def _prefill(name, seed, **kw):
    t = synth.make_prefill(synth.WORKLOADS[name], seed, with_do=True, **kw)
    return {n: x.to(DEV) for n, x in t.items()}


@pytest.mark.parametrize("tau", [0.2, 50.0])
def test_forward_group_vote_matches_oracle(tau):
    t = _prefill("gqa_32k", 5, batch=1, seqlen=1000)          # 32 query heads, 8 KV heads: G = 4
    o, lse, keep = mala.mala_fwd(t["q"], t["k"], t["v"], tau, group_vote=True)
    mala.check_device_error()
    nblk, ntiles, nkept = check_fwd_group(t["q"], t["k"], t["v"], o, lse, keep, tau)
    assert nblk == 8 * 8
    if tau >= 50.0:
        assert nkept < ntiles                                  # the case does skip


def test_forward_group_vote_chunked_prefill():
    t = _prefill("gqa_32k", 6, batch=1, seqlen=1000)
    qc = t["q"][:, -400:].contiguous()                         # the last 400 queries (bottom-right)
    o, lse, keep = mala.mala_fwd(qc, t["k"], t["v"], 50.0, group_vote=True)
    mala.check_device_error()
    check_fwd_group(qc, t["k"], t["v"], o, lse, keep, 50.0)


def test_forward_group_vote_with_single_head_groups_is_per_head():
    t = _prefill("prefill_4k", 7, batch=1, seqlen=700)        # 16 query heads = 16 KV heads
    a = mala.mala_fwd(t["q"], t["k"], t["v"], 1.0)
    b = mala.mala_fwd(t["q"], t["k"], t["v"], 1.0, group_vote=True)
    mala.check_device_error()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_backward_replays_the_group_forward_mask():
    t = _prefill("gqa_32k", 8, batch=1, seqlen=700)
    tau = 50.0
    o, lse, keep = mala.mala_fwd(t["q"], t["k"], t["v"], tau, group_vote=True)
    dq, dk, dv, bkeep = mala.mala_bwd(t["q"], t["k"], t["v"], o, t["do"], lse, tau, keep, with_bwd_mask=True)
    mala.check_device_error()
    rep = check_bwd_blocks(t["q"], t["k"], t["v"], t["do"], keep, bkeep, dq, dk, dv, tau, group_vote=True)
    assert rep["worst_rel_fro"] < 3e-2
