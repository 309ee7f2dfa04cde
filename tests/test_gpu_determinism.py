"""Run-to-run reproducibility of the CUDA kernels at full workload sizes.

Forward and decode have no atomics and a fixed reduction order, and the
backward's dK/dV accumulate in TMEM in a fixed order, so repeated launches
must agree bit for bit; a race between the pipeline roles of a kernel would
show up here as a difference. dQ is summed with fp32 reductions from several
CTAs, so its rounding may differ between launches within a tight bound."""
import pytest
import torch

from tile_skipping_causal_b200 import mala, synth

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tile_skipping_causal_b200 import build
    build.build()
    mala.load_library()


@pytest.mark.parametrize("name,tau", [("gqa_32k", 0.02), ("prefill_4k", 0.1)])
def test_forward_is_bitwise_reproducible(name, tau):
    t = {n: x.to(DEV) for n, x in synth.make_prefill(synth.WORKLOADS[name], 42).items()}
    ref = mala.mala_fwd(t["q"], t["k"], t["v"], tau)
    mala.check_device_error()
    for _ in range(3):
        o, lse, keep = mala.mala_fwd(t["q"], t["k"], t["v"], tau)
        mala.check_device_error()
        assert torch.equal(o, ref[0]) and torch.equal(lse, ref[1]) and torch.equal(keep, ref[2])


def test_backward_reproducible():
    w = synth.WORKLOADS["train_8k"]
    t = {n: x.to(DEV) for n, x in synth.make_prefill(w, 42).items()}
    o, lse, keep = mala.mala_fwd(t["q"], t["k"], t["v"], 0.1)
    ref = mala.mala_bwd(t["q"], t["k"], t["v"], o, t["do"], lse, 0.1, keep, with_bwd_mask=True)
    mala.check_device_error()
    for _ in range(2):
        dq, dk, dv, bk = mala.mala_bwd(t["q"], t["k"], t["v"], o, t["do"], lse, 0.1, keep, with_bwd_mask=True)
        mala.check_device_error()
        assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2]) and torch.equal(bk, ref[3])
        rel = (dq.float() - ref[0].float()).norm() / ref[0].float().norm()
        assert rel < 1e-3


def test_decode_is_bitwise_reproducible():
    w = synth.decode_workload(65536)
    q = synth.make_decode_query(w, 42)
    k, v = synth.fill_decode_cache(w, 42, q, DEV, slices=[])
    qd = q.to(DEV)
    ref = mala.mala_decode(qd, k, v, w.tau)
    mala.check_device_error()
    for _ in range(3):
        o, lse, keep, P = mala.mala_decode(qd, k, v, w.tau)
        mala.check_device_error()
        assert torch.equal(o, ref[0]) and torch.equal(lse, ref[1]) and torch.equal(keep, ref[2])


def test_caller_stream_gives_the_same_results():
    """Calls on a caller-given stream (workspaces allocated by the binding
    are kept alive for that stream) match the calls on the current stream."""
    w = synth.WORKLOADS["train_8k"]
    t = {n: x.to(DEV) for n, x in synth.make_prefill(w, 42, batch=1, seqlen=1024).items()}
    o, lse, keep = mala.mala_fwd(t["q"], t["k"], t["v"], 0.1)
    dq, dk, dv, _ = mala.mala_bwd(t["q"], t["k"], t["v"], o, t["do"], lse, 0.1, keep)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    o2, lse2, keep2 = mala.mala_fwd(t["q"], t["k"], t["v"], 0.1, stream=side)
    dq2, dk2, dv2, _ = mala.mala_bwd(t["q"], t["k"], t["v"], o2, t["do"], lse2, 0.1, keep2, stream=side)
    # allocations on the current stream meanwhile may not reuse the side
    # stream's workspaces while its kernels run
    junk = [torch.full((1 << 20,), 7.0, device=DEV) for _ in range(64)]
    torch.cuda.current_stream().wait_stream(side)
    mala.check_device_error()
    del junk
    assert torch.equal(o, o2) and torch.equal(lse, lse2) and torch.equal(keep, keep2)
    assert torch.equal(dk, dk2) and torch.equal(dv, dv2)
    assert (dq.float() - dq2.float()).norm() <= 1e-3 * dq.float().norm()
