"""mala_decode_noalloc against mala_decode (GPU, through the C ABI).

mala_decode_noalloc serves callers that cannot allocate device memory: code
that is only handed its input and output buffers, for instance a plugin in a
host framework that owns every allocation and offers no workspace, or a
serving loop that allows no allocation once it runs. Instead of a caller
workspace it keeps the split-KV partials in a buffer built into the library.

The test runs both entry points on the same inputs twice in a row, with
different inputs the second time so that stale contents of the shared
built-in buffer would show, and requires the same outputs within the parity
tolerances used by the other tests. This file is collected last so that a
run stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from tile_skipping_causal_b200 import mala, synth
from tests.parity import ATOL, RTOL, assert_close, f64

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tile_skipping_causal_b200 import build
    build.build()
    mala.load_library()


def _inputs(seed, Nk=4096, Hkv=8):
    # decode workload shape with the sink / needle recipe: batch 64, 32 query
    # heads, 8 KV heads; the library picks 3 splits, whose partials (3.2 MB)
    # fit in the built-in 4 MiB buffer
    w = synth.DecodeWorkload("decode_noalloc", 64, 32, Hkv, Nk, 128, 128, 0.05)
    q = synth.make_decode_query(w, seed)
    k, v = synth.fill_decode_cache(w, seed, q, DEV, slices=[])
    return w, q.to(DEV), k, v


def test_noalloc_matches_workspace_decode_on_two_calls():
    for call, seed in enumerate((11, 12)):
        w, q, k, v = _inputs(seed)
        o_ref, lse_ref, keep_ref, p_ref = mala.mala_decode(q, k, v, w.tau, 128, 0)
        o, lse, keep, p = mala.mala_decode_noalloc(q, k, v, w.tau, 128, 0)
        mala.check_device_error()
        assert p == p_ref and p > 1, (call, p, p_ref)
        assert_close(f64(o), f64(o_ref), f"call {call} O", ATOL, RTOL)
        assert_close(lse.cpu().numpy(), lse_ref.cpu().numpy(), f"call {call} LSE", ATOL, RTOL)
        assert torch.equal(keep, keep_ref), f"call {call}: keep masks differ"


def test_noalloc_rejects_partials_larger_than_the_buffer():
    w, q, k, v = _inputs(13, Nk=8192)
    per_split = w.batch * w.heads_q * (128 + 1) * 4
    too_many = mala.DECODE_NOALLOC_SCRATCH_BYTES // per_split + 1
    with pytest.raises(mala.MalaError) as ei:
        mala.mala_decode_noalloc(q, k, v, w.tau, 128, too_many)
    assert ei.value.code == mala.MALA_ERR_WORKSPACE
    assert "built-in buffer" in str(ei.value)
    # within the limit it still agrees with the workspace entry point
    fits = mala.DECODE_NOALLOC_SCRATCH_BYTES // per_split
    o_ref, lse_ref, keep_ref, _ = mala.mala_decode(q, k, v, w.tau, 128, fits)
    o, lse, keep, p = mala.mala_decode_noalloc(q, k, v, w.tau, 128, fits)
    mala.check_device_error()
    assert p == fits
    assert_close(f64(o), f64(o_ref), "O", ATOL, RTOL)
    assert torch.equal(keep, keep_ref)


def test_noalloc_lowers_the_automatic_split_count_to_fit():
    """With 4 KV heads per sequence the automatic choice is 5 splits, whose
    partials (5.3 MB) exceed the built-in buffer; the entry point lowers the
    count until they fit (3 splits, 3.2 MB) and then computes what the
    workspace entry point computes with that many splits."""
    w, q, k, v = _inputs(14, Nk=4096, Hkv=4)
    per_split = w.batch * w.heads_q * (128 + 1) * 4
    _, _, _, p_auto = mala.mala_decode(q, k, v, w.tau, 128, 0)
    o, lse, keep, p = mala.mala_decode_noalloc(q, k, v, w.tau, 128, 0)
    mala.check_device_error()
    assert per_split * p_auto > mala.DECODE_NOALLOC_SCRATCH_BYTES
    assert 1 < p < p_auto and per_split * p <= mala.DECODE_NOALLOC_SCRATCH_BYTES < per_split * (p + 1)
    o_ref, lse_ref, keep_ref, p_ref = mala.mala_decode(q, k, v, w.tau, 128, p)
    assert p_ref == p
    assert_close(f64(o), f64(o_ref), "O", ATOL, RTOL)
    assert_close(lse.cpu().numpy(), lse_ref.cpu().numpy(), "LSE", ATOL, RTOL)
    assert torch.equal(keep, keep_ref)
