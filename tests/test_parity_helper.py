"""The parity checker accepts correct results and rejects wrong ones (CPU).

Feeds tests/parity.py the oracle's own outputs dressed as GPU tensors, then
plants mistakes in copies of them (an output element, an LSE entry, a mask
bit) and checks that each is caught."""
import numpy as np
import pytest
import torch

from oracle import mala_oracle as orc
from tile_skipping_causal_b200 import mala, synth
from tests import parity


def _case(tau):
    t = synth.make_prefill(synth.WORKLOADS["prefill_4k"], 3, batch=1, seqlen=300)
    q, k, v = t["q"], t["k"], t["v"]
    O, lse, keep, margin = orc.forward(parity.f64(q), parity.f64(k), parity.f64(v), 128, 128, tau)
    o = torch.from_numpy(O).to(torch.bfloat16)
    lse_t = torch.from_numpy(lse).float()
    words = torch.from_numpy(mala.pack_mask(keep))
    return q, k, v, o, lse_t, words, keep, margin


@pytest.mark.parametrize("tau", [0.0, 0.1, 1.0])
def test_checker_accepts_oracle_output(tau):
    q, k, v, o, lse, words, keep, _ = _case(tau)
    rep = parity.check_fwd(q, k, v, o, lse, words, tau, 128, 128)
    assert rep.blocks == 16 * 3 and rep.replayed_blocks == 0


def test_checker_rejects_wrong_output():
    q, k, v, o, lse, words, keep, _ = _case(0.1)
    o2 = o.clone()
    o2[0, 200, 9, 17] += 0.25
    with pytest.raises(AssertionError, match="O"):
        parity.check_fwd(q, k, v, o2, lse, words, 0.1, 128, 128)
    lse2 = lse.clone()
    lse2[0, 3, 150] += 0.5            # beyond 1e-2 + 2e-2 * |lse|
    with pytest.raises(AssertionError, match="LSE"):
        parity.check_fwd(q, k, v, o, lse2, words, 0.1, 128, 128)


def test_checker_rejects_wrong_decision():
    q, k, v, o, lse, words, keep, margin = _case(1.0)
    # flip a decision far from the threshold: must be reported
    b, h, i, j = np.argwhere(~np.isnan(margin) & (np.abs(margin) > 0.1) & (np.arange(3)[None, None, :, None] > 0))[0]
    keep2 = keep.copy()
    keep2[b, h, i, j] = not keep2[b, h, i, j]
    with pytest.raises(AssertionError):
        parity.check_fwd(q, k, v, o, lse, torch.from_numpy(mala.pack_mask(keep2)), 1.0, 128, 128)


def test_checker_rejects_bits_above_diagonal():
    q, k, v, o, lse, words, keep, _ = _case(0.1)
    keep2 = keep.copy()
    keep2[0, 0, 0, 2] = True
    with pytest.raises(AssertionError, match="outside"):
        parity.check_fwd(q, k, v, o, lse, torch.from_numpy(mala.pack_mask(keep2)), 0.1, 128, 128)


def _dec_case(tau, P):
    w = synth.DecodeWorkload("d", 1, 8, 2, 700, 128, 128, tau)
    q = synth.make_decode_query(w, 5)
    k, v = synth.fill_decode_cache(w, 5, q, "cpu")
    O, lse, keep, margin = orc.decode(parity.f64(q), parity.f64(k), parity.f64(v), 128, tau, P)
    return q, k, v, torch.from_numpy(O).to(torch.bfloat16), torch.from_numpy(lse).float(), keep, margin


def test_decode_checker_accepts_oracle_output():
    q, k, v, o, lse, keep, _ = _dec_case(0.05, 2)
    rep = parity.check_decode(q, k, v, o, lse, torch.from_numpy(mala.pack_mask(keep)), 0.05, 2)
    assert rep.heads == 8 and rep.replayed == 0


def test_decode_checker_rejects_wrong_decision_and_output():
    q, k, v, o, lse, keep, margin = _dec_case(2.0, 1)
    b, h, j = np.argwhere(~np.isnan(margin) & (np.abs(margin) > 0.1))[0]
    keep2 = keep.copy()
    keep2[b, h, j] = not keep2[b, h, j]
    with pytest.raises(AssertionError):
        parity.check_decode(q, k, v, o, lse, torch.from_numpy(mala.pack_mask(keep2)), 2.0, 1)
    o2 = o.clone()
    o2[0, 0, 3, 5] += 0.3
    with pytest.raises(AssertionError, match="O"):
        parity.check_decode(q, k, v, o2, lse, torch.from_numpy(mala.pack_mask(keep)), 2.0, 1)


def test_backward_checker_accepts_oracle_and_rejects_planted_error():
    t = synth.make_prefill(synth.WORKLOADS["train_8k"], 4, batch=1, seqlen=300, with_do=True)
    q, k, v, do = t["q"], t["k"], t["v"], t["do"]
    tau = 0.1
    O, lse, keep, _ = orc.forward(parity.f64(q), parity.f64(k), parity.f64(v), 128, 128, tau)
    Ob, zf = parity.as_operator_outputs(O, lse)
    dq, dk, dv, bkeep = orc.backward(parity.f64(q), parity.f64(k), parity.f64(v), Ob, parity.f64(do), zf,
                                     128, 128, tau, keep)
    fw = torch.from_numpy(mala.pack_mask(keep))
    bw = torch.from_numpy(mala.pack_mask(bkeep))
    cast = lambda x: torch.from_numpy(x).to(torch.bfloat16)
    rep = parity.check_bwd_blocks(q, k, v, do, fw, bw, cast(dq), cast(dk), cast(dv), tau)
    assert rep["worst_rel_fro"] < 1e-2
    dk_bad = dk.copy()
    dk_bad[0, :, 3] *= 1.5            # one head of 16 off by 50%: about 12% of the tensor
    with pytest.raises(AssertionError, match="dK"):
        parity.check_bwd_blocks(q, k, v, do, fw, bw, cast(dq), cast(dk_bad), cast(dv), tau)
