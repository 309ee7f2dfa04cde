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


# ------------------------------------------------------ group-joint voting

def _group_case(tau, seqlen=300):
    t = synth.make_prefill(synth.WORKLOADS["gqa_32k"], 4, batch=1, seqlen=seqlen)
    q, k, v = t["q"], t["k"], t["v"]
    q64, k64, v64 = parity.f64(q), parity.f64(k), parity.f64(v)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    nQB = nKB = -(-N // 128)
    O = np.zeros((B, N, Hq, d))
    lse = np.zeros((B, Hq, N))
    keep = np.zeros((B, Hq, nQB, nKB), dtype=bool)
    margin = np.full((B, Hkv, nQB, nKB), np.nan)
    for hk in range(Hkv):
        Qg = np.stack([q64[0, :, hk * G + g] for g in range(G)])
        Og, zg, kg, mg = orc.forward_group(Qg, k64[0, :, hk], v64[0, :, hk], 128, 128, tau)
        for g in range(G):
            O[0, :, hk * G + g] = Og[g]
            lse[0, hk * G + g] = zg[g]
            keep[0, hk * G + g] = kg
        margin[0, hk] = mg
    o = torch.from_numpy(O).to(torch.bfloat16)
    return q, k, v, o, torch.from_numpy(lse).float(), keep, margin, G


def test_group_checker_accepts_oracle_output():
    q, k, v, o, lse, keep, _, _ = _group_case(5.0)
    nblk, ntiles, nkept = parity.check_fwd_group(q, k, v, o, lse, torch.from_numpy(mala.pack_mask(keep)), 5.0)
    assert nblk == 8 * 3 and nkept <= ntiles


def test_group_checker_rejects_heads_that_disagree():
    q, k, v, o, lse, keep, _, G = _group_case(5.0)
    keep2 = keep.copy()
    keep2[0, 1, 2, 0] = not keep2[0, 1, 2, 0]          # head 1 alone flips a bit
    with pytest.raises(AssertionError, match="different keep bits"):
        parity.check_fwd_group(q, k, v, o, lse, torch.from_numpy(mala.pack_mask(keep2)), 5.0)


def test_group_checker_rejects_a_wrong_group_decision():
    q, k, v, o, lse, keep, margin, G = _group_case(5.0)
    # a group decision far from the threshold, flipped for all of the group's heads
    b, hk, i, j = np.argwhere(~np.isnan(margin) & np.isfinite(margin) & (np.abs(margin) > 0.1))[0]
    keep2 = keep.copy()
    keep2[b, hk * G:(hk + 1) * G, i, j] = ~keep2[b, hk * G, i, j]
    with pytest.raises(AssertionError):
        parity.check_fwd_group(q, k, v, o, lse, torch.from_numpy(mala.pack_mask(keep2)), 5.0)


def test_group_checker_rejects_wrong_output():
    q, k, v, o, lse, keep, _, _ = _group_case(5.0)
    o2 = o.clone()
    o2[0, 250, 13, 5] += 0.25
    with pytest.raises(AssertionError, match="O"):
        parity.check_fwd_group(q, k, v, o2, lse, torch.from_numpy(mala.pack_mask(keep)), 5.0)


def _group_decode_case(tau, P):
    w = synth.DecodeWorkload("decode_small", 1, 8, 2, 1000, 128, 128, tau)
    q = synth.make_decode_query(w, 9)
    k, v = synth.fill_decode_cache(w, 9, q, "cpu")
    q64, k64, v64 = parity.f64(q), parity.f64(k), parity.f64(v)
    G = 4
    nKB = -(-1000 // 128)
    O = np.zeros((1, 1, 8, 128))
    lse = np.zeros((1, 8))
    keep = np.zeros((1, 8, nKB), dtype=bool)
    for hk in range(2):
        Og, zg, kg, _ = orc.decode_group(q64[0, 0, hk * G:(hk + 1) * G], k64[0, :, hk], v64[0, :, hk], 128, tau, P)
        O[0, 0, hk * G:(hk + 1) * G] = Og
        lse[0, hk * G:(hk + 1) * G] = zg
        keep[0, hk * G:(hk + 1) * G] = kg
    return q, k, v, torch.from_numpy(O).to(torch.bfloat16), torch.from_numpy(lse).float(), keep


def test_group_decode_checker_accepts_and_rejects():
    q, k, v, o, lse, keep = _group_decode_case(5.0, 2)
    rep = parity.check_decode_group(q, k, v, o, lse, torch.from_numpy(mala.pack_mask(keep)), 5.0, 2)
    assert rep.heads == 8
    keep2 = keep.copy()
    keep2[0, 5, 0] = not keep2[0, 5, 0]
    with pytest.raises(AssertionError, match="different keep bits"):
        parity.check_decode_group(q, k, v, o, lse, torch.from_numpy(mala.pack_mask(keep2)), 5.0, 2)
    o2 = o.clone()
    o2[0, 0, 6, 40] += 0.25
    with pytest.raises(AssertionError, match="O"):
        parity.check_decode_group(q, k, v, o2, lse, torch.from_numpy(mala.pack_mask(keep)), 5.0, 2)
