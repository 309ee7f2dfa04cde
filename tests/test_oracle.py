"""Pins for the fp64 oracle, checked against things other than itself:

* the attention tutorial page's worked examples (tests/golden/),
* the tau -> 0 limit, which the MALA paper's cost paragraph says recovers
  FullAttn: dense masked softmax and its autograd gradient (torch, fp64),
* brute force on tiny inputs in the paper's *ratio* form (explicit retained
  key sets, plain exponentials) rather than the oracle's log form,
* invariants stated in the paper: m + log l = log Z over the retained set,
  the contribution ratio upper-bounds the dense probability, backward
  support nests inside forward support, the first legal tile is retained,
* closed forms: tau = inf keeps only the diagonal tile; decode with one split
  equals the causal forward of the last row; split merge at tau = 0 equals
  the dense softmax.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import mala_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, rest = line.partition(" ")
            rows[key] = rest
    return rows


def _nums(s):
    return [float(x) for x in s.split()]


def _rand_case(seed, N, d, H=1, sharp=2.0):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((N, d)) * sharp / math.sqrt(d)
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    return Q, K, V


def _dense_torch(Q, K, V):
    """Dense causal masked softmax attention in fp64 (the tutorial page's
    teaching reference, masked before the softmax)."""
    q = torch.tensor(Q, dtype=torch.float64, requires_grad=True)
    k = torch.tensor(K, dtype=torch.float64, requires_grad=True)
    v = torch.tensor(V, dtype=torch.float64, requires_grad=True)
    N = q.shape[0]
    s = q @ k.T
    allowed = torch.tril(torch.ones(N, N, dtype=torch.bool))
    s = s.masked_fill(~allowed, -float("inf"))
    w = torch.softmax(s, dim=-1)
    out = w @ v
    lse = torch.logsumexp(s, dim=-1)
    return q, k, v, out, lse, w


# ---------------------------------------------------------------- golden

def test_masked_row_worked_example():
    g = _read_golden("masked_row.txt")
    raw = _nums(g["raw_products"])
    dk = float(g["d_k"])
    scaled = _nums(g["scaled_scores"])
    qpos = int(g["query_position"])
    fut = int(g["future_keys"])
    assert np.allclose(np.array(raw) / math.sqrt(dk), scaled)
    # Q row qpos carries the scaled products against K = identity, V = identity
    N = 4
    Q = np.zeros((N, 4))
    Q[qpos] = scaled
    K = np.eye(4)
    V = np.eye(4)
    O, z, keep, _ = orc.forward_head(Q, K, V, 1, 1, 0.0)
    w = O[qpos]                                   # weights, since V = I
    assert w[fut] == 0.0                          # future key: exactly zero
    assert abs(w.sum() - 1.0) < 1e-15
    e = np.exp(np.array(scaled[:qpos + 1]))
    assert np.allclose(w[:qpos + 1], e / e.sum(), rtol=0, atol=1e-15)
    assert abs(z[qpos] - math.log(e.sum())) < 1e-14


def test_online_accumulator_worked_example():
    g = _read_golden("online_accumulator.txt")
    s = _nums(g["scores"])
    vals = np.array([_nums(t) for t in g["values"].split(";")])
    run_max = _nums(g["running_max"])
    # one query at position 3 sees all four keys; K = identity carries the
    # scores; one key per tile, visited in the page's order 0, 1, 2, 3
    q = np.array(s)[None, :]
    K = np.eye(4)
    seen = []
    st = orc.forward_block(q, np.array([3]), K, vals, 1, 0.0, [0, 1, 2, 3],
                           trace=lambda j, x: seen.append(x))
    assert [x["m"][0] for x in seen] == run_max
    # after tile 2 the first tile's weight is expressed relative to max 3
    assert abs(seen[1]["l"][0] - (math.exp(-3.0) + 1.0)) < 1e-15
    O, z = orc.finalize(st)
    e = np.exp(np.array(s))
    assert np.allclose(O[0], (e / e.sum()) @ vals, atol=1e-15)


# ---------------------------------------------------------------- tau -> 0

@pytest.mark.parametrize("N,d,Bq,Bk", [(37, 8, 8, 8), (33, 4, 4, 8), (40, 6, 16, 4), (17, 3, 1, 1)])
def test_tau_zero_is_dense_attention(N, d, Bq, Bk):
    Q, K, V = _rand_case(N * 7 + d, N, d, sharp=3.0)
    O, z, keep, margin = orc.forward_head(Q, K, V, Bq, Bk, 0.0)
    _, _, _, out, lse, _ = _dense_torch(Q, K, V)
    assert np.abs(O - out.detach().numpy()).max() < 1e-12
    assert np.abs(z - lse.detach().numpy()).max() < 1e-12
    # every legal tile retained
    for i in range(keep.shape[0]):
        last = min((i + 1) * Bq, N) - 1
        assert keep[i, : last // Bk + 1].all()
        assert not keep[i, last // Bk + 1:].any()


@pytest.mark.parametrize("N,d,Bq,Bk", [(23, 5, 4, 4), (30, 4, 8, 4), (19, 3, 4, 8)])
def test_tau_zero_backward_is_dense_gradient(N, d, Bq, Bk):
    Q, K, V = _rand_case(N * 3 + d, N, d, sharp=3.0)
    dO = np.random.default_rng(N).standard_normal((N, d))
    q, k, v, out, lse, _ = _dense_torch(Q, K, V)
    out.backward(torch.tensor(dO))
    O, z, keep, _ = orc.forward_head(Q, K, V, Bq, Bk, 0.0)
    dQ, dK, dV, bkeep, _ = orc.backward_head(Q, K, V, O, dO, z, Bq, Bk, 0.0, keep)
    assert np.abs(dQ - q.grad.numpy()).max() < 1e-11
    assert np.abs(dK - k.grad.numpy()).max() < 1e-11
    assert np.abs(dV - v.grad.numpy()).max() < 1e-11
    # pure (mask-free) backward gives the same at tau = 0
    dQ2, dK2, dV2, _, _ = orc.backward_head(Q, K, V, O, dO, z, Bq, Bk, 0.0, None)
    assert np.abs(dQ2 - dQ).max() < 1e-13 and np.abs(dK2 - dK).max() < 1e-13


def test_gqa_backward_sums_group():
    rng = np.random.default_rng(5)
    B, N, Hq, Hkv, d = 1, 12, 4, 2, 4
    q = rng.standard_normal((B, N, Hq, d))
    k = rng.standard_normal((B, N, Hkv, d))
    v = rng.standard_normal((B, N, Hkv, d))
    do = rng.standard_normal((B, N, Hq, d))
    O, lse, keep, _ = orc.forward(q, k, v, 4, 4, 0.0)
    dq, dk, dv, _ = orc.backward(q, k, v, O, do, lse, 4, 4, 0.0, keep)
    qt = torch.tensor(q, requires_grad=True)
    kt = torch.tensor(k, requires_grad=True)
    vt = torch.tensor(v, requires_grad=True)
    ke = kt.repeat_interleave(2, dim=2)
    ve = vt.repeat_interleave(2, dim=2)
    s = torch.einsum("bqhd,bkhd->bhqk", qt, ke)
    s = s.masked_fill(~torch.tril(torch.ones(N, N, dtype=torch.bool)), -float("inf"))
    out = torch.einsum("bhqk,bkhd->bqhd", torch.softmax(s, -1), ve)
    out.backward(torch.tensor(do))
    assert np.abs(O - out.detach().numpy()).max() < 1e-12
    assert np.abs(dq - qt.grad.numpy()).max() < 1e-11
    assert np.abs(dk - kt.grad.numpy()).max() < 1e-11
    assert np.abs(dv - vt.grad.numpy()).max() < 1e-11


# ---------------------------------------------------------------- brute force

def _brute_forward(Q, K, V, Bq, Bk, tau):
    """The paper's test in ratio form with explicit retained key sets:
    r_qj = max_{k in J_j, legal} exp(s_qk) / sum_{k in R_q} exp(s_qk);
    skip iff r < tau / L_q for every row with a legal key (empty R: keep).
    Query row q sits at position q + N_k - N_q (bottom-right alignment), sees
    keys k <= that position, and L_q = position + 1."""
    N, Nk = Q.shape[0], K.shape[0]
    off = Nk - N
    S = Q @ K.T
    nQB, nKB = -(-N // Bq), -(-Nk // Bk)
    keep = np.zeros((nQB, nKB), dtype=bool)
    O = np.zeros((N, V.shape[1]))
    for i in range(nQB):
        rows = list(range(i * Bq, min((i + 1) * Bq, N)))
        R = {q: [] for q in rows}
        for j in range(min((rows[-1] + off) // Bk, nKB - 1), -1, -1):
            cols = list(range(j * Bk, min((j + 1) * Bk, Nk)))
            retain = False
            for q in rows:
                legal = [k for k in cols if k <= q + off]
                if not legal:
                    continue
                if not R[q]:
                    retain = True
                    continue
                Z = sum(math.exp(S[q, k]) for k in R[q])
                r = max(math.exp(S[q, k]) for k in legal) / Z
                if not (r < tau / (q + off + 1)):
                    retain = True
            keep[i, j] = retain
            if retain:
                for q in rows:
                    R[q] += [k for k in cols if k <= q + off]
        for q in rows:
            w = np.array([math.exp(S[q, k]) for k in R[q]])
            O[q] = (w / w.sum()) @ V[R[q]]
    return keep, O


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("tau", [0.05, 0.3, 1.0, 4.0])
def test_forward_matches_brute_force(seed, tau):
    rng = np.random.default_rng(seed)
    N = int(rng.integers(9, 33))
    d = int(rng.integers(2, 9))
    Bq = int(rng.choice([1, 2, 4, 8]))
    Bk = int(rng.choice([1, 2, 4, 8]))
    Q, K, V = _rand_case(100 + seed, N, d, sharp=4.0)
    keep_b, O_b = _brute_forward(Q, K, V, Bq, Bk, tau)
    O, z, keep, margin = orc.forward_head(Q, K, V, Bq, Bk, tau)
    assert (keep == keep_b).all()
    assert np.abs(O - O_b).max() < 1e-12
    # decisions are not degenerate across the parametrisation
    visited = ~np.isnan(margin)
    assert visited.sum() >= keep.sum() > 0


def test_brute_force_sees_skips():
    """Make sure the brute-force comparison actually exercises skipping."""
    Q, K, V = _rand_case(7, 32, 8, sharp=6.0)
    keep, _ = _brute_forward(Q, K, V, 4, 4, 1.0)
    legal = sum(min((i * 4 + 3) // 4, 7) + 1 for i in range(8))
    assert 0 < keep.sum() < legal


def _brute_backward(Q, K, V, O, dO, z, Bq, Bk, tau, fwd_keep):
    """Dense (untiled) restatement of the backward: an entry contributes iff
    its tile was forward-retained and some legal entry of the tile has
    probability exp(s - z) >= tau / L_q."""
    N = Q.shape[0]
    S = Q @ K.T
    P = np.zeros((N, N))
    E = np.zeros((N, N), dtype=bool)
    for i in range(fwd_keep.shape[0]):
        for j in range(fwd_keep.shape[1]):
            if not fwd_keep[i, j]:
                continue
            rows = range(i * Bq, min((i + 1) * Bq, N))
            cols = range(j * Bk, min((j + 1) * Bk, N))
            ent = [(q, k) for q in rows for k in cols if k <= q]
            if not ent:
                continue
            if any(math.exp(S[q, k] - z[q]) >= tau / (q + 1) for (q, k) in ent):
                for (q, k) in ent:
                    E[q, k] = True
    P[E] = np.exp(S - z[:, None])[E]
    D = (dO * O).sum(1)
    dV = P.T @ dO
    dP = dO @ V.T
    dS = np.where(E, P * (dP - D[:, None]), 0.0)
    return dS @ K, dS.T @ Q, dV


@pytest.mark.parametrize("seed", range(5))
@pytest.mark.parametrize("tau", [0.1, 1.0])
def test_backward_matches_brute_force(seed, tau):
    rng = np.random.default_rng(50 + seed)
    N = int(rng.integers(9, 29))
    d = int(rng.integers(2, 7))
    Bq = int(rng.choice([2, 4, 8]))
    Bk = int(rng.choice([2, 4, 8]))
    Q, K, V = _rand_case(200 + seed, N, d, sharp=4.0)
    dO = rng.standard_normal((N, d))
    O, z, keep, _ = orc.forward_head(Q, K, V, Bq, Bk, tau)
    dQ, dK, dV, bkeep, _ = orc.backward_head(Q, K, V, O, dO, z, Bq, Bk, tau, keep)
    bq, bk, bv = _brute_backward(Q, K, V, O, dO, z, Bq, Bk, tau, keep)
    assert np.abs(dQ - bq).max() < 1e-12
    assert np.abs(dK - bk).max() < 1e-12
    assert np.abs(dV - bv).max() < 1e-12


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("tau", [0.02, 0.5, 2.0])
def test_lse_invariant_and_ratio_bound(tau):
    """m + log l = log Z over the retained set after every tile, and the
    contribution ratio upper-bounds the dense probability of the tile."""
    N, d, B = 48, 8, 8
    Q, K, V = _rand_case(11, N, d, sharp=5.0)
    S = Q @ K.T
    lse_dense = np.array([np.log(np.exp(S[q, :q + 1]).sum()) for q in range(N)])
    for i in range(N // B):
        rows = np.arange(i * B, (i + 1) * B)
        retained = {int(q): [] for q in rows}
        prev = {}

        def check(j, st):
            cols = np.arange(j * B, (j + 1) * B)
            for r, q in enumerate(rows):
                legal = cols[cols <= q]
                if len(legal) == 0:
                    continue
                # the ratio bound uses the state *before* this tile's update
                if q in prev and prev[q][1] > 0:
                    m0, l0 = prev[q]
                    ratio = math.exp(S[q, legal].max() - m0) / l0
                    p_dense = math.exp(S[q, legal].max() - lse_dense[q])
                    assert ratio >= p_dense * (1 - 1e-12)
                if st["keep"]:
                    retained[int(q)] += list(legal)
                if retained[int(q)]:
                    logZ = np.log(np.exp(S[q, retained[int(q)]]).sum())
                    assert abs(st["m"][r] + math.log(st["l"][r]) - logZ) < 1e-12
                prev[q] = (st["m"][r], st["l"][r])

        orc.forward_block(Q[rows], rows, K, V, B, tau,
                          orc.causal_tiles(rows[-1], B, N // B), trace=check)


@pytest.mark.parametrize("seed", range(4))
def test_backward_support_nests_in_forward(seed):
    Q, K, V = _rand_case(300 + seed, 64, 8, sharp=5.0)
    dO = np.random.default_rng(seed).standard_normal((64, 8))
    for tau in (0.05, 0.5, 2.0):
        O, z, keep, _ = orc.forward_head(Q, K, V, 8, 8, tau)
        _, _, _, pure_keep, pure_margin = orc.backward_head(Q, K, V, O, dO, z, 8, 8, tau, None)
        bad = pure_keep & ~keep
        assert not bad.any() or np.abs(pure_margin[bad]).max() < 1e-9


def test_first_legal_tile_always_retained():
    Q, K, V = _rand_case(9, 40, 4, sharp=8.0)
    for tau in (0.5, 5.0, 1e6):
        _, _, keep, _ = orc.forward_head(Q, K, V, 8, 8, tau)
        for i in range(5):
            assert keep[i, i]


def test_tau_infinite_keeps_only_diagonal():
    N, d, B = 32, 4, 8
    Q, K, V = _rand_case(21, N, d, sharp=2.0)
    O, z, keep, _ = orc.forward_head(Q, K, V, B, B, math.inf)
    assert (keep == np.eye(N // B, dtype=bool)).all()
    S = Q @ K.T
    for q in range(N):
        k0 = (q // B) * B
        w = np.exp(S[q, k0:q + 1] - S[q, k0:q + 1].max())
        assert np.allclose(O[q], (w / w.sum()) @ V[k0:q + 1], atol=1e-13)
    dO = np.ones((N, d))
    dQ, dK, dV, bkeep, _ = orc.backward_head(Q, K, V, O, dO, z, B, B, math.inf, keep)
    assert not bkeep.any() and not dQ.any() and not dK.any() and not dV.any()


def test_sharper_tau_skips_more_and_omits_more_mass():
    Q, K, V = _rand_case(31, 64, 8, sharp=4.0)
    _, z0, k0, _ = orc.forward_head(Q, K, V, 8, 8, 0.0)
    prev_kept, prev_mass = k0.sum(), 0.0
    for tau in (0.01, 0.1, 1.0):
        _, z, kp, _ = orc.forward_head(Q, K, V, 8, 8, tau)
        omitted = 1.0 - np.exp(z - z0)          # paper's omitted-mass metric
        assert (omitted >= -1e-12).all()
        assert kp.sum() <= prev_kept
        prev_kept = kp.sum()


# ---------------------------------------------------------------- decode

def test_decode_single_split_equals_last_causal_row():
    rng = np.random.default_rng(3)
    N, d, Bk = 8 * 5 + 1, 6, 8                     # last query block holds one row
    Q = rng.standard_normal((N, d)) * 3 / math.sqrt(d)
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    for tau in (0.0, 0.1, 1.0):
        O, z, keep, margin = orc.forward_head(Q, K, V, 8, Bk, tau)
        Od, zd, kd, md, _ = orc.decode_head(Q[-1], K, V, Bk, tau, 1)
        assert np.allclose(Od, O[-1], atol=1e-14) and abs(zd - z[-1]) < 1e-14
        assert (kd == keep[-1]).all()


@pytest.mark.parametrize("P", [1, 2, 3, 7])
def test_decode_splits_at_tau_zero_are_dense(P):
    rng = np.random.default_rng(P)
    N, d, Bk = 61, 5, 8
    q = rng.standard_normal(d)
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    O, z, keep, _, parts = orc.decode_head(q, K, V, Bk, 0.0, P)
    s = K @ q
    w = np.exp(s - s.max())
    assert np.allclose(O, (w / w.sum()) @ V, atol=1e-13)
    assert abs(z - (s.max() + math.log(w.sum()))) < 1e-13
    assert keep.all() and len(parts) == P


def test_decode_first_tile_of_each_split_retained():
    rng = np.random.default_rng(4)
    N, d, Bk, P = 128, 4, 8, 4
    q = rng.standard_normal(d) * 4
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    _, _, keep, _, _ = orc.decode_head(q, K, V, Bk, math.inf, P)
    for (t0, t1) in orc.split_ranges(N // Bk, P):
        assert keep[t1 - 1]
        assert not keep[t0:t1 - 1].any()
    assert orc.split_ranges(10, 3) == [(0, 3), (3, 6), (6, 10)]


def _brute_decode_row(q, K, V, Bk, tau, P):
    """One decoding query in ratio form with explicit retained key sets, per
    split: walking a split's tiles from the last, a tile is retained iff the
    split's retained set is empty or some key of the tile has
    exp(s) / sum over retained keys of exp(s) >= tau / N_k. Each split's
    partial is plain softmax attention over its retained keys; the split
    results combine as sum_p Z_p O_p / sum_p Z_p (Z_p = sum of exp(s) over
    split p's retained keys). Returns O, log sum_p Z_p, keep."""
    N = K.shape[0]
    s = K @ q
    nKB = -(-N // Bk)
    keep = np.zeros(nKB, dtype=bool)
    num = np.zeros(V.shape[1])
    den = 0.0
    for (t0, t1) in orc.split_ranges(nKB, P):
        kept_keys = []
        for j in range(t1 - 1, t0 - 1, -1):
            keys = list(range(j * Bk, min((j + 1) * Bk, N)))
            if kept_keys:
                ratio = math.exp(max(s[keys])) / sum(math.exp(s[k]) for k in kept_keys)
                keep[j] = not (ratio < tau / N)
            else:
                keep[j] = True
            if keep[j]:
                kept_keys += keys
        w = np.array([math.exp(s[k]) for k in kept_keys])
        num += w @ V[kept_keys]
        den += w.sum()
    return num / den, math.log(den), keep


@pytest.mark.parametrize("P,tau", [(1, 0.0), (2, 0.5), (3, 4.0)])
def test_decode_batched_gqa_head_mapping(P, tau):
    """oracle.decode over [B, 1, H_q, d] queries and a [B, N_k, H_kv, d]
    cache: query head h of batch b reads KV head h // (H_q / H_kv) of the same
    batch. Every (b, h) is checked against the brute-force ratio form run on
    that KV head's rows; at tau = 0 also against torch's dense softmax with
    the KV heads repeated G times along the head axis (the usual GQA
    expansion). The cache's KV heads and batches differ, so a transposed
    head map or batch index fails."""
    rng = np.random.default_rng(200 + P)
    B, Hq, Hkv, N, d, Bk = 2, 8, 2, 45, 6, 8
    G = Hq // Hkv
    q = rng.standard_normal((B, 1, Hq, d)) * 4 / math.sqrt(d)
    k = rng.standard_normal((B, N, Hkv, d))
    v = rng.standard_normal((B, N, Hkv, d))
    O, lse, keep, _ = orc.decode(q, k, v, Bk, tau, P)
    for b in range(B):
        for h in range(Hq):
            Ob, zb, kb = _brute_decode_row(q[b, 0, h], k[b, :, h // G], v[b, :, h // G], Bk, tau, P)
            assert (keep[b, h] == kb).all(), (b, h)
            assert np.allclose(O[b, 0, h], Ob, atol=1e-12), (b, h)
            assert abs(lse[b, h] - zb) < 1e-12, (b, h)
            # another KV head gives other values: the map is observable here
            Ow, _, _ = _brute_decode_row(q[b, 0, h], k[b, :, 1 - h // G], v[b, :, 1 - h // G], Bk, tau, P)
            assert not np.allclose(O[b, 0, h], Ow, atol=1e-6)
    if tau == 0.0:
        qt = torch.tensor(q)
        ke = torch.tensor(k).repeat_interleave(G, dim=2)
        ve = torch.tensor(v).repeat_interleave(G, dim=2)
        s = torch.einsum("bqhd,bkhd->bhqk", qt, ke)
        out = torch.einsum("bhqk,bkhd->bqhd", torch.softmax(s, -1), ve)
        assert np.abs(O - out.numpy()).max() < 1e-12
        assert np.abs(lse - torch.logsumexp(s, -1)[:, :, 0].numpy()).max() < 1e-12
    else:
        assert not keep.all()                        # the case skips tiles


def _group_case(seed, G, N, d, sharp=3.0):
    rng = np.random.default_rng(seed)
    Qg = rng.standard_normal((G, d)) * sharp / math.sqrt(d)
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    return Qg, K, V


@pytest.mark.parametrize("P", [1, 3])
def test_decode_group_of_one_is_per_head_decode(P):
    Qg, K, V = _group_case(50 + P, 1, 77, 6)
    for tau in (0.05, 0.5, 4.0):
        O, z, keep, margin = orc.decode_group(Qg, K, V, 8, tau, P)
        Oh, zh, kh, mh, _ = orc.decode_head(Qg[0], K, V, 8, tau, P)
        assert (keep == kh).all()
        assert np.allclose(O[0], Oh, atol=1e-14) and abs(z[0] - zh) < 1e-14


def test_decode_group_of_identical_heads_is_per_head_decode():
    Qg, K, V = _group_case(60, 1, 90, 5)
    Qg = np.repeat(Qg, 4, axis=0)
    O, z, keep, _ = orc.decode_group(Qg, K, V, 8, 0.5, 2)
    Oh, zh, kh, _, _ = orc.decode_head(Qg[0], K, V, 8, 0.5, 2)
    assert (keep == kh).all()
    for g in range(4):
        assert np.allclose(O[g], Oh, atol=1e-14) and abs(z[g] - zh) < 1e-14


@pytest.mark.parametrize("P", [1, 2, 5])
def test_decode_group_at_tau_zero_is_dense(P):
    Qg, K, V = _group_case(70 + P, 4, 61, 5)
    O, z, keep, _ = orc.decode_group(Qg, K, V, 8, 0.0, P)
    assert keep.all()
    for g in range(4):
        s = K @ Qg[g]
        w = np.exp(s - s.max())
        assert np.allclose(O[g], (w / w.sum()) @ V, atol=1e-13)
        assert abs(z[g] - (s.max() + math.log(w.sum()))) < 1e-13


@pytest.mark.parametrize("seed,P,tau", [(80, 1, 0.3), (81, 2, 1.0), (82, 3, 3.0), (83, 1, 20.0)])
def test_decode_group_brute_force(seed, P, tau):
    """The joint decisions re-derived from their definition, in ratio form with
    explicit retained key sets: within a split, walking its tiles from the
    last, a tile is retained iff the retained set is still empty or some head
    has a key in the tile with exp(s) / sum over retained keys of exp(s) >=
    tau / N_k. Every head's output is then plain softmax attention over the
    keys of all retained tiles."""
    G, N, d, Bk = 4, 70, 4, 8
    Qg, K, V = _group_case(seed, G, N, d, sharp=6.0)
    O, z, keep, _ = orc.decode_group(Qg, K, V, Bk, tau, P)
    S = Qg @ K.T                                     # [G, N]
    nKB = -(-N // Bk)
    want = np.zeros(nKB, dtype=bool)
    for (t0, t1) in orc.split_ranges(nKB, P):
        kept_keys = []
        for j in range(t1 - 1, t0 - 1, -1):
            keys = list(range(j * Bk, min((j + 1) * Bk, N)))
            if not kept_keys:
                want[j] = True
            else:
                mass = np.exp(S[:, kept_keys]).sum(axis=1)          # [G]
                ratio = np.exp(S[:, keys]).max(axis=1) / mass
                want[j] = bool((ratio >= tau / N).any())
            if want[j]:
                kept_keys += keys
    assert (keep == want).all()
    if tau >= 3.0:
        assert keep.sum() < nKB                      # the case does skip
    cols = np.concatenate([np.arange(j * Bk, min((j + 1) * Bk, N)) for j in range(nKB) if want[j]])
    for g in range(G):
        w = np.exp(S[g, cols])
        assert np.allclose(O[g], (w / w.sum()) @ V[cols], atol=1e-12)
        assert abs(z[g] - math.log(w.sum())) < 1e-12


def test_decode_group_retains_a_tile_one_head_needs():
    """A tile that only one head of the group needs is retained for all heads;
    per-head decode would read it for that head alone."""
    G, N, d, Bk = 3, 64, 4, 8
    rng = np.random.default_rng(90)
    K = rng.standard_normal((N, d)) * 0.1
    V = rng.standard_normal((N, d))
    Qg = np.zeros((G, d))
    Qg[:, 0] = 1.0
    K[5, 1] = 40.0                                   # a key only head 2 scores highly
    Qg[2, 1] = 1.0
    O, z, keep, _ = orc.decode_group(Qg, K, V, Bk, 2.0, 1)
    _, z0, k0, _, _ = orc.decode_head(Qg[0], K, V, Bk, 2.0, 1)
    _, _, k2, _, _ = orc.decode_head(Qg[2], K, V, Bk, 2.0, 1)
    assert k2[0] and not k0[0] and keep[0]
    assert (keep >= k0).all()
    assert z[0] > z0                                 # head 0 now also holds tile 0's mass


@pytest.mark.parametrize("Nq,Nk", [(40, 40), (29, 45)])
def test_forward_group_of_one_is_forward_head(Nq, Nk):
    rng = np.random.default_rng(100 + Nq)
    Q = rng.standard_normal((1, Nq, 5)) * 4 / math.sqrt(5)
    K = rng.standard_normal((Nk, 5))
    V = rng.standard_normal((Nk, 5))
    for tau in (0.1, 1.0, 10.0):
        O, z, keep, margin = orc.forward_group(Q, K, V, 8, 8, tau)
        Oh, zh, kh, mh = orc.forward_head(Q[0], K, V, 8, 8, tau)
        assert (keep == kh).all()
        assert np.allclose(O[0], Oh, atol=1e-14) and np.allclose(z[0], zh, atol=1e-14)


def test_forward_group_of_identical_heads_is_forward_head():
    rng = np.random.default_rng(110)
    Q1 = rng.standard_normal((37, 4)) * 4 / 2
    K = rng.standard_normal((37, 4))
    V = rng.standard_normal((37, 4))
    O, z, keep, _ = orc.forward_group(np.stack([Q1] * 3), K, V, 8, 8, 1.0)
    Oh, zh, kh, _ = orc.forward_head(Q1, K, V, 8, 8, 1.0)
    assert (keep == kh).all()
    for g in range(3):
        assert np.allclose(O[g], Oh, atol=1e-14) and np.allclose(z[g], zh, atol=1e-14)


def test_forward_group_at_tau_zero_is_dense():
    rng = np.random.default_rng(120)
    G, N, d = 3, 33, 4
    Qg = rng.standard_normal((G, N, d)) * 2
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    O, z, keep, _ = orc.forward_group(Qg, K, V, 8, 8, 0.0)
    for g in range(G):
        _, _, _, Od, zd, _ = _dense_torch(Qg[g], K, V)
        assert np.allclose(O[g], Od.detach().numpy(), atol=1e-12)
        assert np.allclose(z[g], zd.detach().numpy(), atol=1e-12)


@pytest.mark.parametrize("seed,tau,Nq", [(130, 0.5, 48), (131, 300.0, 48), (132, 300.0, 41)])
def test_forward_group_brute_force(seed, tau, Nq):
    """Joint decisions from their definition in ratio form, with explicit
    retained key sets per row: a tile is retained iff some row of some head
    with a legal key in it has an empty retained set or a key whose
    exp(s) / sum over its retained keys of exp(s) is >= tau / L_q; every row's
    output is softmax attention over its legal keys in the retained tiles."""
    G, Nk, d, B = 3, 48, 4, 8
    rng = np.random.default_rng(seed)
    Qg = rng.standard_normal((G, Nq, d)) * 5 / 2
    K = rng.standard_normal((Nk, d))
    V = rng.standard_normal((Nk, d))
    O, z, keep, _ = orc.forward_group(Qg, K, V, B, B, tau)
    off = Nk - Nq
    nQB, nKB = -(-Nq // B), -(-Nk // B)
    skipped = 0
    for i in range(nQB):
        rows = range(i * B, min((i + 1) * B, Nq))
        j_diag = (rows[-1] + off) // B
        kept_tiles = []
        for j in range(j_diag, -1, -1):
            want = False
            for g in range(G):
                for r in rows:
                    p = r + off
                    legal = [k for k in range(j * B, min((j + 1) * B, Nk)) if k <= p]
                    if not legal:
                        continue
                    mine = [k for t in kept_tiles for k in range(t * B, min((t + 1) * B, Nk)) if k <= p]
                    if not mine:
                        want = True
                        continue
                    mass = sum(math.exp(Qg[g, r] @ K[k]) for k in mine)
                    best = max(math.exp(Qg[g, r] @ K[k]) for k in legal)
                    if best / mass >= tau / (p + 1):
                        want = True
            assert keep[i, j] == want, (i, j)
            if want:
                kept_tiles.append(j)
            else:
                skipped += 1
        for g in range(G):
            for r in rows:
                p = r + off
                ks = [k for t in kept_tiles for k in range(t * B, min((t + 1) * B, Nk)) if k <= p]
                w = np.array([math.exp(Qg[g, r] @ K[k]) for k in ks])
                assert np.allclose(O[g, r], (w / w.sum()) @ V[ks], atol=1e-11)
                assert abs(z[g, r] - math.log(w.sum())) < 1e-11
    if tau >= 100.0:
        assert skipped > 0                           # the case does skip


def test_replay_forces_decisions_but_keeps_margins():
    Q, K, V = _rand_case(41, 32, 4, sharp=5.0)
    O, z, keep, margin = orc.forward_head(Q, K, V, 8, 8, 0.5)
    O2, z2, keep2, margin2 = orc.forward_head(Q, K, V, 8, 8, 0.5, replay_mask=keep)
    assert (keep2 == keep).all() and np.allclose(O2, O) and np.allclose(margin2, margin, equal_nan=True)
    flipped = keep.copy()
    flipped[3, 1] = not flipped[3, 1]
    _, _, keep3, _ = orc.forward_head(Q, K, V, 8, 8, 0.5, replay_mask=flipped)
    assert keep3[3, 1] == flipped[3, 1]


# ------------------------------------------- bottom-right causal alignment
# A chunk of N_q queries at the end of an N_k-key context: query q is at
# position q + N_k - N_q ("Setup": C_q are the keys up to the query's
# position, L_q = |C_q|; N_q = 1 is the decoding case L_0 = N_k).

def _dense_bottom_right(Q, K, V):
    q = torch.tensor(Q, dtype=torch.float64, requires_grad=True)
    k = torch.tensor(K, dtype=torch.float64, requires_grad=True)
    v = torch.tensor(V, dtype=torch.float64, requires_grad=True)
    Nq, Nk = q.shape[0], k.shape[0]
    allowed = torch.arange(Nk)[None, :] <= (torch.arange(Nq)[:, None] + (Nk - Nq))
    s = (q @ k.T).masked_fill(~allowed, -float("inf"))
    out = torch.softmax(s, dim=-1) @ v
    return q, k, v, out, torch.logsumexp(s, dim=-1)


@pytest.mark.parametrize("Nq,Nk,d,Bq,Bk", [(13, 37, 5, 4, 8), (20, 21, 4, 8, 4), (9, 40, 3, 4, 4), (1, 29, 6, 8, 8)])
def test_bottom_right_tau_zero_is_dense(Nq, Nk, d, Bq, Bk):
    rng = np.random.default_rng(Nq * 31 + Nk)
    Q = rng.standard_normal((Nq, d)) * 3 / math.sqrt(d)
    K = rng.standard_normal((Nk, d))
    V = rng.standard_normal((Nk, d))
    dO = rng.standard_normal((Nq, d))
    q, k, v, out, lse = _dense_bottom_right(Q, K, V)
    out.backward(torch.tensor(dO))
    O, z, keep, _ = orc.forward_head(Q, K, V, Bq, Bk, 0.0)
    assert np.abs(O - out.detach().numpy()).max() < 1e-12
    assert np.abs(z - lse.detach().numpy()).max() < 1e-12
    dQ, dK, dV, _, _ = orc.backward_head(Q, K, V, O, dO, z, Bq, Bk, 0.0, keep)
    assert np.abs(dQ - q.grad.numpy()).max() < 1e-11
    assert np.abs(dK - k.grad.numpy()).max() < 1e-11
    assert np.abs(dV - v.grad.numpy()).max() < 1e-11


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("tau", [0.05, 0.5, 2.0])
def test_bottom_right_matches_brute_force(seed, tau):
    rng = np.random.default_rng(500 + seed)
    Nk = int(rng.integers(12, 33))
    Nq = int(rng.integers(1, Nk + 1))
    d = int(rng.integers(2, 7))
    Bq = int(rng.choice([1, 2, 4, 8]))
    Bk = int(rng.choice([1, 2, 4, 8]))
    Q = rng.standard_normal((Nq, d)) * 4 / math.sqrt(d)
    K = rng.standard_normal((Nk, d))
    V = rng.standard_normal((Nk, d))
    keep_b, O_b = _brute_forward(Q, K, V, Bq, Bk, tau)
    O, z, keep, _ = orc.forward_head(Q, K, V, Bq, Bk, tau)
    assert (keep == keep_b).all()
    assert np.abs(O - O_b).max() < 1e-12


@pytest.mark.parametrize("tau", [0.1, 1.0])
def test_bottom_right_aligned_chunk_is_the_last_rows_of_the_full_problem(tau):
    """With an offset that is a multiple of both block sizes, the chunk's
    query blocks are the full problem's last query blocks: same decisions,
    outputs and, with dO zero on the other rows, the same gradients."""
    rng = np.random.default_rng(77)
    Nk, off, d, B = 48, 16, 5, 8
    Q = rng.standard_normal((Nk, d)) * 5 / math.sqrt(d)
    K = rng.standard_normal((Nk, d))
    V = rng.standard_normal((Nk, d))
    dO = rng.standard_normal((Nk, d))
    dO[:off] = 0.0
    O_f, z_f, keep_f, _ = orc.forward_head(Q, K, V, B, B, tau)
    O_c, z_c, keep_c, _ = orc.forward_head(Q[off:], K, V, B, B, tau)
    assert np.abs(O_c - O_f[off:]).max() < 1e-12 and np.abs(z_c - z_f[off:]).max() < 1e-12
    assert (keep_c == keep_f[off // B:]).all()
    assert keep_c.sum() < keep_c.size             # the case exercises skipping
    dQ_f, dK_f, dV_f, bk_f, _ = orc.backward_head(Q, K, V, O_f, dO, z_f, B, B, tau, keep_f)
    dQ_c, dK_c, dV_c, bk_c, _ = orc.backward_head(Q[off:], K, V, O_c, dO[off:], z_c, B, B, tau, keep_c)
    assert np.abs(dQ_c - dQ_f[off:]).max() < 1e-12
    assert np.abs(dK_c - dK_f).max() < 1e-12 and np.abs(dV_c - dV_f).max() < 1e-12
    assert (bk_c == bk_f[off // B:]).all()


def test_bottom_right_single_query_is_decoding():
    rng = np.random.default_rng(9)
    Nk, d, Bk = 45, 6, 8
    Q = rng.standard_normal((1, d)) * 3 / math.sqrt(d)
    K = rng.standard_normal((Nk, d))
    V = rng.standard_normal((Nk, d))
    for tau in (0.0, 0.2, 1.5):
        O, z, keep, _ = orc.forward_head(Q, K, V, 4, Bk, tau)
        Od, zd, kd, _, _ = orc.decode_head(Q[0], K, V, Bk, tau, 1)
        assert np.allclose(Od, O[0], atol=1e-14) and abs(zd - z[0]) < 1e-14
        assert (kd == keep[0]).all()
