"""fp64 CPU oracle for MassAlloc Attention (MALA).

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this module:
only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it. It shares no code with the CUDA path.

Source: "MassAlloc Attention: Let Attention Allocate Its Own Compute"
(signal-papers page 2609.32712). Section names below are the run-in headings
of that page's method text:

* "Setup"                         - notation, tiles I_i / J_j, L_q, tau / L_q
* "Online Sparse Softmax"         - Algorithm 1, the forward skip test
* "Offline Sparse Probability"    - Algorithm 2, the backward skip test
* cost paragraph after it         - tau -> 0 recovers FullAttn, split-KV decode
* Appendix A.1 "Fused forward / backward / decoding execution" - traversal
  orders (forward: key blocks descending from the diagonal; backward:
  key-major, query blocks ascending from the diagonal; decode: per-split
  normalizers, standard normalizer-aware merge)

The page's display equations and algorithm listings were lost when it was
extracted, so each test is restated from the surrounding prose:

* forward (Online Sparse Softmax): a tile is skipped only when, for every
  valid query row q with at least one legal key in the tile,
      max_k s_qk - (m_q + log l_q) < log tau - log L_q
  A row whose retained set is still empty (l_q = 0) has log-ratio +inf and
  therefore retains the tile. Rows with no legal key do not constrain.
  Retained tiles take the standard online-softmax update; skipped tiles
  leave m, l, O unchanged. At the end z_q = m_q + log l_q.
* backward (Offline Sparse Probability): key-major tile S_ji = K_j Q_i^T; the
  tile is skipped only when s_qk - z_q < log tau - log L_q holds for every
  legal (k, q) entry. Retained tiles run P = exp(S - z), dV += P^T dO,
  dP = dO V^T, dS = P * (dP - D) with D_q = sum_d dO_q O_q, dQ += dS K,
  dK += dS^T Q.
* decode: L_0 = N_k (the current token included); split p covers key tiles
  [floor(p T / P), floor((p+1) T / P)) of the T tiles, visited descending,
  with its own (m, l); partial outputs merge by their log-normalizers.
* group-joint decode and prefill (the pages only say that every valid row
  of a query block must pass for a tile to be skipped): the query heads of a
  GQA group are taken as the rows of one block (decode: the heads' single
  rows; prefill: the heads' rows of the same query block), so the group
  takes one decision per tile and every head accumulates the retained tiles.

Readings taken where the page is silent (each also listed in the design
notes): skip is the strict "<" so a tie retains; tau = 0 means log tau = -inf
(nothing is skipped); the "margin" of a tile is the smallest per-row slack
  (log tau - log L_q) - (max_k s_qk - m_q - log l_q)   (forward)
  (log tau - log L_q) - (s_qk - z_q), minimised over legal entries (backward)
so that a tile is retained iff margin <= 0.

Every function here is pinned in tests/test_oracle.py against values the
pages print, closed forms and brute force; none is "parity unpinned".
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence

import numpy as np

NEG_INF = -math.inf


def _log(x: float) -> float:
    """Natural log with log(0) = -inf and log(inf) = inf, no warnings."""
    if x == 0.0:
        return NEG_INF
    return math.log(x)


def num_blocks(n: int, b: int) -> int:
    return (n + b - 1) // b


# --------------------------------------------------------------------------
# Algorithm 1 on one query block ("Online Sparse Softmax")
# --------------------------------------------------------------------------

def forward_block(Q_i: np.ndarray, pos_i: np.ndarray, K: np.ndarray,
                  V: np.ndarray, B_k: int, tau: float,
                  tiles: Sequence[int], L_i: Optional[np.ndarray] = None,
                  replay: Optional[dict] = None, trace=None):
    """Run the forward traversal of one query block over ``tiles``.

    Q_i   [R, d]  query rows of block I_i (valid rows only), scale folded in
    pos_i [R]     zero-based positions of those rows; key k is legal for row
                  q iff k <= pos_i[q] (causal visibility C_q)
    K, V  [N_k, d]
    tiles         key-block indices J_j in visiting order
    L_i   [R]     |C_q| per row; defaults to pos + 1 (equal-length training)
    replay        optional {j: bool} forcing the keep decision of tile j
                  (the margin is still evaluated at the current state)
    trace         optional callable(j, state) for invariant checks

    Returns dict with m, l (running state), acc (un-normalised output),
    keep {j: bool}, margin {j: float}.
    """
    Q_i = np.asarray(Q_i, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    R, d = Q_i.shape
    N_k = K.shape[0]
    pos_i = np.asarray(pos_i, dtype=np.int64)
    if L_i is None:
        L_i = pos_i + 1
    log_thr = np.array([_log(tau) - math.log(float(L)) for L in L_i])  # log tau - log L_q

    m = np.full(R, NEG_INF)          # running row maximum m_i
    l = np.zeros(R)                  # shifted normalisation sum l_i
    acc = np.zeros((R, V.shape[1]))  # output accumulator O_i (un-normalised)
    keep, margin = {}, {}

    for j in tiles:
        k0, k1 = j * B_k, min((j + 1) * B_k, N_k)
        keys = np.arange(k0, k1)
        # score discovery: S_ij = Q_i K_j^T over every legal entry
        S = Q_i @ K[k0:k1].T
        legal = keys[None, :] <= pos_i[:, None]
        S = np.where(legal, S, NEG_INF)
        has_key = legal.any(axis=1)          # rows that constrain this tile

        # per-row slack of the skip test; rows without a legal key do not
        # constrain (+inf), rows with an empty retained set force retention
        rmax = np.where(has_key, S.max(axis=1), NEG_INF)
        with np.errstate(divide="ignore", invalid="ignore"):
            log_ratio = rmax - (m + np.log(l))
            row_margin = np.where(has_key, np.where(l > 0.0, log_thr - log_ratio, NEG_INF), math.inf)
        M = float(row_margin.min()) if R else math.inf
        margin[j] = M
        decide = (M <= 0.0)                  # skip iff every row is strictly below
        if replay is not None and j in replay:
            decide = bool(replay[j])
        keep[j] = decide

        if decide:
            # standard online-softmax update of the rows with a legal key
            rows = np.nonzero(has_key)[0]
            m_new = np.maximum(m[rows], rmax[rows])
            p = np.exp(S[rows] - m_new[:, None])            # exp(-inf) = 0 on illegal keys
            alpha = np.where(l[rows] > 0.0, np.exp(m[rows] - m_new), 0.0)
            l[rows] = l[rows] * alpha + p.sum(axis=1)
            acc[rows] = acc[rows] * alpha[:, None] + p @ V[k0:k1]
            m[rows] = m_new
        if trace is not None:
            trace(j, dict(m=m.copy(), l=l.copy(), keep=decide, S=S, margin=M))

    return dict(m=m, l=l, acc=acc, keep=keep, margin=margin)


def finalize(state):
    """O = acc / l and z = m + log l (the final log-normaliser)."""
    l = state["l"]
    with np.errstate(divide="ignore", invalid="ignore"):
        O = state["acc"] / l[:, None]
        z = state["m"] + np.log(l)
    return O, z


def causal_tiles(pos_last: int, B_k: int, n_kblocks: int) -> list:
    """Key blocks of a query block, descending from its diagonal block."""
    j_diag = min(pos_last // B_k, n_kblocks - 1)
    return list(range(j_diag, -1, -1))


def forward_head(Q: np.ndarray, K: np.ndarray, V: np.ndarray, B_q: int,
                 B_k: int, tau: float, replay_mask: Optional[np.ndarray] = None,
                 blocks: Optional[Iterable[int]] = None):
    """Algorithm 1 for one (batch, query-head) pair, causal.

    N_q <= N_k with bottom-right alignment: query q sits at position
    q + N_k - N_q, sees keys k <= that position, and L_q = position + 1
    (N_q = N_k is the training case L_q = q + 1; N_q = 1 is single-token
    decoding with L_0 = N_k, "Setup"). Query blocks are formed from the
    first query row.

    Returns O [N_q, d], z [N_q], keep [nQB, nKB] bool, margin [nQB, nKB]
    (NaN where a tile is never visited). ``blocks`` restricts the query
    blocks computed (rows of other blocks are left NaN).
    """
    N_q, d = Q.shape
    N_k = K.shape[0]
    assert N_q <= N_k, "causal mode needs N_q <= N_k (bottom-right alignment)"
    off = N_k - N_q
    nQB, nKB = num_blocks(N_q, B_q), num_blocks(N_k, B_k)
    O = np.full((N_q, V.shape[1]), np.nan)
    z = np.full(N_q, np.nan)
    keep = np.zeros((nQB, nKB), dtype=bool)
    margin = np.full((nQB, nKB), np.nan)
    for i in (range(nQB) if blocks is None else blocks):
        q0, q1 = i * B_q, min((i + 1) * B_q, N_q)
        pos = np.arange(q0, q1) + off
        tiles = causal_tiles(q1 - 1 + off, B_k, nKB)
        rep = None
        if replay_mask is not None:
            rep = {j: bool(replay_mask[i, j]) for j in tiles}
        st = forward_block(Q[q0:q1], pos, K, V, B_k, tau, tiles, replay=rep)
        O[q0:q1], z[q0:q1] = finalize(st)
        for j in tiles:
            keep[i, j] = st["keep"][j]
            margin[i, j] = st["margin"][j]
    return O, z, keep, margin


def forward_group(Qg: np.ndarray, K: np.ndarray, V: np.ndarray, B_q: int,
                  B_k: int, tau: float, replay_mask: Optional[np.ndarray] = None,
                  blocks: Optional[Iterable[int]] = None):
    """Group-joint prefill: the G query heads that share one KV head take one
    decision per (query block, key tile). For query block i the G heads'
    rows are taken together as the rows of one block under the test of
    "Online Sparse Softmax" (skipped only when every row of every head
    passes; a retained tile updates every head). Causal, N_q <= N_k,
    bottom-right aligned as in ``forward_head``.

    Qg [G, N_q, d]. Returns O [G, N_q, d], z [G, N_q], keep [nQB, nKB] bool,
    margin [nQB, nKB] (NaN where a tile is never visited)."""
    Qg = np.asarray(Qg, dtype=np.float64)
    G, N_q, d = Qg.shape
    N_k = K.shape[0]
    assert N_q <= N_k, "causal mode needs N_q <= N_k (bottom-right alignment)"
    off = N_k - N_q
    nQB, nKB = num_blocks(N_q, B_q), num_blocks(N_k, B_k)
    O = np.full((G, N_q, V.shape[1]), np.nan)
    z = np.full((G, N_q), np.nan)
    keep = np.zeros((nQB, nKB), dtype=bool)
    margin = np.full((nQB, nKB), np.nan)
    for i in (range(nQB) if blocks is None else blocks):
        q0, q1 = i * B_q, min((i + 1) * B_q, N_q)
        R = q1 - q0
        rows = Qg[:, q0:q1].reshape(G * R, d)            # head-major stack of the block's rows
        pos = np.tile(np.arange(q0, q1) + off, G)
        tiles = causal_tiles(q1 - 1 + off, B_k, nKB)
        rep = None
        if replay_mask is not None:
            rep = {j: bool(replay_mask[i, j]) for j in tiles}
        st = forward_block(rows, pos, K, V, B_k, tau, tiles, replay=rep)
        Ob, zb = finalize(st)
        O[:, q0:q1] = Ob.reshape(G, R, -1)
        z[:, q0:q1] = zb.reshape(G, R)
        for j in tiles:
            keep[i, j] = st["keep"][j]
            margin[i, j] = st["margin"][j]
    return O, z, keep, margin


def forward(q, k, v, B_q: int, B_k: int, tau: float, replay_mask=None,
            heads=None):
    """Algorithm 1 over [B, N_q, Hq, d] / [B, N_k, Hkv, d] arrays (GQA: query
    head h reads key/value head h // (Hq / Hkv); N_q <= N_k, bottom-right
    aligned as in forward_head).

    replay_mask: optional bool [B, Hq, nQB, nKB]. ``heads`` optionally lists
    (b, h) pairs to compute. Returns O [B, N_q, Hq, d], lse [B, Hq, N_q],
    keep [B, Hq, nQB, nKB], margin (same shape)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    nQB, nKB = num_blocks(N, B_q), num_blocks(k.shape[1], B_k)
    O = np.full(q.shape[:3] + (v.shape[3],), np.nan)
    lse = np.full((B, Hq, N), np.nan)
    keep = np.zeros((B, Hq, nQB, nKB), dtype=bool)
    margin = np.full((B, Hq, nQB, nKB), np.nan)
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for (b, h) in pairs:
        rm = None if replay_mask is None else replay_mask[b, h]
        Oh, zh, kh, mh = forward_head(q[b, :, h], k[b, :, h // G], v[b, :, h // G],
                                      B_q, B_k, tau, rm)
        O[b, :, h], lse[b, h], keep[b, h], margin[b, h] = Oh, zh, kh, mh
    return O, lse, keep, margin


# --------------------------------------------------------------------------
# Algorithm 2 ("Offline Sparse Probability"), key-major
# --------------------------------------------------------------------------

def backward_head(Q, K, V, O, dO, z, B_q: int, B_k: int, tau: float,
                  fwd_mask: Optional[np.ndarray] = None,
                  kblocks: Optional[Iterable[int]] = None,
                  qblocks: Optional[Iterable[int]] = None):
    """Algorithm 2 for one query head against its key/value head.

    Q, O, dO [N_q, d]; K, V [N_k, d]; z [N_q] the saved log-normaliser;
    N_q <= N_k, bottom-right aligned as in forward_head.
    fwd_mask  optional bool [nQB, nKB]: when given, only tiles the forward
              retained are visited (mask replay); when None every legal tile
              is visited (the page's pure form).
    kblocks / qblocks restrict the key / query blocks visited (for sampled
    checks); dQ rows of other query blocks and dK/dV rows of other key
    blocks are then partial.

    Returns dQ, dK, dV [N, d], keep [nQB, nKB] bool, margin [nQB, nKB]."""
    Q, K, V, O, dO = (np.asarray(x, dtype=np.float64) for x in (Q, K, V, O, dO))
    z = np.asarray(z, dtype=np.float64)
    N, d = Q.shape
    N_k = K.shape[0]
    assert N <= N_k, "causal mode needs N_q <= N_k (bottom-right alignment)"
    off = N_k - N
    nQB, nKB = num_blocks(N, B_q), num_blocks(N_k, B_k)
    D = (dO * O).sum(axis=1)                         # D_q = rowsum(dO o O)
    log_tau = _log(tau)
    log_L = np.log(np.arange(1, N + 1, dtype=np.float64) + off)   # L_q = position + 1
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    keep = np.zeros((nQB, nKB), dtype=bool)
    margin = np.full((nQB, nKB), np.nan)
    qset = None if qblocks is None else set(qblocks)
    for j in (range(nKB) if kblocks is None else kblocks):
        k0, k1 = j * B_k, min((j + 1) * B_k, N_k)
        i_diag = max(0, k0 - off) // B_q             # first block with a legal row
        for i in range(i_diag, nQB):                 # ascending from the diagonal
            if qset is not None and i not in qset:
                continue
            if fwd_mask is not None and not fwd_mask[i, j]:
                continue
            q0, q1 = i * B_q, min((i + 1) * B_q, N)
            qpos = np.arange(q0, q1) + off
            kpos = np.arange(k0, k1)
            S_ji = K[k0:k1] @ Q[q0:q1].T             # recomputed key-major tile
            legal = kpos[:, None] <= qpos[None, :]
            if not legal.any():
                continue
            slack = (log_tau - log_L[q0:q1])[None, :] - (S_ji - z[q0:q1][None, :])
            M = float(np.where(legal, slack, math.inf).min())
            margin[i, j] = M
            if not (M <= 0.0):
                continue                            # skipped: no dO load, no P
            keep[i, j] = True
            P_ji = np.where(legal, np.exp(S_ji - z[q0:q1][None, :]), 0.0)
            dV[k0:k1] += P_ji @ dO[q0:q1]
            dP_ji = V[k0:k1] @ dO[q0:q1].T
            dS_ji = P_ji * (dP_ji - D[q0:q1][None, :])
            dQ[q0:q1] += dS_ji.T @ K[k0:k1]
            dK[k0:k1] += dS_ji @ Q[q0:q1]
    return dQ, dK, dV, keep, margin


def backward(q, k, v, o, do, lse, B_q: int, B_k: int, tau: float,
             fwd_mask=None):
    """Algorithm 2 over [B, N, H, d] arrays; dK/dV of a key/value head sum
    the contributions of its Hq / Hkv query heads.

    fwd_mask optional bool [B, Hq, nQB, nKB]. Returns dq, dk, dv, keep."""
    q, k, v, o, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, o, do))
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    nQB, nKB = num_blocks(N, B_q), num_blocks(k.shape[1], B_k)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    keep = np.zeros((B, Hq, nQB, nKB), dtype=bool)
    for b in range(B):
        for h in range(Hq):
            fm = None if fwd_mask is None else fwd_mask[b, h]
            dQh, dKh, dVh, kh, _ = backward_head(
                q[b, :, h], k[b, :, h // G], v[b, :, h // G], o[b, :, h],
                do[b, :, h], lse[b, h], B_q, B_k, tau, fm)
            dq[b, :, h] = dQh
            dk[b, :, h // G] += dKh
            dv[b, :, h // G] += dVh
            keep[b, h] = kh
    return dq, dk, dv, keep


# --------------------------------------------------------------------------
# Split-KV decoding (cost paragraph + Appendix A.1 "Fused decoding execution")
# --------------------------------------------------------------------------

def split_ranges(n_tiles: int, num_splits: int):
    """Contiguous key-tile ranges of the splits: [floor(pT/P), floor((p+1)T/P))."""
    return [(p * n_tiles // num_splits, (p + 1) * n_tiles // num_splits)
            for p in range(num_splits)]


def decode_head(q_row: np.ndarray, K: np.ndarray, V: np.ndarray, B_k: int,
                tau: float, num_splits: int = 1, replay=None):
    """One decoding query (position N_k - 1, L_0 = N_k) against a KV cache.

    replay: optional bool [nKB] forcing the per-tile decisions.
    Returns O [d], z, keep [nKB] bool, margin [nKB], partials list of
    (O_p, z_p)."""
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    N_k = K.shape[0]
    nKB = num_blocks(N_k, B_k)
    Qb = np.asarray(q_row, dtype=np.float64)[None, :]
    pos = np.array([N_k - 1])
    L = np.array([N_k])
    keep = np.zeros(nKB, dtype=bool)
    margin = np.full(nKB, np.nan)
    partials = []
    for (t0, t1) in split_ranges(nKB, num_splits):
        tiles = list(range(t1 - 1, t0 - 1, -1))      # descending within the split
        rep = None if replay is None else {j: bool(replay[j]) for j in tiles}
        st = forward_block(Qb, pos, K, V, B_k, tau, tiles, L_i=L, replay=rep)
        O_p, z_p = finalize(st)
        partials.append((O_p[0], float(z_p[0])))
        for j in tiles:
            keep[j] = st["keep"][j]
            margin[j] = st["margin"][j]
    O, z = merge_partials(partials)
    return O, z, keep, margin, partials


def decode_group(Q_rows: np.ndarray, K: np.ndarray, V: np.ndarray, B_k: int,
                 tau: float, num_splits: int = 1, replay=None):
    """Group-joint decoding: the G query heads that share one KV head take one
    decision per key tile. The heads' query rows (each at position N_k - 1,
    L_0 = N_k) are treated like the rows of one query block under the test of
    "Online Sparse Softmax": a tile is skipped only when every head passes the
    skip test, and a retained tile updates every head. Splits as in
    ``decode_head``, each with its own (m, l) per head.

    replay: optional bool [nKB] forcing the per-tile decisions.
    Returns O [G, d], z [G], keep [nKB] bool, margin [nKB]."""
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    Qg = np.asarray(Q_rows, dtype=np.float64)
    G = Qg.shape[0]
    N_k = K.shape[0]
    nKB = num_blocks(N_k, B_k)
    pos = np.full(G, N_k - 1)
    L = np.full(G, N_k)
    keep = np.zeros(nKB, dtype=bool)
    margin = np.full(nKB, np.nan)
    partials = [[] for _ in range(G)]
    for (t0, t1) in split_ranges(nKB, num_splits):
        tiles = list(range(t1 - 1, t0 - 1, -1))
        rep = None if replay is None else {j: bool(replay[j]) for j in tiles}
        st = forward_block(Qg, pos, K, V, B_k, tau, tiles, L_i=L, replay=rep)
        O_p, z_p = finalize(st)
        for g in range(G):
            partials[g].append((O_p[g], float(z_p[g])))
        for j in tiles:
            keep[j] = st["keep"][j]
            margin[j] = st["margin"][j]
    O = np.zeros((G, V.shape[1]))
    z = np.zeros(G)
    for g in range(G):
        O[g], z[g] = merge_partials(partials[g])
    return O, z, keep, margin


def merge_partials(partials):
    """Normalizer-aware merge: z = log sum_p exp(z_p), O = sum_p exp(z_p - z) O_p."""
    zs = np.array([zp for (_, zp) in partials])
    zmax = zs.max()
    z = zmax + math.log(np.exp(zs - zmax).sum())
    O = sum(math.exp(zp - z) * Op for (Op, zp) in partials)
    return O, z


def decode(q, k, v, B_k: int, tau: float, num_splits: int = 1, heads=None,
           replay_mask=None):
    """Decoding over q [B, 1, Hq, d] and a cache k/v [B, N_k, Hkv, d].

    Returns O [B, 1, Hq, d] (NaN outside ``heads``), lse [B, Hq],
    keep [B, Hq, nKB], margin (same)."""
    q = np.asarray(q, dtype=np.float64)
    B, _, Hq, d = q.shape
    N_k, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    nKB = num_blocks(N_k, B_k)
    O = np.full((B, 1, Hq, v.shape[3]), np.nan)
    lse = np.full((B, Hq), np.nan)
    keep = np.zeros((B, Hq, nKB), dtype=bool)
    margin = np.full((B, Hq, nKB), np.nan)
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for (b, h) in pairs:
        rep = None if replay_mask is None else replay_mask[b, h]
        Oh, zh, kh, mh, _ = decode_head(q[b, 0, h], k[b, :, h // G], v[b, :, h // G],
                                        B_k, tau, num_splits, rep)
        O[b, 0, h], lse[b, h], keep[b, h], margin[b, h] = Oh, zh, kh, mh
    return O, lse, keep, margin
