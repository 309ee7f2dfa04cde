"""Parity helpers shared by the GPU tests: compare CUDA results with the fp64
oracle on the same seeded inputs.

Tolerances (fixed for this operator):
* keep masks identical, except tiles whose oracle margin is within
  MARGIN_BAND = 1e-3 nats of the threshold;
* O and LSE within ATOL = 1e-2 absolute + RTOL = 2e-2 relative, measured
  against the oracle replaying the GPU's decisions (so that a legitimate
  near-tie decision does not change the reference);
* dQ, dK, dV within GRAD_RFE = 3e-2 relative Frobenius error.

Mask replay: the oracle first runs on its own. If its decisions equal the
GPU's, outputs are compared directly. Otherwise the oracle re-runs with the
GPU's decisions forced, still evaluating every tile's margin at its own
state; each GPU decision must then agree with the sign of that margin or
lie inside the band.
"""
import math

import numpy as np
import torch

from oracle import mala_oracle as orc
from tile_skipping_causal_b200 import mala

MARGIN_BAND = 1e-3
ATOL = 1e-2
RTOL = 2e-2
GRAD_RFE = 3e-2


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close(got, ref, what, atol=ATOL, rtol=RTOL):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite GPU values"
    err = np.abs(got - ref)
    bad = err > atol + rtol * np.abs(ref)
    if bad.any():
        idx = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} / {bad.size} elements out of tolerance; "
                             f"first at {tuple(idx)}: got {got[tuple(idx)]}, ref {ref[tuple(idx)]}, "
                             f"max abs err {err.max():.3e}")


def rel_fro(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))


class FwdReport:
    def __init__(self):
        self.blocks = 0
        self.tiles = 0
        self.kept = 0
        self.band_flips = 0
        self.replayed_blocks = 0


def check_fwd_block(Q, K, V, pos, tiles, B_k, tau, gpu_keep_row, gpu_O, gpu_lse, rep, what,
                    L=None):
    """One query block: Q [R, d] fp64 (valid rows), K/V [N_k, d], gpu_keep_row
    bool [nKB], gpu_O [R, d], gpu_lse [R]."""
    st = orc.forward_block(Q, pos, K, V, B_k, tau, tiles, L_i=L)
    gdec = {j: bool(gpu_keep_row[j]) for j in tiles}
    if any(st["keep"][j] != gdec[j] for j in tiles):
        rep.replayed_blocks += 1
        st = orc.forward_block(Q, pos, K, V, B_k, tau, tiles, L_i=L, replay=gdec)
    for j in tiles:
        mj = st["margin"][j]
        if gdec[j] != (mj <= 0.0):
            assert abs(mj) <= MARGIN_BAND, f"{what}: tile {j} decided {gdec[j]} with margin {mj:.3e}"
            rep.band_flips += 1
    others = np.ones(len(gpu_keep_row), dtype=bool)
    others[list(tiles)] = False
    assert not np.asarray(gpu_keep_row)[others].any(), f"{what}: bits set outside the causal tiles"
    O, z = orc.finalize(st)
    assert_close(gpu_O, O, f"{what} O")
    assert_close(gpu_lse, z, f"{what} LSE")
    rep.blocks += 1
    rep.tiles += len(tiles)
    rep.kept += sum(gdec.values())


def check_fwd(q, k, v, o, lse, keep_words, tau, B_q, B_k, samples=None, rep=None):
    """Compare mala_fwd outputs with the oracle on query blocks ``samples``
    (list of (b, h, i); None = all)."""
    rep = rep or FwdReport()
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    off = k.shape[1] - N                          # bottom-right alignment when N_q < N_k
    nQB, nKB = orc.num_blocks(N, B_q), orc.num_blocks(k.shape[1], B_k)
    keep = mala.unpack_mask(keep_words, nKB)
    o64 = None
    if samples is None:
        samples = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(nQB)]
    by_head = {}
    for (b, h, i) in samples:
        by_head.setdefault((b, h), []).append(i)
    lse_c = lse.detach().cpu().numpy()
    for (b, h), blocks in by_head.items():
        Qh, Kh, Vh = f64(q[b, :, h]), f64(k[b, :, h // G]), f64(v[b, :, h // G])
        Oh = f64(o[b, :, h])
        for i in blocks:
            q0, q1 = i * B_q, min((i + 1) * B_q, N)
            pos = np.arange(q0, q1) + off
            tiles = orc.causal_tiles(q1 - 1 + off, B_k, nKB)
            check_fwd_block(Qh[q0:q1], Kh, Vh, pos, tiles, B_k, tau, keep[b, h, i], Oh[q0:q1],
                            lse_c[b, h, q0:q1], rep, f"fwd b={b} h={h} i={i}")
    return rep


class DecReport:
    def __init__(self):
        self.heads = 0
        self.tiles = 0
        self.kept = 0
        self.band_flips = 0
        self.replayed = 0


def check_decode_head(q_row, K, V, B_k, tau, P, gpu_keep_row, gpu_o, gpu_lse, rep, what):
    """One (batch, query head) of mala_decode against the oracle's split-KV
    decode with the same split count."""
    O, z, keep, margin, _ = orc.decode_head(q_row, K, V, B_k, tau, P)
    nKB = len(keep)
    gk = np.asarray(gpu_keep_row[:nKB], dtype=bool)
    if (keep != gk).any():
        rep.replayed += 1
        O, z, keep, margin, _ = orc.decode_head(q_row, K, V, B_k, tau, P, replay=gk)
    for j in range(nKB):
        if gk[j] != (margin[j] <= 0.0):
            assert abs(margin[j]) <= MARGIN_BAND, f"{what}: tile {j} decided {gk[j]} with margin {margin[j]:.3e}"
            rep.band_flips += 1
    assert_close(gpu_o, O, f"{what} O")
    assert_close(np.array([gpu_lse]), np.array([z]), f"{what} LSE")
    rep.heads += 1
    rep.tiles += nKB
    rep.kept += int(gk.sum())


def check_decode(q, k, v, o, lse, keep_words, tau, P, B_k=128, heads=None, rep=None):
    """mala_decode outputs vs the oracle for (b, h) pairs ``heads`` (None = all).
    q [B, 1, Hq, d]; k/v [B, Nk, Hkv, d] (device or host tensors)."""
    rep = rep or DecReport()
    B, _, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    nKB = orc.num_blocks(Nk, B_k)
    keep = mala.unpack_mask(keep_words, nKB)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    o_c = f64(o)
    lse_c = lse.detach().cpu().numpy()
    by_kv = {}
    for (b, h) in heads:
        by_kv.setdefault((b, h // G), []).append(h)
    for (b, hk), hs in by_kv.items():
        K, V = f64(k[b, :, hk]), f64(v[b, :, hk])
        for h in hs:
            check_decode_head(f64(q[b, 0, h]), K, V, B_k, tau, P, keep[b, h], o_c[b, 0, h],
                              float(lse_c[b, h]), rep, f"decode b={b} h={h}")
    return rep


def check_decode_group(q, k, v, o, lse, keep_words, tau, P, B_k=128, groups=None, rep=None):
    """mala_decode(group_vote=True) vs the oracle's group-joint decoding for
    (batch, KV head) pairs ``groups`` (None = all), default head map. The
    heads of a group must carry identical keep bits; a decision that differs
    from the oracle's must lie inside the margin band (the oracle then
    replays the GPU's decisions); every head's O and LSE must match."""
    rep = rep or DecReport()
    B, _, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    nKB = orc.num_blocks(Nk, B_k)
    keep = mala.unpack_mask(keep_words, nKB)
    if groups is None:
        groups = [(b, hk) for b in range(B) for hk in range(Hkv)]
    o_c = f64(o)
    lse_c = lse.detach().cpu().numpy()
    for (b, hk) in groups:
        h0 = hk * G
        gk = np.asarray(keep[b, h0, :nKB], dtype=bool)
        for h in range(h0 + 1, h0 + G):
            assert (np.asarray(keep[b, h, :nKB], dtype=bool) == gk).all(), \
                f"group b={b} hk={hk}: heads {h0} and {h} carry different keep bits"
        Qg = f64(q[b, 0, h0:h0 + G])
        K, V = f64(k[b, :, hk]), f64(v[b, :, hk])
        O, z, okeep, margin = orc.decode_group(Qg, K, V, B_k, tau, P)
        if (okeep != gk).any():
            rep.replayed += 1
            O, z, okeep, margin = orc.decode_group(Qg, K, V, B_k, tau, P, replay=gk)
        for j in range(nKB):
            if gk[j] != (margin[j] <= 0.0):
                assert abs(margin[j]) <= MARGIN_BAND, \
                    f"group b={b} hk={hk}: tile {j} decided {gk[j]} with margin {margin[j]:.3e}"
                rep.band_flips += 1
        for i in range(G):
            assert_close(o_c[b, 0, h0 + i], O[i], f"group decode b={b} h={h0 + i} O")
            assert_close(np.array([lse_c[b, h0 + i]]), np.array([z[i]]), f"group decode b={b} h={h0 + i} LSE")
            rep.heads += 1
        rep.tiles += nKB
        rep.kept += int(gk.sum())
    return rep


def check_fwd_group(q, k, v, o, lse, keep_words, tau, groups=None, B_q=128, B_k=128):
    """mala_fwd(group_vote=True) vs the oracle's group-joint prefill for
    (batch, KV head) pairs ``groups`` (None = all), default head map, all
    query blocks. The heads of a group must carry identical keep bits; a
    decision that differs from the oracle's must lie inside the margin band
    (the oracle then replays the GPU's decisions); O and LSE of every row of
    every head must match. Returns (blocks, tiles visited, tiles kept)."""
    B, N, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    nQB, nKB = orc.num_blocks(N, B_q), orc.num_blocks(Nk, B_k)
    keep = mala.unpack_mask(keep_words, nKB)             # [B, Hq, nQB, nKB]
    if groups is None:
        groups = [(b, hk) for b in range(B) for hk in range(Hkv)]
    o_c, lse_c = f64(o), lse.detach().cpu().numpy()
    q64, k64, v64 = f64(q), f64(k), f64(v)
    nblk = ntiles = nkept = 0
    for (b, hk) in groups:
        h0 = hk * G
        gk = np.asarray(keep[b, h0], dtype=bool)
        for h in range(h0 + 1, h0 + G):
            assert (np.asarray(keep[b, h], dtype=bool) == gk).all(), \
                f"group b={b} hk={hk}: heads {h0} and {h} carry different keep bits"
        Qg = np.stack([q64[b, :, h0 + g] for g in range(G)])
        K, V = k64[b, :, hk], v64[b, :, hk]
        O, z, okeep, margin = orc.forward_group(Qg, K, V, B_q, B_k, tau)
        visited = ~np.isnan(margin)
        if (okeep[visited] != gk[visited]).any():
            O, z, okeep, margin = orc.forward_group(Qg, K, V, B_q, B_k, tau, replay_mask=gk)
        for (i, j) in zip(*np.nonzero(visited)):
            if gk[i, j] != (margin[i, j] <= 0.0):
                assert abs(margin[i, j]) <= MARGIN_BAND, \
                    f"group b={b} hk={hk} block {i} tile {j}: decided {gk[i, j]} with margin {margin[i, j]:.3e}"
        assert not gk[~visited].any(), f"group b={b} hk={hk}: bits set on tiles never visited"
        for g in range(G):
            assert_close(o_c[b, :, h0 + g], O[g], f"group fwd b={b} h={h0 + g} O")
            assert_close(lse_c[b, h0 + g], z[g], f"group fwd b={b} h={h0 + g} LSE")
        nblk += nQB
        ntiles += int(visited.sum())
        nkept += int(gk[visited].sum())
    return nblk, ntiles, nkept


def oracle_forward_replaying(q64, k64, v64, b, h, G, blocks, gpu_keep_bh, B_q, B_k, tau, rep=None):
    """Oracle O and z for query blocks ``blocks`` of head (b, h), with the
    GPU's forward decisions forced; every forced decision that differs from
    the oracle's own must lie inside the margin band. Returns full-length
    O [N, d] and z [N] arrays (NaN outside the blocks)."""
    Q, K, V = q64[b, :, h], k64[b, :, h // G], v64[b, :, h // G]
    N = Q.shape[0]
    off = K.shape[0] - N
    nKB = orc.num_blocks(K.shape[0], B_k)
    O = np.full((N, V.shape[1]), np.nan)
    z = np.full(N, np.nan)
    for i in blocks:
        q0, q1 = i * B_q, min((i + 1) * B_q, N)
        tiles = orc.causal_tiles(q1 - 1 + off, B_k, nKB)
        gdec = {j: bool(gpu_keep_bh[i, j]) for j in tiles}
        st = orc.forward_block(Q[q0:q1], np.arange(q0, q1) + off, K, V, B_k, tau, tiles, replay=gdec)
        for j in tiles:
            mj = st["margin"][j]
            if gdec[j] != (mj <= 0.0):
                assert abs(mj) <= MARGIN_BAND, f"fwd b={b} h={h} i={i} tile {j}: margin {mj:.3e}"
                if rep is not None:
                    rep["fwd_band_flips"] = rep.get("fwd_band_flips", 0) + 1
        O[q0:q1], z[q0:q1] = orc.finalize(st)
    return O, z


def as_operator_outputs(O, z):
    """The forward operator emits O in bf16 and the log-normaliser in fp32;
    the backward consumes exactly those. Round the oracle's fp64 values the
    same way before they feed the oracle's backward (D = rowsum(dO o O) is a
    cancelling difference for sharp rows, so the O precision matters)."""
    Ob = torch.from_numpy(np.ascontiguousarray(O)).to(torch.bfloat16).to(torch.float64).numpy()
    zf = np.asarray(z, dtype=np.float32).astype(np.float64)
    return Ob, zf


def check_bwd_blocks(q, k, v, do, fwd_keep_words, bwd_keep_words, dq, dk, dv, tau,
                     kv_samples=None, q_samples=None, B_q=128, B_k=128, group_vote=False):
    """Backward parity. kv_samples: (b, hk, j) key blocks whose dK/dV rows are
    checked (None = all); q_samples: (b, h, i) query blocks whose dQ rows are
    checked (None = all). Gradients by relative Frobenius error per block;
    backward decisions by the margin band. group_vote: the forward mask came
    from group-joint voting, so the oracle's forward outputs are those of its
    group-joint prefill replaying that mask (default head map)."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    Nk = k.shape[1]
    off = Nk - N                                  # bottom-right alignment when N_q < N_k
    nQB, nKB = orc.num_blocks(N, B_q), orc.num_blocks(Nk, B_k)
    fkeep = mala.unpack_mask(fwd_keep_words, nKB)
    bkeep = mala.unpack_mask(bwd_keep_words, nKB) if bwd_keep_words is not None else None
    q64, k64, v64, do64 = f64(q), f64(k), f64(v), f64(do)
    dq64, dk64, dv64 = f64(dq), f64(dk), f64(dv)
    if kv_samples is None:
        kv_samples = [(b, hk, j) for b in range(B) for hk in range(Hkv) for j in range(nKB)]
    if q_samples is None:
        q_samples = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(nQB)]
    worst = 0.0
    rep = {}
    cache = {}
    err2 = {"dQ": 0.0, "dK": 0.0, "dV": 0.0}
    ref2 = {"dQ": 0.0, "dK": 0.0, "dV": 0.0}

    def fwd_rows_group(b, h):
        if (b, h) not in cache:
            hk = h // G
            h0 = hk * G
            gm = np.asarray(fkeep[b, h0], dtype=bool)
            Qg = np.stack([q64[b, :, h0 + g] for g in range(G)])
            O, z, _, margin = orc.forward_group(Qg, k64[b, :, hk], v64[b, :, hk], B_q, B_k, tau, replay_mask=gm)
            for (i, j) in zip(*np.nonzero(~np.isnan(margin))):
                if gm[i, j] != (margin[i, j] <= 0.0):
                    assert abs(margin[i, j]) <= MARGIN_BAND, \
                        f"group fwd b={b} hk={hk} tile ({i},{j}): margin {margin[i, j]:.3e}"
            for g in range(G):
                cache[(b, h0 + g)] = (O[g], z[g])
        return as_operator_outputs(*cache[(b, h)])

    def fwd_rows(b, h, blocks):
        if group_vote:
            return fwd_rows_group(b, h)
        key = (b, h)
        O, z = cache.get(key, (None, None))
        need = [i for i in blocks if O is None or np.isnan(z[i * B_q])]
        if need:
            O2, z2 = oracle_forward_replaying(q64, k64, v64, b, h, G, need, fkeep[b, h], B_q, B_k, tau, rep)
            if O is None:
                O, z = O2, z2
            else:
                sel = ~np.isnan(z2)
                O[sel], z[sel] = O2[sel], z2[sel]
            cache[key] = (O, z)
        return as_operator_outputs(*cache[key])

    def check_bmask(b, h, bk_ref, bm_ref, blocks_i, blocks_j):
        if bkeep is None:
            return
        for i in blocks_i:
            for j in blocks_j:
                if np.isnan(bm_ref[i, j]):
                    continue
                if bool(bkeep[b, h, i, j]) != bool(bk_ref[i, j]):
                    assert abs(bm_ref[i, j]) <= MARGIN_BAND, \
                        f"bwd b={b} h={h} tile ({i},{j}): margin {bm_ref[i, j]:.3e}"

    for (b, hk, j) in kv_samples:
        k0, k1 = j * B_k, min((j + 1) * B_k, Nk)
        dK = np.zeros((k1 - k0, d))
        dV = np.zeros((k1 - k0, d))
        i_first = max(0, k0 - off) // B_q
        for h in range(hk * G, (hk + 1) * G):
            blocks = [i for i in range(i_first, nQB) if fkeep[b, h, i, j]]
            if not blocks:
                continue
            O, z = fwd_rows(b, h, blocks)
            dQh, dKh, dVh, bk_ref, bm_ref = orc.backward_head(
                q64[b, :, h], k64[b, :, hk], v64[b, :, hk], O, do64[b, :, h], z, B_q, B_k, tau,
                fkeep[b, h], kblocks=[j], qblocks=blocks)
            dK += dKh[k0:k1]
            dV += dVh[k0:k1]
            check_bmask(b, h, bk_ref, bm_ref, blocks, [j])
        for name, got, ref in (("dK", dk64[b, k0:k1, hk], dK), ("dV", dv64[b, k0:k1, hk], dV)):
            assert np.isfinite(got).all(), f"{name} b={b} hk={hk} j={j}: non-finite"
            if np.linalg.norm(ref) == 0.0:
                # an exactly cancelling reference (e.g. a single key: dS = dP - D = 0)
                # leaves only fp32 summation-order residue on the GPU
                assert np.abs(got).max() <= 1e-3, f"{name} b={b} hk={hk} j={j}: expected ~zeros"
                continue
            err2[name] += float(np.sum((got - ref) ** 2))
            ref2[name] += float(np.sum(ref ** 2))
            worst = max(worst, rel_fro(got, ref))

    for (b, h, i) in q_samples:
        q0, q1 = i * B_q, min((i + 1) * B_q, N)
        O, z = fwd_rows(b, h, [i])
        dQh, _, _, bk_ref, bm_ref = orc.backward_head(
            q64[b, :, h], k64[b, :, h // G], v64[b, :, h // G], O, do64[b, :, h], z, B_q, B_k, tau,
            fkeep[b, h], qblocks=[i])
        check_bmask(b, h, bk_ref, bm_ref, [i], range(0, min(nKB, (q1 - 1 + off) // B_k + 1)))
        got, ref = dq64[b, q0:q1, h], dQh[q0:q1]
        assert np.isfinite(got).all(), f"dQ b={b} h={h} i={i}: non-finite"
        if np.linalg.norm(ref) == 0.0:
            assert np.abs(got).max() <= 1e-3, f"dQ b={b} h={h} i={i}: expected ~zeros"
            continue
        err2["dQ"] += float(np.sum((got - ref) ** 2))
        ref2["dQ"] += float(np.sum(ref ** 2))
        worst = max(worst, rel_fro(got, ref))
    # the tolerance is a relative Frobenius error of each gradient tensor
    # (over the checked rows); single blocks whose gradient nearly cancels
    # can carry a larger relative error without mattering for the tensor
    for name in err2:
        if ref2[name] > 0.0:
            e = (err2[name] / ref2[name]) ** 0.5
            rep[name] = e
            assert e <= GRAD_RFE, f"{name}: rel. Frobenius error {e:.3e} over the checked rows"
    rep["worst_block_rel_fro"] = worst
    rep["worst_rel_fro"] = max([rep[n] for n in err2 if n in rep] or [0.0])
    return rep
