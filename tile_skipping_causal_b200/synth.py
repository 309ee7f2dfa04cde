"""Seeded synthetic workloads shaped like the MALA operator benchmarks.

This module only draws random tensors and plants structure in them; it holds
none of the attention arithmetic. Both the CUDA path (via the binding) and the
CPU oracle (via the tests) read the same tensors from here, so a parity test
compares the two on bit-identical inputs.

Conventions (MassAlloc Attention paper, "Setup" paragraph of the method):
the softmax scale 1/sqrt(d) is folded into Q, natural exp/log throughout.
Layout follows the FlashAttention interface shown on the attention tutorial
page ("Hardware paths and kernel contracts"): Q/O/dO are [B, Nq, Hq, d] and
K/V are [B, Nk, Hkv, d], last dimension contiguous.

All draws come from torch CPU generators seeded from (seed, stream-id, ...)
so that every tensor, and every (batch, kv-head) slice of a decode cache, can
be regenerated on its own. Low-precision copies are made with torch's
round-to-nearest-even float32 -> bfloat16 conversion.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

__all__ = [
    "PrefillWorkload", "DecodeWorkload", "WORKLOADS", "make_prefill",
    "make_decode_query", "make_decode_slice", "fill_decode_cache",
]

_MASK63 = (1 << 63) - 1


def _seed(*parts: int) -> int:
    """Mix integers into a 63-bit generator seed (splitmix64 finaliser)."""
    x = 0x9E3779B97F4A7C15
    for p in parts:
        x = (x ^ (int(p) & 0xFFFFFFFFFFFFFFFF)) & 0xFFFFFFFFFFFFFFFF
        x = (x * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
        x ^= x >> 31
        x = (x * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
        x ^= x >> 29
    return x & _MASK63


def _gen(*parts: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*parts))
    return g


# stream ids, so that adding a tensor never shifts another tensor's draws
_Q, _K, _V, _DO, _DELTA, _RETR, _NEEDLE_POS, _NEEDLE_DIR = range(1, 9)


@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    """A causal prefill/training workload (Nq = Nk = seqlen)."""
    name: str
    batch: int
    heads_q: int
    heads_kv: int
    seqlen: int
    head_dim: int
    block_q: int
    block_k: int
    dtype: str            # "bf16" or "fp32"
    recipe: str           # "planted_prev", "sharp_diffuse", "gqa_thirds"
    taus: tuple
    backward: bool = False

    @property
    def group(self) -> int:
        return self.heads_q // self.heads_kv


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """Single-token decoding over a bf16 KV cache (query at position Nk-1)."""
    name: str
    batch: int
    heads_q: int
    heads_kv: int
    seqlen_k: int
    head_dim: int
    block_k: int
    tau: float

    @property
    def group(self) -> int:
        return self.heads_q // self.heads_kv


WORKLOADS = {
    # one head, fp32, 64x64 tiles, planted previous-token attention
    "toy_fp32_512": PrefillWorkload("toy_fp32_512", 1, 1, 1, 512, 64, 64, 64,
                                    "fp32", "planted_prev", (0.0, 0.05, 0.5)),
    # prefill, half diffuse / half sharp (sink + planted offset) heads
    "prefill_4k": PrefillWorkload("prefill_4k", 2, 16, 16, 4096, 128, 128, 128,
                                  "bf16", "sharp_diffuse", (0.01, 0.1, 1.0)),
    # long-context GQA prefill, heads in thirds: diffuse / local / retrieval
    "gqa_32k": PrefillWorkload("gqa_32k", 1, 32, 8, 32768, 128, 128, 128,
                               "bf16", "gqa_thirds", (0.02, 0.2)),
    # attention-only training step (forward + backward)
    "train_8k": PrefillWorkload("train_8k", 4, 16, 16, 8192, 128, 128, 128,
                                "bf16", "sharp_diffuse", (0.1,), backward=True),
}

DECODE_SEQLENS = (4096, 16384, 65536, 131072)


def decode_workload(seqlen_k: int) -> DecodeWorkload:
    return DecodeWorkload(f"decode_{seqlen_k}", 64, 32, 8, seqlen_k, 128, 128, 0.05)


def _dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def make_prefill(w: PrefillWorkload, seed: int, with_do: Optional[bool] = None,
                 batch: Optional[int] = None, seqlen: Optional[int] = None):
    """Build (q, k, v[, do]) on the CPU in the workload's dtype.

    ``batch``/``seqlen`` shrink the workload while keeping its recipe (used
    for oracle-sized parity cases). Returns a dict of contiguous tensors.
    """
    B = w.batch if batch is None else batch
    N = w.seqlen if seqlen is None else seqlen
    Hq, Hkv, d = w.heads_q, w.heads_kv, w.head_dim
    G = Hq // Hkv
    q = torch.randn((B, N, Hq, d), generator=_gen(seed, _Q))
    k = torch.randn((B, N, Hkv, d), generator=_gen(seed, _K))
    v = torch.randn((B, N, Hkv, d), generator=_gen(seed, _V))
    scale = 1.0 / math.sqrt(d)

    if w.recipe == "planted_prev":
        # Q_q += 3 K_{q-1} on the unscaled query, then fold the scale
        q[:, 1:] += 3.0 * k[:, :-1].repeat_interleave(G, dim=2)
        q *= scale
    elif w.recipe == "sharp_diffuse":
        # heads [H/2, H) are sharp: attention-sink key 0 with norm x4, then
        # Q_q += 2 K_{q - delta_h} with delta_h ~ U{1..64} per head
        delta = torch.randint(1, 65, (Hq,), generator=_gen(seed, _DELTA))
        for hk in sorted({h // G for h in range(Hq // 2, Hq)}):
            k[:, 0, hk] *= 4.0
        for h in range(Hq // 2, Hq):
            hk, dl = h // G, int(delta[h])
            if dl < N:
                q[:, dl:, h] += 2.0 * k[:, : N - dl, hk]
        q *= scale
    elif w.recipe == "gqa_thirds":
        third = Hq // 3 + (1 if Hq % 3 else 0)       # 11 / 11 / 10 for 32 heads
        local = range(third, 2 * third)
        retr = range(2 * third, Hq)
        g = _gen(seed, _RETR)
        # retrieval: every 1024th key copied (x3) into 8 random later queries
        for h in retr:
            hk = h // G
            for b in range(B):
                for key in range(1024, N, 1024):
                    if N - key - 1 < 8:
                        continue
                    tgt = key + 1 + torch.randperm(N - key - 1, generator=g)[:8]
                    q[b, tgt, h] = 3.0 * k[b, key, hk]
        q *= scale
        # local: +4 nats on average over a 256-key window, added after the fold:
        # Q_q += (4 / d) * sum_{k in [q-256, q]} K_k
        csum = torch.cumsum(k.double(), dim=1)
        lo = torch.clamp(torch.arange(N) - 257, min=-1)
        for h in local:
            hk = h // G
            win = csum[:, :, hk] - torch.where(
                (lo >= 0)[None, :, None], csum[:, lo.clamp(min=0), hk],
                torch.zeros_like(csum[:, :, hk]))
            q[:, :, h] += (4.0 / d) * win.float()
    else:
        raise ValueError(w.recipe)

    dt = _dtype(w.dtype)
    out = {"q": q.to(dt).contiguous(), "k": k.to(dt).contiguous(),
           "v": v.to(dt).contiguous()}
    if with_do is None:
        with_do = w.backward
    if with_do:
        do = torch.randn((B, N, Hq, d), generator=_gen(seed, _DO))
        out["do"] = do.to(dt).contiguous()
    return out


def rademacher_like(shape, seed: int, dtype=torch.bfloat16) -> torch.Tensor:
    """Deterministic +/-1 probe for dO (operator-fidelity protocol, paper's
    experiments section)."""
    g = _gen(seed, 0xDAD)
    return (torch.randint(0, 2, shape, generator=g) * 2 - 1).to(dtype)


def make_decode_query(w: DecodeWorkload, seed: int) -> torch.Tensor:
    """Query for decoding, [B, 1, Hq, d] bf16, scale folded in."""
    q = torch.randn((w.batch, 1, w.heads_q, w.head_dim), generator=_gen(seed, _Q))
    return (q / math.sqrt(w.head_dim)).to(torch.bfloat16)


def _plant_decode(qs: torch.Tensor, k: torch.Tensor, g: torch.Generator,
                  n_needles: int = 16):
    """Sink key (x4 norm) at position 0 and needles aligned with the group's
    queries (cosine 0.8) at random positions in [1, Nk-1).

    qs: [G, d] fp32 queries of the group, k: [Nk, d] fp32 (modified)."""
    Nk, d = k.shape
    G = qs.shape[0]
    k[0] *= 4.0
    n = min(n_needles, max(Nk - 2, 0))
    pos = 1 + torch.randperm(max(Nk - 2, 1), generator=g)[:n]
    u = torch.randn((n, d), generator=g)
    for t in range(n):
        qh = qs[t % G] / qs[t % G].norm()
        ut = u[t] - (u[t] @ qh) * qh
        ut = ut / ut.norm()
        p = int(pos[t])
        k[p] = k[p].norm() * (0.8 * qh + 0.6 * ut)
    return pos


def make_decode_slice(w: DecodeWorkload, seed: int, b: int, hk: int,
                      q: Optional[torch.Tensor] = None):
    """K and V of one (batch, kv-head) cache slice, each [Nk, d] bf16 (CPU).

    ``q`` is the workload's query from :func:`make_decode_query`."""
    if q is None:
        q = make_decode_query(w, seed)
    Nk, d, G = w.seqlen_k, w.head_dim, w.group
    k = torch.randn((Nk, d), generator=_gen(seed, _K, b, hk))
    v = torch.randn((Nk, d), generator=_gen(seed, _V, b, hk))
    qs = q[b, 0, hk * G:(hk + 1) * G].float()
    _plant_decode(qs, k, _gen(seed, _NEEDLE_POS, b, hk))
    return k.to(torch.bfloat16), v.to(torch.bfloat16)


def fill_decode_cache(w: DecodeWorkload, seed: int, q: torch.Tensor,
                      device, slices=None, filler_seed: int = 0):
    """Allocate the [B, Nk, Hkv, d] bf16 K/V cache on ``device``.

    Slices listed in ``slices`` (pairs (b, hk)) are the exact CPU slices of
    :func:`make_decode_slice`; every other slice is drawn on the device with
    the same recipe from a device generator (fast, but not reproducible on
    the CPU). ``slices=None`` means all slices come from the CPU.
    """
    B, Nk, Hkv, d, G = w.batch, w.seqlen_k, w.heads_kv, w.head_dim, w.group
    k = torch.empty((B, Nk, Hkv, d), dtype=torch.bfloat16, device=device)
    v = torch.empty_like(k)
    if slices is None:
        slices = [(b, h) for b in range(B) for h in range(Hkv)]
        exact = set(slices)
    else:
        exact = set(slices)
        dg = _gen(seed, filler_seed, 0xF111, device=device)
        qd = q.to(device).float()
        for b in range(B):
            kb = torch.randn((Nk, Hkv, d), generator=dg, device=device)
            vb = torch.randn((Nk, Hkv, d), generator=dg, device=device)
            for h in range(Hkv):
                if (b, h) in exact:
                    continue
                kh = kb[:, h]
                kh[0] *= 4.0
                n = min(16, max(Nk - 2, 0))
                pos = 1 + torch.randperm(max(Nk - 2, 1), generator=dg, device=device)[:n]
                qs = qd[b, 0, h * G:(h + 1) * G]
                qh = qs[torch.arange(n, device=device) % G]
                qh = qh / qh.norm(dim=1, keepdim=True)
                u = torch.randn((n, d), generator=dg, device=device)
                u = u - (u * qh).sum(1, keepdim=True) * qh
                u = u / u.norm(dim=1, keepdim=True)
                kh[pos] = kh[pos].norm(dim=1, keepdim=True) * (0.8 * qh + 0.6 * u)
            k[b] = kb.to(torch.bfloat16)
            v[b] = vb.to(torch.bfloat16)
            del kb, vb
    for (b, h) in sorted(exact):
        ks, vs = make_decode_slice(w, seed, b, h, q)
        k[b, :, h] = ks.to(device)
        v[b, :, h] = vs.to(device)
    return k, v
