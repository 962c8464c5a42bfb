"""Seeded synthetic inputs shaped like the workloads the pages evaluate.

This module only draws random tensors and builds index structures (chunk
tables, needle positions, duplicated blocks).  It holds none of the method's
arithmetic: no scoring, no selection, no attention.  Both the CUDA path and
the float64 oracle receive the tensors made here (the oracle gets host copies
of the same bf16 values).

Seeds: workload c, layer l -> torch generator seed 1000*c + l; structural
choices (needle pages, chunk lengths, planted pairs) use
numpy.random.default_rng(1000*c + 999) unless a caller passes its own.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

D = 128


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn_bf16(shape, gen: torch.Generator, device, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def chunk_lengths(rng: np.random.Generator, n_tokens: int, lo: int = 16, hi: int = 256) -> np.ndarray:
    """Structure-aligned chunk lengths drawn uniformly in [lo, hi] until the
    sequence is covered; the final chunk is cut to the remaining tokens."""
    lens = []
    total = 0
    while total < n_tokens:
        L = int(rng.integers(lo, hi + 1))
        L = min(L, n_tokens - total)
        lens.append(L)
        total += L
    return np.array(lens, dtype=np.int64)


@dataclass
class DecodeLayer:
    """One layer of a decode step: the current query rows and the KV cache
    (which already holds the current token)."""
    q: torch.Tensor            # [B, Hq, D] bf16
    k: torch.Tensor            # [B, Hkv, cap, D] bf16
    v: torch.Tensor            # [B, Hkv, cap, D] bf16
    seq_len: torch.Tensor      # [B] int32
    chunk_off: torch.Tensor | None = None   # [B, max_chunks + 1] int32 (variable chunks)
    n_chunks: torch.Tensor | None = None    # [B] int32
    extra: dict = field(default_factory=dict)


def _chunk_table(chunk_lens_per_seq, device):
    B = len(chunk_lens_per_seq)
    maxc = max(len(x) for x in chunk_lens_per_seq)
    off = np.zeros((B, maxc + 1), dtype=np.int32)
    nch = np.zeros(B, dtype=np.int32)
    for b, lens in enumerate(chunk_lens_per_seq):
        o = np.concatenate([[0], np.cumsum(lens)])
        off[b, :len(o)] = o
        off[b, len(o):] = o[-1]
        nch[b] = len(lens)
    return torch.from_numpy(off).to(device), torch.from_numpy(nch).to(device)


def make_decode_layer(*, B: int, Hq: int, Hkv: int, seq_lens, seed: int, device,
                      cap: int | None = None, key_scale: str = "none",
                      chunk_lens=None, chunk_offset_std: float = 0.0,
                      needles: dict | None = None) -> DecodeLayer:
    """Q, K, V drawn i.i.d. N(0,1) in bf16, with optional structure:

    key_scale='channel': every key channel of a (KV head) is multiplied by a
      scale drawn log-uniformly in [0.5, 4], shared over tokens and batch.
    chunk_lens: per-sequence list of chunk lengths (variable chunking).  With
      chunk_offset_std > 0 every (chunk, KV head, channel) gets a random mean
      offset N(0, std^2) added to all of the chunk's keys.
    needles: {'pages': [[p0, p1, p2] per KV head], 'page_size': 16,
      'strength': 4.0}: in the listed pages every key becomes N(0,1) plus
      strength * q_h / |q_h|, needle j of KV head g using query head g*G + j.
    """
    seq_lens = [int(x) for x in (seq_lens if hasattr(seq_lens, "__len__") else [seq_lens] * B)]
    assert len(seq_lens) == B
    if cap is None:
        cap = max(seq_lens)
    gen = _gen(device, seed)
    q = randn_bf16((B, Hq, D), gen, device)
    k = torch.randn((B, Hkv, cap, D), generator=gen, device=device, dtype=torch.float32)
    if key_scale == "channel":
        u = torch.rand((Hkv, D), generator=gen, device=device, dtype=torch.float32)
        scale = torch.exp(np.log(0.5) + u * (np.log(4.0) - np.log(0.5)))
        k.mul_(scale[None, :, None, :])
    chunk_off = n_chunks = None
    if chunk_lens is not None:
        if chunk_offset_std > 0:
            for b in range(B):
                lens = torch.as_tensor(np.asarray(chunk_lens[b]), device=device)
                C = len(lens)
                offs = torch.randn((Hkv, C, D), generator=gen, device=device,
                                   dtype=torch.float32) * chunk_offset_std
                tok = torch.repeat_interleave(offs, lens, dim=1)  # [Hkv, N_b, D]
                k[b, :, :tok.shape[1]] += tok
        chunk_off, n_chunks = _chunk_table(chunk_lens, device)
    v = randn_bf16((B, Hkv, cap, D), gen, device)
    if needles is not None:
        G = Hq // Hkv
        ps = needles.get("page_size", 16)
        strength = needles.get("strength", 4.0)
        qf = q.float()
        for b in range(B):
            for g, pages in enumerate(needles["pages"]):
                for j, p in enumerate(pages):
                    h = g * G + j
                    dirn = qf[b, h] / qf[b, h].norm()
                    k[b, g, p * ps:(p + 1) * ps] += strength * dirn
    k = k.to(torch.bfloat16)
    sl = torch.tensor(seq_lens, dtype=torch.int32, device=device)
    return DecodeLayer(q, k, v, sl, chunk_off, n_chunks)


# --------------------------------------------------------------------------
# The five workloads.  Sizes follow the shapes of the models the pages name.
# --------------------------------------------------------------------------

@dataclass
class Workload:
    name: str
    layers: int
    B: int
    Hq: int
    Hkv: int
    N: int
    page_size: int          # 0 = variable chunks
    idx: int                # workload number, used for seeds


WORKLOADS = {
    1: Workload("needle-2k", 1, 1, 32, 4, 2048, 16, 1),
    2: Workload("qwen3vl30b-a3b-decode-29.5k", 48, 1, 32, 4, 29504, 16, 2),
    3: Workload("tsa-chunks-29.5k-b4", 48, 4, 32, 4, 29504, 0, 3),
    4: Workload("qwen3-32b-ratio-32k-b8", 64, 8, 64, 8, 32768, 16, 4),
    5: Workload("router-qwen2.5-7b-128k", 1, 1, 28, 4, 131072, 64, 5),
}


def needle_pages(Hkv: int, n_pages: int, rng: np.random.Generator, per_head: int = 3):
    return [sorted(int(x) for x in rng.choice(n_pages, per_head, replace=False))
            for _ in range(Hkv)]


def workload1_layer(device, seed_offset: int = 0) -> DecodeLayer:
    w = WORKLOADS[1]
    rng = np.random.default_rng(1000 * w.idx + 999 + seed_offset)
    pages = needle_pages(w.Hkv, w.N // 16, rng)
    lay = make_decode_layer(B=w.B, Hq=w.Hq, Hkv=w.Hkv, seq_lens=w.N,
                            seed=1000 * w.idx + seed_offset, device=device,
                            needles={"pages": pages, "page_size": 16, "strength": 4.0})
    lay.extra["needle_pages"] = pages
    return lay


def workload2_layer(layer: int, device, N: int | None = None, cap: int | None = None) -> DecodeLayer:
    w = WORKLOADS[2]
    return make_decode_layer(B=w.B, Hq=w.Hq, Hkv=w.Hkv, seq_lens=N or w.N, cap=cap,
                             seed=1000 * w.idx + layer, device=device, key_scale="channel")


def workload3_chunks(B: int, N: int, seed_offset: int = 0):
    rng = np.random.default_rng(1000 * 3 + 999 + seed_offset)
    return [chunk_lengths(rng, N) for _ in range(B)]


def workload3_layer(layer: int, device, N: int | None = None, B: int | None = None,
                    chunk_lens=None) -> DecodeLayer:
    w = WORKLOADS[3]
    N = N or w.N
    B = B or w.B
    if chunk_lens is None:
        chunk_lens = workload3_chunks(B, N)
    return make_decode_layer(B=B, Hq=w.Hq, Hkv=w.Hkv, seq_lens=N, seed=1000 * w.idx + layer,
                             device=device, chunk_lens=chunk_lens, chunk_offset_std=0.5)


def workload4_layer(layer: int, device, B: int | None = None, N: int | None = None) -> DecodeLayer:
    w = WORKLOADS[4]
    return make_decode_layer(B=B or w.B, Hq=w.Hq, Hkv=w.Hkv, seq_lens=N or w.N,
                             seed=1000 * w.idx + layer, device=device)


WORKLOAD4_RATIOS = (0.5, 0.375, 0.25, 0.125, 0.0625, 0.03125, 0.015625)


@dataclass
class RouterLayer:
    q: torch.Tensor   # [rows, Hq, D] bf16, rows at positions q_pos0 ..
    k: torch.Tensor   # [1, Hkv, N, D] bf16
    v: torch.Tensor   # [1, Hkv, N, D] bf16
    q_pos0: int
    N: int


def make_router_layer(*, Hq: int = 28, Hkv: int = 4, N: int = 131072, rows: int = 2048,
                      seed: int = 5000, device) -> RouterLayer:
    """Chunked-prefill rows: the last `rows` positions of an N-token cache."""
    gen = _gen(device, seed)
    q = randn_bf16((rows, Hq, D), gen, device)
    k = randn_bf16((1, Hkv, N, D), gen, device)
    v = randn_bf16((1, Hkv, N, D), gen, device)
    return RouterLayer(q, k, v, N - rows, N)


def duplicate_block(k: torch.Tensor, g: int, src: int, dst: int, block: int,
                    eps: float, gen: torch.Generator) -> None:
    """Overwrite block `dst` of KV head g with the keys of block `src` plus
    N(0, eps^2) noise (a near-tie pair).  In place, on k's device."""
    s = k[0, g, src * block:(src + 1) * block].float()
    noise = torch.randn(s.shape, generator=gen, device=k.device, dtype=torch.float32) * eps
    k[0, g, dst * block:(dst + 1) * block] = (s + noise).to(k.dtype)
