"""Seeded synthetic workloads for the QSA hot path.

This module only draws random tensors and lays them out; it holds none of the
method's arithmetic (no block means, no scores, no selection, no attention), so
that both the CUDA path and the fp64 oracle can consume the very same bytes
without sharing any computation.

Layouts (all row-major, the innermost index last):
  q    [batch][n_q][Hq][d]        query rows (post-projection, post-RoPE)
  qi   [batch][n_q][Hi][di]       indexer query heads
  k, v [batch][Hkv][kv_cap][d]    attention keys / values, one KV head plane each
  ki   [batch][kv_cap][di]        the single indexer key head
  kv_start[b]  storage index of the sequence's first real token (left pad)
  kv_len[b]    number of real tokens (relative positions 0 .. kv_len-1)
  q_first[b]   relative position of query row 0 (negative rows are padding)

Decode workloads additionally carry the new token's k/v/ki (k_new, v_new:
[batch][Hkv][d]; ki_new: [batch][di]); the cache rows before kv_len-1 are
filled, row kv_len-1 is poisoned until the append writes it.

Regions that a correct implementation must never read (left pads, cache rows
at or beyond the visible length) are filled with NaN when ``poison`` is set, so
that a stray read shows up as a NaN in the output.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    mode: str  # "prefill" | "decode"
    batch: int
    seq: int  # padded prefill length, or cache capacity for decode
    Hq: int
    Hkv: int
    d: int
    Hi: int
    di: int
    block: int  # indexer_compress_ratio
    topk: int  # blocks per query; indexer_budget = topk * block
    dtype: str  # "bf16" | "fp32"
    seed: int
    std: float
    pad_max: int = 0  # left pad drawn uniform in [0, pad_max]
    len_min: int = 0  # decode: cache length range
    len_max: int = 0
    planted: int = 0  # planted high-similarity blocks (long prefill)
    planted_std: float = 0.1

    @property
    def budget(self) -> int:
        return self.topk * self.block

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the benchmark description, by what they are, and two at head_dim 256.
WORKLOADS: Dict[str, Workload] = {
    "tiny_fp32_prefill_s256": Workload(
        name="tiny_fp32_prefill_s256", mode="prefill", batch=1, seq=256, Hq=4, Hkv=1,
        d=64, Hi=2, di=32, block=32, topk=4, dtype="fp32", seed=0, std=1.0),
    "bf16_prefill_s8192": Workload(
        name="bf16_prefill_s8192", mode="prefill", batch=1, seq=8192, Hq=16, Hkv=2,
        d=128, Hi=4, di=64, block=64, topk=32, dtype="bf16", seed=1, std=0.5),
    "bf16_decode_b64_l4k_32k": Workload(
        name="bf16_decode_b64_l4k_32k", mode="decode", batch=64, seq=32768, Hq=16,
        Hkv=2, d=128, Hi=4, di=64, block=64, topk=32, dtype="bf16", seed=2, std=0.5,
        len_min=4096, len_max=32768),
    "bf16_prefill_s65536_planted": Workload(
        name="bf16_prefill_s65536_planted", mode="prefill", batch=1, seq=65536, Hq=16,
        Hkv=2, d=128, Hi=4, di=64, block=64, topk=64, dtype="bf16", seed=3, std=0.5,
        planted=32),
    "bf16_prefill_varlen_b8_s16384_leftpad": Workload(
        name="bf16_prefill_varlen_b8_s16384_leftpad", mode="prefill", batch=8,
        seq=16384, Hq=32, Hkv=4, d=128, Hi=8, di=64, block=128, topk=16, dtype="bf16",
        seed=4, std=0.5, pad_max=2048),
    # the 8K prefill and the 64-sequence decode at head_dim 256, Qwen4ExpTextConfig's
    # default head width
    "bf16_prefill_s8192_hd256": Workload(
        name="bf16_prefill_s8192_hd256", mode="prefill", batch=1, seq=8192, Hq=16, Hkv=2,
        d=256, Hi=4, di=64, block=64, topk=32, dtype="bf16", seed=1, std=0.5),
    "bf16_decode_b64_l4k_32k_hd256": Workload(
        name="bf16_decode_b64_l4k_32k_hd256", mode="decode", batch=64, seq=32768, Hq=16,
        Hkv=2, d=256, Hi=4, di=64, block=64, topk=32, dtype="bf16", seed=2, std=0.5,
        len_min=4096, len_max=32768),
}


def _randn(gen: torch.Generator, shape, std: float, dtype: torch.dtype) -> torch.Tensor:
    # Draw in fp32, scale, round once to the storage type (round-to-nearest-even).
    return (torch.randn(shape, generator=gen, dtype=torch.float32) * std).to(dtype)


def draw_decode_lengths(gen: torch.Generator, batch: int, lo: int, hi: int, block: int):
    """Lengths uniform in [lo, hi], redrawn while divisible by the block size."""
    out = []
    for _ in range(batch):
        while True:
            L = int(torch.randint(lo, hi + 1, (1,), generator=gen).item())
            if L % block != 0:
                break
        out.append(L)
    return out


def make_inputs(w: Workload, poison: bool = True) -> Dict[str, torch.Tensor]:
    """Return CPU tensors for workload ``w`` (seeded, deterministic)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed)
    dt = w.torch_dtype
    nan = float("nan")
    B, S = w.batch, w.seq
    if w.mode == "prefill":
        if w.pad_max > 0:
            pads = [int(x) for x in torch.randint(0, w.pad_max + 1, (B,), generator=gen)]
        else:
            pads = [0] * B
        q = _randn(gen, (B, S, w.Hq, w.d), w.std, dt)
        k = _randn(gen, (B, w.Hkv, S, w.d), w.std, dt)
        v = _randn(gen, (B, w.Hkv, S, w.d), w.std, dt)
        qi = _randn(gen, (B, S, w.Hi, w.di), w.std, dt)
        ki = _randn(gen, (B, S, w.di), w.std, dt)
        if w.planted > 0:
            _plant_blocks(gen, w, q, k, qi, ki, pads)
        if poison:
            for b, p in enumerate(pads):
                if p:
                    q[b, :p] = nan
                    qi[b, :p] = nan
                    k[b, :, :p] = nan
                    v[b, :, :p] = nan
                    ki[b, :p] = nan
        kv_start = torch.tensor(pads, dtype=torch.int32)
        kv_len = torch.tensor([S - p for p in pads], dtype=torch.int32)
        q_first = torch.tensor([-p for p in pads], dtype=torch.int32)
        return dict(q=q, k=k, v=v, qi=qi, ki=ki, kv_start=kv_start, kv_len=kv_len,
                    q_first=q_first)

    # decode: one new query per sequence against a cache of capacity S
    lens = draw_decode_lengths(gen, B, w.len_min, w.len_max, w.block)
    fill = nan if poison else 0.0
    k = torch.full((B, w.Hkv, S, w.d), fill, dtype=dt)
    v = torch.full((B, w.Hkv, S, w.d), fill, dtype=dt)
    ki = torch.full((B, S, w.di), fill, dtype=dt)
    for b, L in enumerate(lens):
        k[b, :, : L - 1] = _randn(gen, (w.Hkv, L - 1, w.d), w.std, dt)
        v[b, :, : L - 1] = _randn(gen, (w.Hkv, L - 1, w.d), w.std, dt)
        ki[b, : L - 1] = _randn(gen, (L - 1, w.di), w.std, dt)
    k_new = _randn(gen, (B, w.Hkv, w.d), w.std, dt)
    v_new = _randn(gen, (B, w.Hkv, w.d), w.std, dt)
    ki_new = _randn(gen, (B, w.di), w.std, dt)
    q = _randn(gen, (B, 1, w.Hq, w.d), w.std, dt)
    qi = _randn(gen, (B, 1, w.Hi, w.di), w.std, dt)
    kv_len = torch.tensor(lens, dtype=torch.int32)
    return dict(q=q, qi=qi, k=k, v=v, ki=ki, k_new=k_new, v_new=v_new, ki_new=ki_new,
                kv_start=torch.zeros(B, dtype=torch.int32), kv_len=kv_len,
                q_first=kv_len - 1)


def _plant_blocks(gen, w: Workload, q, k, qi, ki, pads):
    """Plant ``w.planted`` whole blocks whose keys sit near the query mean.

    Indexer keys of a planted block are the mean indexer query (over positions
    and indexer heads) plus N(0, planted_std) noise; attention keys of KV head g
    are the mean of the queries of g's head group plus the same kind of noise.
    """
    G = w.Hq // w.Hkv
    for b in range(w.batch):
        p = pads[b]
        n_blocks = (w.seq - p) // w.block
        blocks = torch.randperm(n_blocks, generator=gen)[: w.planted].tolist()
        mu_i = qi[b, p:].float().mean(dim=(0, 1))  # [di]
        mu_g = [q[b, p:, g * G:(g + 1) * G].float().mean(dim=(0, 1)) for g in range(w.Hkv)]
        for j in sorted(blocks):
            lo, hi = p + j * w.block, p + (j + 1) * w.block
            noise = torch.randn((w.block, w.di), generator=gen) * w.planted_std
            ki[b, lo:hi] = (mu_i + noise).to(ki.dtype)
            for g in range(w.Hkv):
                noise = torch.randn((w.block, w.d), generator=gen) * w.planted_std
                k[b, g, lo:hi] = (mu_g[g] + noise).to(k.dtype)


def planted_block_ids(w: Workload) -> Optional[list]:
    """Replay the generator to report which blocks were planted (diagnostics)."""
    if w.planted == 0:
        return None
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed)
    B, S = w.batch, w.seq
    if w.pad_max > 0:
        pads = [int(x) for x in torch.randint(0, w.pad_max + 1, (B,), generator=gen)]
    else:
        pads = [0] * B
    for shape in [(B, S, w.Hq, w.d), (B, w.Hkv, S, w.d), (B, w.Hkv, S, w.d),
                  (B, S, w.Hi, w.di), (B, S, w.di)]:
        torch.randn(shape, generator=gen)
    out = []
    for b in range(B):
        n_blocks = (S - pads[b]) // w.block
        blocks = torch.randperm(n_blocks, generator=gen)[: w.planted].tolist()
        out.append(sorted(blocks))
        for _ in blocks:
            torch.randn((w.block, w.di), generator=gen)
            for g in range(w.Hkv):
                torch.randn((w.block, w.d), generator=gen)
    return out


def small_variant(w: Workload, seq: int, batch: Optional[int] = None, **kw) -> Workload:
    """Same heads/indexer/block settings at a size the oracle finishes quickly."""
    fields = dict(seq=seq, name=f"{w.name}__s{seq}")
    if batch is not None:
        fields["batch"] = batch
    fields.update(kw)
    return w.replace(**fields)
