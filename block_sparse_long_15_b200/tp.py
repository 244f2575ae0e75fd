"""Head-sharded tensor parallelism of the QSA prefill path ("Qwen4-Exp" Usage tips:
tp_plan="auto" shards QSA, and the QSA projection dims must be divisible by the TP
size).

Reading taken: a TP group of size `tp` splits the query heads, the KV heads and the
indexer query heads into `tp` equal consecutive shards; rank r holds shard r of each.
The single indexer key head (and so the compressed keys) is replicated. Because the
block score is a sum over indexer heads of max(0, qi_h . kbar_j), rank r's partial
score over its indexer heads, summed over ranks, is the full score: the ranks
all-reduce the [batch][n_q][n_blocks] fp32 score matrix, every rank then selects the
same blocks from it, and attends its own query / KV heads with that selection.

Everything numeric runs in libqsa.so (qsa_compress_blocks, qsa_index_scores,
qsa_select_topk, qsa_sparse_attn); the all-reduce is the caller's collective
(torch.distributed over NCCL by default). This module only slices and sequences.
"""
from __future__ import annotations

from typing import Callable, Dict, Optional

import torch

from . import qsa


def check_divisible(w, tp: int):
    """The pages' rule: projection dims (here the head counts) divisible by the TP size."""
    for name, n in (("num_attention_heads", w.Hq), ("num_key_value_heads", w.Hkv),
                    ("indexer_n_heads", w.Hi)):
        if n % tp != 0:
            raise ValueError(f"{name}={n} is not divisible by the TP size {tp}")


def shard_workload(w, tp: int):
    """The workload description of one rank's shard (heads divided by tp)."""
    check_divisible(w, tp)
    return w.replace(Hq=w.Hq // tp, Hkv=w.Hkv // tp, Hi=w.Hi // tp, name=f"{w.name}__tp{tp}")


def shard_inputs(inp: Dict[str, torch.Tensor], w, tp: int, rank: int) -> Dict[str, torch.Tensor]:
    """Rank `rank`'s slices: query heads [r Hq/tp, (r+1) Hq/tp), the KV heads and
    indexer query heads likewise; the indexer keys and lengths are replicated."""
    check_divisible(w, tp)
    hq, hkv, hi = w.Hq // tp, w.Hkv // tp, w.Hi // tp
    out = dict(inp)
    out["q"] = inp["q"][:, :, rank * hq:(rank + 1) * hq].contiguous()
    out["qi"] = inp["qi"][:, :, rank * hi:(rank + 1) * hi].contiguous()
    out["k"] = inp["k"][:, rank * hkv:(rank + 1) * hkv].contiguous()
    out["v"] = inp["v"][:, rank * hkv:(rank + 1) * hkv].contiguous()
    return out


def gather_heads(outs, dim: int = 2) -> torch.Tensor:
    """Concatenate the ranks' outputs [batch][n_q][Hq/tp][d] along the head axis."""
    return torch.cat(list(outs), dim=dim)


def _dist_all_reduce(t: torch.Tensor, group=None):
    import torch.distributed as dist
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)


class QSAPrefillTP:
    """One rank of a head-sharded prefill.

    partial_scores() -> this rank's partial score matrix (qsa_index_scores);
    finish(scores)   -> selection from the reduced scores (qsa_select_topk) and the
                        attention of this rank's heads (qsa_sparse_attn);
    __call__()       -> both, with the all-reduce in between (`all_reduce`, default
                        torch.distributed SUM over `group`).
    The compressed keys come from the replicated indexer keys (qsa_compress_blocks),
    so every rank holds the same k̄.
    """

    def __init__(self, w, inp: Dict[str, torch.Tensor], tp: int, rank: int, device="cuda",
                 all_reduce: Optional[Callable[[torch.Tensor], None]] = None, group=None):
        self.w_full, self.tp, self.rank = w, tp, rank
        self.w = shard_workload(w, tp)
        self.cfg = qsa.config_for(self.w)
        self.k = qsa.qsa_topk_blocks(self.cfg)
        s = shard_inputs(inp, w, tp, rank)
        g = {k: v.to(device).contiguous() for k, v in s.items()}
        B, n_q = g["q"].shape[0], g["q"].shape[1]
        self.kv_cap = g["k"].shape[2]
        nb = self.kv_cap // w.block
        self.g = g
        self.kbar = torch.zeros(B, nb, w.di, dtype=torch.float32, device=device)
        self.scores = torch.zeros(B, n_q, nb, dtype=torch.float32, device=device)
        self.sel = torch.empty(B, n_q, self.k, dtype=torch.int32, device=device)
        self.out = torch.empty_like(g["q"])
        self.ws = qsa.alloc_workspace(self.cfg, qsa.QSA_PREFILL, B, n_q, self.kv_cap, device)
        self.all_reduce = all_reduce or (lambda t: _dist_all_reduce(t, group))

    def partial_scores(self, stream=None) -> torch.Tensor:
        g = self.g
        qsa.qsa_compress_blocks(self.cfg, g["ki"], g["kv_start"], g["kv_len"], self.kbar, stream=stream)
        qsa.qsa_index_scores(self.cfg, g["qi"], self.kbar, g["kv_len"], g["q_first"], self.kv_cap, self.scores,
                             self.ws, stream)
        return self.scores

    def finish(self, scores: torch.Tensor, stream=None):
        g = self.g
        qsa.qsa_select_topk(self.cfg, scores, g["kv_len"], g["q_first"], self.kv_cap, self.sel, self.ws, stream)
        qsa.qsa_sparse_attn(self.cfg, g["q"], g["k"], g["v"], self.sel, g["kv_start"], g["kv_len"], g["q_first"],
                            self.out, self.ws, stream)
        return self.out, self.sel

    def __call__(self, stream=None):
        s = self.partial_scores(stream)
        self.all_reduce(s)
        return self.finish(s, stream)

    def status(self) -> int:
        return qsa.qsa_read_device_status(self.ws)
