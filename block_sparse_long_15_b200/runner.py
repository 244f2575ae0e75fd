"""Device-side buffers and calls for the QSA path through the C ABI.

QSAPrefill / QSADecode own the caller-side device memory that the library
expects (caches, indexer state, outputs, workspace) as torch CUDA tensors and
call ``qsa_forward``. All arithmetic runs in libqsa.so.
"""
from __future__ import annotations

from typing import Dict

import torch

from . import qsa


def to_device(inp: Dict[str, torch.Tensor], device="cuda") -> Dict[str, torch.Tensor]:
    return {k: v.to(device, non_blocking=True).contiguous() for k, v in inp.items()}


class QSAPrefill:
    """One prefill call: compress every complete block, score, select, attend."""

    def __init__(self, w, inp: Dict[str, torch.Tensor], device="cuda"):
        self.cfg = qsa.config_for(w)
        self.k = qsa.qsa_topk_blocks(self.cfg)
        g = to_device(inp, device)
        B, n_q = g["q"].shape[0], g["q"].shape[1]
        kv_cap = g["k"].shape[2]
        self.t = dict(q=g["q"], qi=g["qi"], k_cache=g["k"], v_cache=g["v"], ki_cache=g["ki"],
                      kbar_cache=torch.zeros(B, kv_cap // w.block, w.di, dtype=torch.float32, device=device),
                      kbar_blocks=torch.zeros(B, dtype=torch.int32, device=device),
                      kv_start=g["kv_start"], kv_len=g["kv_len"], q_first=g["q_first"],
                      sel=torch.empty(B, n_q, self.k, dtype=torch.int32, device=device),
                      out=torch.empty_like(g["q"]))
        self.ws = qsa.alloc_workspace(self.cfg, qsa.QSA_PREFILL, B, n_q, kv_cap, device)

    def __call__(self, stream=None):
        qsa.qsa_forward(self.cfg, qsa.QSA_PREFILL, self.t, self.ws, stream)
        return self.t["out"], self.t["sel"]

    def status(self) -> int:
        return qsa.qsa_read_device_status(self.ws)


class QSADecode:
    """One decode step per sequence against caches holding kv_len - 1 tokens.

    The indexer state (k̄ for the complete blocks already in the cache) is built
    once by qsa_compress_blocks; each call appends the new token and runs the path.
    Calling again with the same kv_len re-appends the same token (the benchmark's
    steady-state step) -- reset_state() rewinds kbar_blocks for that.
    """

    def __init__(self, w, inp: Dict[str, torch.Tensor], device="cuda"):
        self.cfg = qsa.config_for(w)
        self.k = qsa.qsa_topk_blocks(self.cfg)
        self.w = w
        g = to_device(inp, device)
        B = g["q"].shape[0]
        kv_cap = g["k"].shape[2]
        self.t = dict(q=g["q"], qi=g["qi"], k_cache=g["k"], v_cache=g["v"], ki_cache=g["ki"],
                      kbar_cache=torch.zeros(B, kv_cap // w.block, w.di, dtype=torch.float32, device=device),
                      kbar_blocks=torch.zeros(B, dtype=torch.int32, device=device),
                      k_new=g["k_new"], v_new=g["v_new"], ki_new=g["ki_new"],
                      kv_start=g["kv_start"], kv_len=g["kv_len"],
                      sel=torch.empty(B, 1, self.k, dtype=torch.int32, device=device),
                      out=torch.empty_like(g["q"]))
        self.prev_len = (g["kv_len"] - 1).contiguous()
        # indexer state for the tokens already cached: blocks [0, (L-1)/B)
        qsa.qsa_compress_blocks(self.cfg, self.t["ki_cache"], self.t["kv_start"], self.prev_len,
                                self.t["kbar_cache"])
        self.ws = qsa.alloc_workspace(self.cfg, qsa.QSA_DECODE, B, 1, kv_cap, device)
        self.reset_state()

    def reset_state(self):
        self.t["kbar_blocks"].copy_(torch.div(self.prev_len, self.w.block, rounding_mode="floor"))

    def __call__(self, stream=None):
        qsa.qsa_forward(self.cfg, qsa.QSA_DECODE, self.t, self.ws, stream)
        return self.t["out"], self.t["sel"]

    def status(self) -> int:
        return qsa.qsa_read_device_status(self.ws)


class QSADecodeOffload(QSADecode):
    """QSADecode with the attention K/V cache in page-locked host memory: each call
    appends the new token to the host cache, selects on the device and copies only
    the attended blocks to the device staging buffer (qsa_decode_offload)."""

    def __init__(self, w, inp: Dict[str, torch.Tensor], device="cuda"):
        super().__init__(w, inp, device)
        self.t["k_cache"] = self.t["k_cache"].cpu().pin_memory()
        self.t["v_cache"] = self.t["v_cache"].cpu().pin_memory()
        self.staging = qsa.alloc_offload_staging(self.cfg, self.t["q"].shape[0], device)

    def __call__(self, stream=None):
        qsa.qsa_decode_offload(self.cfg, self.t, self.staging, self.ws, stream)
        return self.t["out"], self.t["sel"]
