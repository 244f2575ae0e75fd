"""Input projections + RoPE (qsa_project) through the C ABI against the fp64 oracle.

Hidden size 2048 (Qwen4ExpTextConfig's default), the heads of the 8K prefill and of
the varlen workload, weights N(0, 1) / sqrt(2048) and hidden states N(0, 1), seeded,
rounded to bf16 once. Every output element within the bf16 tolerance of the parity
tests, |g - o| <= 1e-2 + 2e-2 |o| (the GPU accumulates in fp32, forms the rotary angle
in fp32 and rounds the result to bf16 once)."""
import types

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_15_b200 import workloads as W

pytestmark = pytest.mark.gpu

ATOL, RTOL = 1e-2, 2e-2


def _inputs(w, n_rows, hidden, seed):
    g = torch.Generator().manual_seed(seed)
    n_out = w.Hq * w.d + 2 * w.Hkv * w.d + w.Hi * w.di + w.di
    x = torch.randn(n_rows, hidden, generator=g).to(torch.bfloat16)
    wt = (torch.randn(n_out, hidden, generator=g) / hidden ** 0.5).to(torch.bfloat16)
    return x, wt


def _check(got, want, name):
    g = got.double().cpu().numpy()
    assert np.all(np.isfinite(g)), name
    exc = np.abs(g - want) - (ATOL + RTOL * np.abs(want))
    assert exc.max() <= 0, f"{name}: max excess {exc.max():.3e}, max err {np.abs(g - want).max():.3e}"


def run_project(qsa, w, x, wt, q_first, batch, n_tok, pc, kv_cap=None, kv_row0=0):
    dev = "cuda"
    kv_cap = kv_cap or n_tok
    bf = torch.bfloat16
    out = dict(q=torch.full((batch, n_tok, w.Hq, w.d), float("nan"), dtype=bf, device=dev),
               qi=torch.full((batch, n_tok, w.Hi, w.di), float("nan"), dtype=bf, device=dev),
               k=torch.full((batch, w.Hkv, kv_cap, w.d), float("nan"), dtype=bf, device=dev),
               v=torch.full((batch, w.Hkv, kv_cap, w.d), float("nan"), dtype=bf, device=dev),
               ki=torch.full((batch, kv_cap, w.di), float("nan"), dtype=bf, device=dev))
    cfg = qsa.config_for(w)
    ws = qsa.qsa_project(cfg, pc, x.view(batch, n_tok, -1).cuda(), wt.cuda(), q_first.cuda(), out["q"],
                         out["qi"], out["k"], out["v"], out["ki"], kv_row0)
    torch.cuda.synchronize()
    assert qsa.qsa_read_device_status(ws) == qsa.QSA_OK
    return out


@pytest.mark.parametrize("name,rd,rd_idx,theta", [
    ("bf16_prefill_s8192", 128, 64, 1e6),
    ("bf16_prefill_s8192", 64, 0, 1e4),            # partial rotary, indexer heads not rotated
    ("bf16_prefill_varlen_b8_s16384_leftpad", 128, 32, 1e7),
])
def test_projection_rope_all_rows(cuda_lib, name, rd, rd_idx, theta):
    qsa = cuda_lib
    w = W.WORKLOADS[name]
    batch, n_tok, hidden = 2, 333, 2048  # ragged: 666 rows over 6 row tiles
    x, wt = _inputs(w, batch * n_tok, hidden, 11)
    q_first = torch.tensor([-40, 0], dtype=torch.int32)  # row r of sequence b sits at q_first[b] + r
    pc = qsa.qsa_proj_config_t(hidden, theta, rd, rd_idx)
    out = run_project(qsa, w, x, wt, q_first, batch, n_tok, pc)
    pos = np.concatenate([int(q_first[b]) + np.arange(n_tok) for b in range(batch)])
    opc = types.SimpleNamespace(Hq=w.Hq, Hkv=w.Hkv, d=w.d, Hi=w.Hi, di=w.di, rope_theta=theta, rd_attn=rd,
                                rd_idx=rd_idx)
    ref = oracle.project_rope(opc, x, wt, pos)
    _check(out["q"].reshape(-1, w.Hq, w.d), ref["q"], "q")
    _check(out["qi"].reshape(-1, w.Hi, w.di), ref["qi"], "qi")
    _check(out["k"].transpose(1, 2).reshape(-1, w.Hkv, w.d), ref["k"], "k")
    _check(out["v"].transpose(1, 2).reshape(-1, w.Hkv, w.d), ref["v"], "v")
    _check(out["ki"].reshape(-1, w.di), ref["ki"], "ki")


def test_projection_long_positions_sampled(cuda_lib):
    """The 8K prefill's full size (8192 rows x 2880 outputs) at positions near 60000
    (the largest rotary angles the long workloads reach), checked on sampled rows."""
    qsa = cuda_lib
    w = W.WORKLOADS["bf16_prefill_s8192"]
    n_tok, hidden, theta = 8192, 2048, 1e6
    x, wt = _inputs(w, n_tok, hidden, 12)
    q_first = torch.tensor([57000], dtype=torch.int32)
    pc = qsa.qsa_proj_config_t(hidden, theta, 128, 64)
    out = run_project(qsa, w, x, wt, q_first, 1, n_tok, pc)
    rows = sorted(set(np.random.default_rng(5).integers(0, n_tok, 200).tolist()) | {0, 127, 128, 8191})
    opc = types.SimpleNamespace(Hq=w.Hq, Hkv=w.Hkv, d=w.d, Hi=w.Hi, di=w.di, rope_theta=theta, rd_attn=128,
                                rd_idx=64)
    ref = oracle.project_rope(opc, x[rows], wt, 57000 + np.array(rows))
    _check(out["q"][0, rows], ref["q"], "q")
    _check(out["qi"][0, rows], ref["qi"], "qi")
    _check(out["k"][0][:, rows].transpose(0, 1), ref["k"], "k")
    _check(out["v"][0][:, rows].transpose(0, 1), ref["v"], "v")
    _check(out["ki"][0, rows], ref["ki"], "ki")


def test_projection_decode_step_into_new_token_buffers(cuda_lib):
    """A decode step: one token per sequence at position kv_len - 1, k / v / ki into the
    [batch][Hkv][d] and [batch][di] buffers qsa_forward appends."""
    qsa = cuda_lib
    w = W.WORKLOADS["bf16_decode_b64_l4k_32k"]
    batch, hidden, theta = 64, 2048, 1e6
    x, wt = _inputs(w, batch, hidden, 13)
    kv_len = torch.randint(4097, 32768, (batch,), generator=torch.Generator().manual_seed(2)).to(torch.int32)
    pc = qsa.qsa_proj_config_t(hidden, theta, 128, 64)
    out = run_project(qsa, w, x, wt, kv_len - 1, batch, 1, pc, kv_cap=1)
    opc = types.SimpleNamespace(Hq=w.Hq, Hkv=w.Hkv, d=w.d, Hi=w.Hi, di=w.di, rope_theta=theta, rd_attn=128,
                                rd_idx=64)
    ref = oracle.project_rope(opc, x, wt, (kv_len - 1).numpy())
    _check(out["q"][:, 0], ref["q"], "q")
    _check(out["k"][:, :, 0], ref["k"], "k")
    _check(out["v"][:, :, 0], ref["v"], "v")
    _check(out["qi"][:, 0], ref["qi"], "qi")
    _check(out["ki"][:, 0], ref["ki"], "ki")
