"""CUDA path vs the fp64 oracle on identical seeded inputs, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_15_b200 import workloads as W
from tests.parity_util import compare, sample_rows

pytestmark = pytest.mark.gpu

WL = W.WORKLOADS


def run_prefill(qsa, w, inp):
    """qsa_forward(PREFILL) with guard bands around out and sel, checked after the call."""
    from block_sparse_long_15_b200.runner import QSAPrefill
    p = QSAPrefill(w, inp, guard=True)
    out, sel = p()
    torch.cuda.synchronize()
    assert p.status() == qsa.QSA_OK
    assert p.guards_intact(), "a kernel wrote outside out / sel"
    return out.cpu(), sel.cpu(), p


def oracle_rows(w, inp, n_random, seed):
    return {b: sample_rows(inp["q"].shape[1], int(inp["q_first"][b]), int(inp["kv_len"][b]), w.block,
                           n_random, seed + b) for b in range(w.batch)}


def assert_kbar_close(g, o):
    """Compressed keys: the kernel's fp32 block means against the oracle's fp64 ones,
    |g - o| <= 1e-6 + 1e-5 |o| (an fp32 sum of B bf16/fp32 keys in key order, then a
    division by B, is within a few fp32 ulps of the exact mean)."""
    g = g.double().cpu().numpy()
    assert g.shape == o.shape, (g.shape, o.shape)
    err = np.abs(g - o) - (1e-6 + 1e-5 * np.abs(o))
    assert err.max() <= 0, f"kbar off by {np.abs(g - o).max():.3e}"


def assert_report(rep, w, max_near_tie_frac=0.01):
    print(w.name, rep)
    assert rep.ok(), str(rep)
    assert rep.near_tie_rows <= max(1, max_near_tie_frac * rep.rows), str(rep)
    assert rep.near_tie_checked == rep.near_tie_rows, str(rep)


# ----------------------------------------------------------------------------- fp32 tiny
def test_tiny_fp32_full(cuda_lib):
    w = WL["tiny_fp32_prefill_s256"]
    inp = W.make_inputs(w)
    out, sel, p = run_prefill(cuda_lib, w, inp)
    orc = oracle.run(w, inp, want_kbar=True)
    rep = compare(w, inp, out, sel, orc)
    assert_report(rep, w, 0.0)
    assert rep.sel_exact == rep.rows == 256
    assert_kbar_close(p.t["kbar_cache"][0, : 256 // w.block], orc["kbar"][0])


# ----------------------------------------------------------------------------- bf16 prefill
@pytest.mark.parametrize("seq", [64, 1000, 2112])
def test_bf16_prefill_small_full_rows(cuda_lib, seq):
    """Every row at sizes spanning several tiles and a ragged tail."""
    w = W.small_variant(WL["bf16_prefill_s8192"], seq=seq)
    inp = W.make_inputs(w)
    out, sel, p = run_prefill(cuda_lib, w, inp)
    orc = oracle.run(w, inp, want_kbar=True)
    rep = compare(w, inp, out, sel, orc)
    assert_report(rep, w)
    assert_kbar_close(p.t["kbar_cache"][0, : seq // w.block], orc["kbar"][0])


def test_bf16_prefill_s8192_sampled(cuda_lib):
    w = WL["bf16_prefill_s8192"]
    inp = W.make_inputs(w)
    out, sel, _ = run_prefill(cuda_lib, w, inp)
    rep = compare(w, inp, out, sel, oracle.run(w, inp, rows=oracle_rows(w, inp, 256, 100)))
    assert_report(rep, w)


def test_long_prefill_s65536_sampled(cuda_lib):
    w = WL["bf16_prefill_s65536_planted"]
    inp = W.make_inputs(w)
    out, sel, _ = run_prefill(cuda_lib, w, inp)
    rep = compare(w, inp, out, sel, oracle.run(w, inp, rows=oracle_rows(w, inp, 64, 200)))
    assert_report(rep, w)


def test_varlen_leftpad_full_size_sampled(cuda_lib):
    w = WL["bf16_prefill_varlen_b8_s16384_leftpad"]
    inp = W.make_inputs(w)
    out, sel, _ = run_prefill(cuda_lib, w, inp)
    rows = oracle_rows(w, inp, 24, 300)
    rep = compare(w, inp, out, sel, oracle.run(w, inp, rows=rows))
    assert_report(rep, w)
    # padding rows: zero output, -1 selection
    for b in range(w.batch):
        p = int(inp["kv_start"][b])
        assert torch.all(out[b, :p] == 0) and torch.all(sel[b, :p] == -1)


def test_varlen_leftpad_small_full_rows(cuda_lib):
    w = W.small_variant(WL["bf16_prefill_varlen_b8_s16384_leftpad"], seq=700, batch=3, pad_max=300)
    inp = W.make_inputs(w)
    out, sel, p = run_prefill(cuda_lib, w, inp)
    orc = oracle.run(w, inp, want_kbar=True)
    rep = compare(w, inp, out, sel, orc)
    assert_report(rep, w)
    for b in range(w.batch):  # k̄ rows count from each sequence's first real token
        n_blk = int(inp["kv_len"][b]) // w.block
        assert_kbar_close(p.t["kbar_cache"][b, :n_blk], orc["kbar"][b])


# ----------------------------------------------------------------------------- edge cases
@pytest.mark.parametrize("seq,topk", [(40, 32), (64, 1), (192, 32), (130, 2)])
def test_prefill_edges(cuda_lib, seq, topk):
    """Shorter than a block, exactly one block, budget covering everything (dense), tiny budget."""
    w = W.small_variant(WL["bf16_prefill_s8192"], seq=seq, topk=topk)
    inp = W.make_inputs(w)
    out, sel, _ = run_prefill(cuda_lib, w, inp)
    rep = compare(w, inp, out, sel, oracle.run(w, inp))
    assert_report(rep, w)


def test_empty_sequence_in_batch(cuda_lib):
    """A sequence that is all padding produces zeros and -1 everywhere."""
    w = W.small_variant(WL["bf16_prefill_s8192"], seq=256, batch=2)
    inp = W.make_inputs(w)
    inp["kv_start"][1] = 256
    inp["kv_len"][1] = 0
    inp["q_first"][1] = -256
    out, sel, _ = run_prefill(cuda_lib, w, inp)
    assert torch.all(out[1] == 0) and torch.all(sel[1] == -1)
    rep = compare(w, inp, out, sel, oracle.run(w, inp, rows={0: list(range(256))}))
    assert_report(rep, w)


# ----------------------------------------------------------------------------- stage API
def test_stage_api_equals_forward(cuda_lib):
    qsa = cuda_lib
    w = W.small_variant(WL["bf16_prefill_varlen_b8_s16384_leftpad"], seq=640, batch=2, pad_max=200)
    inp = W.make_inputs(w)
    out_f, sel_f, p = run_prefill(qsa, w, inp)
    g = {k: v.cuda() for k, v in inp.items()}
    cfg = qsa.config_for(w)
    kbar = torch.zeros(w.batch, w.seq // w.block, w.di, dtype=torch.float32, device="cuda")
    qsa.qsa_compress_blocks(cfg, g["ki"], g["kv_start"], g["kv_len"], kbar)
    # k̄ matches what qsa_forward left in the indexer state
    assert torch.equal(kbar, p.t["kbar_cache"])
    ws = qsa.alloc_workspace(cfg, qsa.QSA_PREFILL, w.batch, w.seq, w.seq)
    # scoring reads k̄ rows relative to each sequence's first token
    sel = torch.empty(w.batch, w.seq, w.topk, dtype=torch.int32, device="cuda")
    qsa.qsa_index_score_topk(cfg, g["qi"], kbar, g["kv_len"], g["q_first"], w.seq, sel, ws)
    out = torch.empty_like(g["q"])
    qsa.qsa_sparse_attn(cfg, g["q"], g["k"], g["v"], sel, g["kv_start"], g["kv_len"], g["q_first"], out, ws)
    torch.cuda.synchronize()
    assert torch.equal(sel.cpu(), sel_f)
    assert torch.equal(out.cpu(), out_f)
    assert qsa.qsa_read_device_status(ws) == qsa.QSA_OK


# ----------------------------------------------------------------------------- decode
def test_decode_b64_full(cuda_lib):
    from block_sparse_long_15_b200.runner import QSADecode
    w = WL["bf16_decode_b64_l4k_32k"]
    inp = W.make_inputs(w)
    d = QSADecode(w, inp, guard=True)
    out, sel = d()
    torch.cuda.synchronize()
    assert d.status() == cuda_lib.QSA_OK
    assert d.guards_intact()
    orc = oracle.run(w, inp)
    rep = compare(w, inp, out.cpu(), sel.cpu(), orc, decode=True)
    assert_report(rep, w, 0.05)
    # the appended token landed in the cache
    L = inp["kv_len"]
    for b in (0, 17, 63):
        assert torch.equal(d.t["k_cache"][b, :, L[b] - 1].cpu(), inp["k_new"][b])
        assert torch.equal(d.t["ki_cache"][b, L[b] - 1].cpu(), inp["ki_new"][b])


def test_decode_steps_across_block_boundary_match_prefill_rows(cuda_lib):
    """Successive decode steps (one crossing a block boundary, so a block gets
    compressed) equal the prefill rows of the same sequence."""
    from block_sparse_long_15_b200 import qsa
    w = W.small_variant(WL["bf16_prefill_s8192"], seq=400, batch=2, topk=2)
    inp = W.make_inputs(w)
    orc = oracle.run(w, inp)
    dev = {k: v.cuda() for k, v in inp.items()}
    cfg = qsa.config_for(w)
    L0 = 250  # caches hold 249 tokens; steps append tokens 249 .. 260 (block 3 completes at 256)
    kv_cap = w.seq
    k_cache = dev["k"].clone()
    v_cache = dev["v"].clone()
    ki_cache = dev["ki"].clone()
    k_cache[:, :, L0 - 1:] = float("nan")
    v_cache[:, :, L0 - 1:] = float("nan")
    ki_cache[:, L0 - 1:] = float("nan")
    kbar = torch.zeros(w.batch, kv_cap // w.block, w.di, dtype=torch.float32, device="cuda")
    prev = torch.full((w.batch,), L0 - 1, dtype=torch.int32, device="cuda")
    zero = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
    qsa.qsa_compress_blocks(cfg, ki_cache, zero, prev, kbar)
    blocks = torch.div(prev, w.block, rounding_mode="floor").to(torch.int32)
    ws = qsa.alloc_workspace(cfg, qsa.QSA_DECODE, w.batch, 1, kv_cap)
    for L in range(L0, L0 + 12):
        t = dict(q=dev["q"][:, L - 1:L].contiguous(), qi=dev["qi"][:, L - 1:L].contiguous(),
                 k_cache=k_cache, v_cache=v_cache, ki_cache=ki_cache, kbar_cache=kbar, kbar_blocks=blocks,
                 k_new=dev["k"][:, :, L - 1].contiguous(), v_new=dev["v"][:, :, L - 1].contiguous(),
                 ki_new=dev["ki"][:, L - 1].contiguous(), kv_start=zero,
                 kv_len=torch.full((w.batch,), L, dtype=torch.int32, device="cuda"),
                 sel=torch.empty(w.batch, 1, w.topk, dtype=torch.int32, device="cuda"),
                 out=torch.empty(w.batch, 1, w.Hq, w.d, dtype=torch.bfloat16, device="cuda"))
        qsa.qsa_forward(cfg, qsa.QSA_DECODE, t, ws)
        torch.cuda.synchronize()
        assert qsa.qsa_read_device_status(ws) == qsa.QSA_OK
        assert int(blocks[0]) == L // w.block
        for b in range(w.batch):
            assert t["sel"][b, 0].cpu().tolist() == orc["sel"][b][L - 1].tolist(), (L, b)
            err = (t["out"][b, 0].double().cpu().numpy() - orc["o"][b][L - 1])
            assert np.all(np.abs(err) <= 1e-2 + 2e-2 * np.abs(orc["o"][b][L - 1])), (L, b)
    # the compressed block matches a fresh compression of the same keys
    ref = torch.zeros_like(kbar)
    qsa.qsa_compress_blocks(cfg, ki_cache, zero, torch.full_like(prev, L0 + 11), ref)
    torch.cuda.synchronize()
    assert torch.equal(ref[:, :(L0 + 11) // w.block], kbar[:, :(L0 + 11) // w.block])


def test_decode_crop_is_rejected(cuda_lib):
    """Cache cropping is unsupported with QSA: a decode whose length went backwards
    records QSA_ERR_UNSUPPORTED and leaves the cache and indexer state untouched."""
    from block_sparse_long_15_b200.runner import QSADecode
    qsa = cuda_lib
    w = W.small_variant(WL["bf16_decode_b64_l4k_32k"], seq=8192, batch=4, len_min=1000, len_max=8000)
    inp = W.make_inputs(w)
    d = QSADecode(w, inp)
    d()
    torch.cuda.synchronize()
    assert d.status() == qsa.QSA_OK
    # the state advanced only if a block completed; now shrink the length by two blocks
    d.t["kv_len"][0] -= 2 * w.block
    before_k = d.t["k_cache"].clone()
    before_blocks = d.t["kbar_blocks"].clone()
    d()
    torch.cuda.synchronize()
    assert d.status() == qsa.QSA_ERR_UNSUPPORTED
    assert torch.equal(d.t["kbar_blocks"][0], before_blocks[0])
    # compare bit patterns: the unused cache rows hold NaN poison
    assert torch.equal(d.t["k_cache"][0].view(torch.int16), before_k[0].view(torch.int16))


def test_device_check_on_bad_lengths(cuda_lib):
    qsa = cuda_lib
    w = W.small_variant(WL["bf16_prefill_s8192"], seq=256)
    inp = W.make_inputs(w)
    inp["kv_len"][0] = 300  # beyond capacity
    from block_sparse_long_15_b200.runner import QSAPrefill
    p = QSAPrefill(w, inp)
    p()
    torch.cuda.synchronize()
    assert p.status() == qsa.QSA_ERR_DEVICE_CHECK
    assert p.status() == qsa.QSA_OK  # reading clears it
