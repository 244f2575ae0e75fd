"""Every attention and scoring kernel that qsa_forward / qsa_sparse_attn can dispatch,
against the fp64 oracle on the same seeded inputs (through the C ABI):

  - the per-split decode kernel, taken when a decode batch has more than 2048
    (sequence, KV head) units;
  - the CUDA-core attention kernel on bf16 inputs, for shapes the tensor-core kernels
    do not take (head_dim 64; block size 32 at head_dim 128);
  - an fp32 decode step (CTA-per-row scoring with the decode prologue, then the
    CUDA-core attention on one row);
  - the compressed keys (k̄) a decode step writes when its token completes a block.
Tolerances are those of tests/parity_util.py (fp32 ids bit-exact, outputs 1e-4; bf16
outputs 1e-2 + 2e-2 |o|, near-tie selections only).
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_15_b200 import workloads as W
from tests.parity_util import compare
from tests.test_parity_gpu import assert_kbar_close, assert_report, run_prefill

pytestmark = pytest.mark.gpu

WL = W.WORKLOADS


def run_decode(qsa, w, inp):
    from block_sparse_long_15_b200.runner import QSADecode
    d = QSADecode(w, inp, guard=True)
    out, sel = d()
    torch.cuda.synchronize()
    assert d.status() == qsa.QSA_OK
    assert d.guards_intact(), "a kernel wrote outside out / sel"
    return out.cpu(), sel.cpu(), d


def test_decode_split_kernel_more_than_2048_units(cuda_lib):
    """1100 sequences x 2 KV heads = 2200 units: past the persistent streaming kernel's
    limit, so the decode attention runs as one CTA per (split, KV head, sequence)."""
    w = W.small_variant(WL["bf16_decode_b64_l4k_32k"], seq=1024, batch=1100, len_min=70, len_max=1000)
    assert w.batch * w.Hkv > 2048
    inp = W.make_inputs(w)
    out, sel, _ = run_decode(cuda_lib, w, inp)
    rep = compare(w, inp, out, sel, oracle.run(w, inp), decode=True)
    assert_report(rep, w, 0.05)
    assert rep.rows == w.batch


@pytest.mark.parametrize("shape", [
    dict(Hq=8, Hkv=2, d=64, Hi=4, di=64, block=64, topk=4),     # head_dim 64
    dict(Hq=16, Hkv=2, d=128, Hi=4, di=64, block=32, topk=6),   # block 32 at head_dim 128
])
def test_bf16_cuda_core_attention_full_rows(cuda_lib, shape):
    """bf16 shapes that neither tensor-core prefill kernel serves go to the CUDA-core
    kernel; every row of a left-padded batch against the oracle."""
    qsa = cuda_lib
    w = W.small_variant(WL["bf16_prefill_varlen_b8_s16384_leftpad"], seq=520, batch=2, pad_max=150,
                        **shape)
    assert qsa.qsa_attn_kernel_name(qsa.config_for(w)) == "simt"
    inp = W.make_inputs(w)
    out, sel, p = run_prefill(qsa, w, inp)
    orc = oracle.run(w, inp, want_kbar=True)
    rep = compare(w, inp, out, sel, orc)
    assert_report(rep, w)
    for b in range(w.batch):
        assert_kbar_close(p.t["kbar_cache"][b, : int(inp["kv_len"][b]) // w.block], orc["kbar"][b])


def test_bf16_decode_step_on_cuda_core_attention(cuda_lib):
    """A bf16 decode step at a shape the split-KV decode kernel does not serve (head_dim
    64): qsa_forward runs the CUDA-core attention kernel on the one query row."""
    qsa = cuda_lib
    w = W.small_variant(WL["bf16_decode_b64_l4k_32k"], seq=2048, batch=5, len_min=100, len_max=2000,
                        Hq=8, Hkv=2, d=64)
    assert qsa.qsa_attn_kernel_name(qsa.config_for(w), qsa.QSA_DECODE) == "simt"
    inp = W.make_inputs(w)
    out, sel, _ = run_decode(qsa, w, inp)
    rep = compare(w, inp, out, sel, oracle.run(w, inp), decode=True)
    assert_report(rep, w, 0.05)


def test_fp32_decode_step(cuda_lib):
    """fp32 decode: CTA-per-row scoring fused with the decode prologue, then the
    CUDA-core attention on one row; selected ids bit-exact, outputs within 1e-4."""
    qsa = cuda_lib
    base = WL["tiny_fp32_prefill_s256"]
    w = base.replace(name="tiny_fp32_decode", mode="decode", batch=6, seq=640, len_min=40, len_max=630)
    assert qsa.qsa_attn_kernel_name(qsa.config_for(w), qsa.QSA_DECODE) == "simt"
    inp = W.make_inputs(w)
    out, sel, _ = run_decode(qsa, w, inp)
    rep = compare(w, inp, out, sel, oracle.run(w, inp), decode=True)
    assert_report(rep, w, 0.0)
    assert rep.sel_exact == rep.rows == w.batch


def test_decode_completed_block_kbar_matches_oracle(cuda_lib):
    """A decode step whose token completes a block compresses it: the indexer state's
    new k̄ row against the oracle's fp64 block mean (over the cached keys and the new
    indexer key)."""
    qsa = cuda_lib
    w = W.small_variant(WL["bf16_decode_b64_l4k_32k"], seq=4096, batch=4, len_min=600, len_max=4000)
    inp = W.make_inputs(w)
    # make every length a multiple of the block size: this step's token completes a block
    L = (inp["kv_len"] // w.block) * w.block
    inp["kv_len"] = L.to(torch.int32)
    inp["q_first"] = (L - 1).to(torch.int32)
    for b in range(w.batch):  # cache rows 0 .. L-2 drawn, the rest poisoned
        inp["k"][b, :, int(L[b]) - 1:] = float("nan")
        inp["v"][b, :, int(L[b]) - 1:] = float("nan")
        inp["ki"][b, int(L[b]) - 1:] = float("nan")
    _, _, d = run_decode(qsa, w, inp)
    orc = oracle.run(w, inp, decode=True, want_kbar=True)
    assert torch.equal(d.t["kbar_blocks"].cpu(), (L // w.block).to(torch.int32))
    for b in range(w.batch):
        n_blk = int(L[b]) // w.block
        assert_kbar_close(d.t["kbar_cache"][b, :n_blk], orc["kbar"][b])
