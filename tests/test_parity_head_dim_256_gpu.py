"""head_dim 256 (the Qwen4ExpTextConfig default) against the fp64 oracle.

Prefill goes to the one-tile tcgen05 kernel (O takes 256 TMEM columns); a decode
step with head_dim 256 takes the same kernel with one query row per tile.
"""
import pytest
import torch

import oracle
from block_sparse_long_15_b200 import workloads as W
from tests.parity_util import compare
from tests.test_parity_gpu import assert_report, run_prefill

pytestmark = pytest.mark.gpu

WL = W.WORKLOADS


def test_kernel_name_head_dim_256(cuda_lib):
    qsa = cuda_lib
    w = W.small_variant(WL["bf16_prefill_s8192"], seq=256, d=256)
    assert qsa.qsa_attn_kernel_name(qsa.config_for(w)) == "tcgen05 one-tile"


@pytest.mark.parametrize("seq", [64, 1000, 2112])
def test_head_dim_256_prefill_full_rows(cuda_lib, seq):
    """Every row, over several tiles and a ragged tail (GQA 16/2, block 64)."""
    w = W.small_variant(WL["bf16_prefill_s8192"], seq=seq, d=256)
    inp = W.make_inputs(w)
    out, sel, _ = run_prefill(cuda_lib, w, inp)
    rep = compare(w, inp, out, sel, oracle.run(w, inp))
    assert_report(rep, w)


def test_head_dim_256_varlen_leftpad_full_rows(cuda_lib):
    """Left padding (NaN in the padded rows), GQA 32/4, block 128 (two chunks per block)."""
    w = W.small_variant(WL["bf16_prefill_varlen_b8_s16384_leftpad"], seq=900, batch=3, pad_max=300, d=256)
    inp = W.make_inputs(w)
    out, sel, _ = run_prefill(cuda_lib, w, inp)
    rep = compare(w, inp, out, sel, oracle.run(w, inp))
    assert_report(rep, w)
    for b in range(w.batch):
        p = int(inp["kv_start"][b])
        assert torch.all(out[b, :p] == 0)


@pytest.mark.parametrize("seq,topk", [(40, 32), (192, 32), (130, 2)])
def test_head_dim_256_prefill_edges(cuda_lib, seq, topk):
    """Shorter than a block, budget covering everything, tiny budget."""
    w = W.small_variant(WL["bf16_prefill_s8192"], seq=seq, topk=topk, d=256)
    inp = W.make_inputs(w)
    out, sel, _ = run_prefill(cuda_lib, w, inp)
    rep = compare(w, inp, out, sel, oracle.run(w, inp))
    assert_report(rep, w)


def test_head_dim_256_decode(cuda_lib):
    from block_sparse_long_15_b200.runner import QSADecode
    w = W.small_variant(WL["bf16_decode_b64_l4k_32k"], seq=4096, batch=6, len_min=300, len_max=4000, d=256)
    inp = W.make_inputs(w)
    d = QSADecode(w, inp)
    out, sel = d()
    torch.cuda.synchronize()
    assert d.status() == cuda_lib.QSA_OK
    rep = compare(w, inp, out.cpu(), sel.cpu(), oracle.run(w, inp), decode=True)
    assert_report(rep, w, 0.2)
