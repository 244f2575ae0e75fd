"""Query positions and cache offsets the other parity tests do not reach.

- Chunked prefill: the queries are the last rows of a longer cache (q_first > 0),
  as when a prompt is prefilled in pieces.
- Decode of left-padded sequences: each sequence starts at kv_start > 0 in its cache.
- Decode with a block size and a head grouping that the streaming decode kernel does
  not serve (B = 128, GQA 32/4): the tensor-core prefill kernel takes the single row.
"""
import pytest
import torch

import oracle
from block_sparse_long_15_b200 import workloads as W
from tests.parity_util import compare
from tests.test_parity_gpu import assert_report, run_prefill

pytestmark = pytest.mark.gpu

WL = W.WORKLOADS


@pytest.mark.parametrize("base,seq,n_q", [("bf16_prefill_s8192", 2000, 300),
                                          ("bf16_prefill_varlen_b8_s16384_leftpad", 1500, 257)])
def test_chunked_prefill_suffix_queries(cuda_lib, base, seq, n_q):
    w = W.small_variant(WL[base], seq=seq, batch=2, pad_max=0)
    inp = W.make_inputs(w)
    inp["q"] = inp["q"][:, seq - n_q:].contiguous()
    inp["qi"] = inp["qi"][:, seq - n_q:].contiguous()
    inp["q_first"] = inp["kv_len"] - n_q
    out, sel, _ = run_prefill(cuda_lib, w, inp)
    assert out.shape[1] == n_q
    rep = compare(w, inp, out, sel, oracle.run(w, inp))
    assert_report(rep, w)
    assert rep.rows == 2 * n_q


def _left_padded_decode(w, pads):
    """The workload's decode caches shifted right by pads[b] rows (NaN in front)."""
    inp = W.make_inputs(w)
    cap = w.seq + max(pads)
    for name in ("k", "v"):
        x = torch.full(inp[name].shape[:2] + (cap,) + inp[name].shape[3:], float("nan"), dtype=inp[name].dtype)
        for b, p in enumerate(pads):
            x[b, :, p:p + w.seq] = inp[name][b]
        inp[name] = x
    ki = torch.full((w.batch, cap, w.di), float("nan"), dtype=inp["ki"].dtype)
    for b, p in enumerate(pads):
        ki[b, p:p + w.seq] = inp["ki"][b]
    inp["ki"] = ki
    inp["kv_start"] = torch.tensor(pads, dtype=torch.int32)
    return w.replace(seq=cap), inp


def test_decode_left_padded_sequences(cuda_lib):
    from block_sparse_long_15_b200.runner import QSADecode
    base = W.small_variant(WL["bf16_decode_b64_l4k_32k"], seq=4096, batch=6, len_min=100, len_max=4000)
    w, inp = _left_padded_decode(base, [0, 37, 64, 129, 300, 511])
    d = QSADecode(w, inp)
    out, sel = d()
    torch.cuda.synchronize()
    assert d.status() == cuda_lib.QSA_OK
    rep = compare(w, inp, out.cpu(), sel.cpu(), oracle.run(w, inp), decode=True)
    assert_report(rep, w, 0.2)
    for b in range(w.batch):
        p, L = int(inp["kv_start"][b]), int(inp["kv_len"][b])
        assert torch.equal(d.t["k_cache"][b, :, p + L - 1].cpu(), inp["k_new"][b])


def test_decode_block_128_gqa_32_4(cuda_lib):
    qsa = cuda_lib
    from block_sparse_long_15_b200.runner import QSADecode
    w = W.small_variant(WL["bf16_decode_b64_l4k_32k"], seq=4096, batch=5, len_min=200, len_max=4000,
                        Hq=32, Hkv=4, Hi=8, block=128, topk=16)
    inp = W.make_inputs(w)
    d = QSADecode(w, inp)
    assert qsa.qsa_attn_kernel_name(d.cfg, qsa.QSA_DECODE) == "tcgen05"
    out, sel = d()
    torch.cuda.synchronize()
    assert d.status() == qsa.QSA_OK
    rep = compare(w, inp, out.cpu(), sel.cpu(), oracle.run(w, inp), decode=True)
    assert_report(rep, w, 0.2)
