"""Decode with the attention K/V cache offloaded to page-locked host memory
(qsa_decode_offload): only the attended blocks cross to the device, and the results
equal the on-device decode step bit for bit (same keys, same order)."""
import pytest
import torch

import oracle
from block_sparse_long_15_b200 import workloads as W
from tests.parity_util import compare
from tests.test_parity_gpu import assert_report

pytestmark = pytest.mark.gpu


def _workload(batch=10, seq=4096, d=128):
    w = W.small_variant(W.WORKLOADS["bf16_decode_b64_l4k_32k"], seq=seq, batch=batch, len_min=40, len_max=4000,
                        d=d)
    inp = W.make_inputs(w)
    # one sequence whose new token completes a block, one shorter than the budget
    inp["kv_len"][0] = 1024
    inp["kv_len"][1] = 700
    for b in (0, 1):
        L = int(inp["kv_len"][b])
        inp["k"][b, :, :L - 1] = torch.randn(w.Hkv, L - 1, w.d).to(inp["k"].dtype) * w.std
        inp["v"][b, :, :L - 1] = torch.randn(w.Hkv, L - 1, w.d).to(inp["v"].dtype) * w.std
        inp["ki"][b, :L - 1] = torch.randn(L - 1, w.di).to(inp["ki"].dtype) * w.std
    inp["q_first"] = inp["kv_len"] - 1
    return w, inp


@pytest.mark.parametrize("d", [128, 256])
def test_offload_decode_equals_device_decode(cuda_lib, d):
    qsa = cuda_lib
    from block_sparse_long_15_b200.runner import QSADecode, QSADecodeOffload
    w, inp = _workload(d=d)
    dev = QSADecode(w, inp)
    out_d, sel_d = dev()
    off = QSADecodeOffload(w, inp)
    assert not off.t["k_cache"].is_cuda and off.t["k_cache"].is_pinned()
    out_o, sel_o = off()
    torch.cuda.synchronize()
    assert dev.status() == qsa.QSA_OK and off.status() == qsa.QSA_OK
    assert torch.equal(sel_o.cpu(), sel_d.cpu())
    assert torch.equal(out_o.cpu().view(torch.int16), out_d.cpu().view(torch.int16))
    # the appended token is in the host cache, the indexer state advanced alike
    L = inp["kv_len"]
    for b in range(w.batch):
        assert torch.equal(off.t["k_cache"][b, :, L[b] - 1], inp["k_new"][b])
        assert torch.equal(off.t["v_cache"][b, :, L[b] - 1], inp["v_new"][b])
    assert torch.equal(off.t["kbar_blocks"].cpu(), dev.t["kbar_blocks"].cpu())
    assert torch.equal(off.t["kbar_cache"].cpu(), dev.t["kbar_cache"].cpu())
    # and against the oracle
    rep = compare(w, inp, out_o.cpu(), sel_o.cpu(), oracle.run(w, inp), decode=True)
    assert_report(rep, w, 0.2)


def test_offload_rejects_pageable_host_memory(cuda_lib):
    qsa = cuda_lib
    from block_sparse_long_15_b200.runner import QSADecodeOffload
    w, inp = _workload(batch=2)
    off = QSADecodeOffload(w, inp)
    off.t["k_cache"] = off.t["k_cache"].clone()  # a plain (pageable) CPU tensor
    assert not off.t["k_cache"].is_pinned()
    with pytest.raises(qsa.QSAError) as e:
        off()
    assert e.value.status == qsa.QSA_ERR_INVALID_ARG
    assert "page-locked" in qsa.qsa_last_error()
