"""Decode attention without a caller workspace (qsa_sparse_attn_decode_noalloc).

Callers such as a plugin that its host framework gives only input and output
buffers, or a server whose device memory all sits in its own pool, cannot hand the
library scratch memory; this entry point keeps the decode partials in a fixed array
inside the library instead. The GPU test checks it against qsa_sparse_attn with a
workspace, through the C ABI, on two calls in a row: the two run the same kernels on
the same inputs, so the outputs must match bit for bit (tighter than the bf16 output
tolerance of the parity tests). This file is collected last.
"""
import ctypes

import pytest
import torch

from block_sparse_long_15_b200 import workloads as W


def test_sizes_beyond_the_static_scratch_are_rejected_on_host():
    from block_sparse_long_15_b200 import build
    build.build()
    from block_sparse_long_15_b200 import qsa
    cfg = qsa.make_config(Hq=16, Hkv=2, d=128, Hi=4, di=64, block=64, topk=32)
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    # 2000 sequences x 2 KV heads: past the streaming kernel's unit limit, and the
    # per-split partials (17 splits x 8 heads x 130 floats per unit, about 283 MB)
    # do not fit the 16 MiB array
    st = qsa.library().qsa_sparse_attn_decode_noalloc(ctypes.byref(cfg), fake, fake, fake, fake, fake, fake,
                                                      2000, 4096, fake, None)
    assert st == qsa.QSA_ERR_UNSUPPORTED
    assert "static scratch" in qsa.qsa_last_error()


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_path_twice(cuda_lib):
    """Both entry points run the same decode kernels over the same inputs with the same
    split of the work, so the outputs must be identical bit for bit."""
    qsa = cuda_lib
    from block_sparse_long_15_b200.runner import QSADecode
    w = W.small_variant(W.WORKLOADS["bf16_decode_b64_l4k_32k"], seq=8192, batch=24, len_min=700,
                        len_max=8000)
    d = QSADecode(w, W.make_inputs(w))
    d()  # appends the new token and selects the blocks (sel) for this step
    torch.cuda.synchronize()
    assert d.status() == qsa.QSA_OK
    t = d.t

    def with_workspace(n):
        args = [x[:n].contiguous() for x in (t["q"], t["k_cache"], t["v_cache"], t["sel"], t["kv_start"],
                                             t["kv_len"])]
        q_first = (args[5] - 1).contiguous()
        ref = torch.empty_like(args[0])
        ws = qsa.alloc_workspace(d.cfg, qsa.QSA_DECODE, n, 1, w.seq)
        qsa.qsa_sparse_attn(d.cfg, *args[:3], args[3], args[4], args[5], q_first, ref, ws)
        torch.cuda.synchronize()
        assert qsa.qsa_read_device_status(ws) == qsa.QSA_OK
        assert torch.isfinite(ref.float()).all()
        return args, ref

    # first call: the whole batch
    args, ref = with_workspace(w.batch)
    out1 = torch.full_like(t["q"], float("nan"))
    qsa.qsa_sparse_attn_decode_noalloc(d.cfg, *args, out1)
    torch.cuda.synchronize()
    assert torch.equal(out1.view(torch.int16), ref.view(torch.int16))

    # second call right after: a smaller batch, so the array holds the first call's partials
    n = 9
    args, ref = with_workspace(n)
    out2 = torch.full_like(ref, float("nan"))
    qsa.qsa_sparse_attn_decode_noalloc(d.cfg, *args, out2)
    torch.cuda.synchronize()
    assert torch.equal(out2.view(torch.int16), ref.view(torch.int16))
