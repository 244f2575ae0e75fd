"""The persistent prefill attention kernel: its CTAs take units from a ticket counter kept
in the workspace's status page, and the last CTA sets the counters back to zero. These
tests check that every call leaves the workspace at zero (its contract) and that the
dynamic assignment of units to CTAs does not change a single output bit."""
import pytest
import torch

from block_sparse_long_15_b200 import workloads as W

pytestmark = pytest.mark.gpu

WL = W.WORKLOADS


def _status_page(ws):
    return ws[:256].cpu()


@pytest.mark.parametrize("name", ["bf16_prefill_s8192", "bf16_prefill_varlen_b8_s16384_leftpad"])
def test_repeated_calls_bit_identical_and_workspace_zero(cuda_lib, name):
    from block_sparse_long_15_b200.runner import QSAPrefill
    w = WL[name]
    p = QSAPrefill(w, W.make_inputs(w))
    outs = []
    for _ in range(3):
        out, sel = p()
        torch.cuda.synchronize()
        # status word and the attention's unit counters: all zero after the call
        assert torch.count_nonzero(_status_page(p.ws)) == 0
        outs.append((out.clone(), sel.clone()))
    for out, sel in outs[1:]:
        assert torch.equal(sel, outs[0][1])
        assert torch.equal(out, outs[0][0])


def test_standalone_attention_shares_the_workspace(cuda_lib):
    """qsa_sparse_attn on the workspace qsa_forward used: same output, counters back at zero."""
    qsa = cuda_lib
    from block_sparse_long_15_b200.runner import QSAPrefill
    w = W.small_variant(WL["bf16_prefill_s8192"], seq=2112)
    p = QSAPrefill(w, W.make_inputs(w))
    out_f, _ = p()
    out_f = out_f.clone()
    t = p.t
    out = torch.empty_like(t["q"])
    for _ in range(2):
        qsa.qsa_sparse_attn(p.cfg, t["q"], t["k_cache"], t["v_cache"], t["sel"], t["kv_start"], t["kv_len"],
                            t["q_first"], out, p.ws)
        torch.cuda.synchronize()
        assert torch.count_nonzero(_status_page(p.ws)) == 0
        assert torch.equal(out, out_f)


@pytest.mark.parametrize("shape", [
    dict(seq=1100, Hq=2, Hkv=2, block=64, topk=12),   # G = 1: 256 tokens a unit, lists beyond the slot
    dict(seq=1100, Hq=4, Hkv=2, block=64, topk=20),   # G = 2: lists beyond the slot, read from global
    dict(seq=1100, Hq=8, Hkv=2, block=64, topk=5),    # G = 4: k not a multiple of 4
    dict(seq=1100, Hq=16, Hkv=2, block=192, topk=3),  # a block size that is not a power of two
    dict(seq=2200, Hq=16, Hkv=2, block=256, topk=4),  # a block of two chunks
    dict(seq=1100, Hq=32, Hkv=2, block=64, topk=8),   # G = 16: a softmax warp's rows are one token
    dict(seq=1100, Hq=32, Hkv=1, block=128, topk=4),  # G = 32: 4 tokens a tile
])
def test_tc_attention_unit_shapes_full_rows(cuda_lib, shape):
    """Unit shapes that take the builder's other paths (the lists loaded from global
    memory, read entry by entry, blocks of several chunks): every row of a left-padded
    batch against the oracle."""
    import oracle
    from tests.parity_util import compare
    from tests.test_parity_gpu import assert_report, run_prefill
    qsa = cuda_lib
    w = W.small_variant(WL["bf16_prefill_varlen_b8_s16384_leftpad"], batch=2, pad_max=130, **shape)
    assert qsa.qsa_attn_kernel_name(qsa.config_for(w)) == "tcgen05"
    inp = W.make_inputs(w)
    out, sel, _ = run_prefill(qsa, w, inp)
    rep = compare(w, inp, out, sel, oracle.run(w, inp))
    assert_report(rep, w)


@pytest.mark.parametrize("name,shape,calls", [
    ("bf16_prefill_s8192", None, 200),
    ("bf16_prefill_varlen_b8_s16384_leftpad", dict(seq=1100, Hq=2, Hkv=2, block=64, topk=12), 150),
    ("bf16_prefill_varlen_b8_s16384_leftpad", dict(seq=2200, Hq=16, Hkv=2, block=256, topk=4), 150),
])
def test_soak_many_calls(cuda_lib, name, shape, calls):
    """Many calls in a row on one workspace: the status word stays clear, every output
    equals the first bit for bit, and the counters are back at zero at the end -- the
    dynamic assignment of units to CTAs differs from call to call."""
    from block_sparse_long_15_b200.runner import QSAPrefill
    w = WL[name] if shape is None else W.small_variant(WL[name], batch=2, pad_max=130, **shape)
    p = QSAPrefill(w, W.make_inputs(w))
    ref, _ = p()
    torch.cuda.synchronize()
    ref = ref.clone()
    for i in range(calls):
        out, _ = p()
        if i % 25 == 24 or i == calls - 1:
            torch.cuda.synchronize()
            assert p.status() == cuda_lib.QSA_OK, i
            assert torch.equal(out, ref), i
    assert torch.count_nonzero(_status_page(p.ws)) == 0
