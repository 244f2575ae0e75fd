"""Head-sharded tensor parallelism through the C ABI on one GPU: the shards of a TP
group run one after the other on the same device (qsa_index_scores for each shard's
indexer heads), their partial scores are summed on the device as the all-reduce
would, and each shard selects (qsa_select_topk) and attends its own heads
(qsa_sparse_attn). Checked against the fp64 oracle of the unsharded path, and
against the unsharded GPU path: every row whose selection agrees has a bit-identical
output (the attention of a head does not depend on the other heads). The NCCL
all-reduce itself needs more than one GPU and is not exercised here."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_15_b200 import tp as TP
from block_sparse_long_15_b200 import workloads as W
from tests.parity_util import compare
from tests.test_parity_gpu import assert_report, run_prefill

pytestmark = pytest.mark.gpu

WL = W.WORKLOADS


def run_tp(w, inp, tp):
    ranks = [TP.QSAPrefillTP(w, inp, tp, r) for r in range(tp)]
    parts = [x.partial_scores() for x in ranks]
    total = torch.stack(parts).sum(0)
    for x in ranks:
        x.finish(total.clone())
    torch.cuda.synchronize()
    for x in ranks:
        assert x.status() == 0
    sels = [x.sel.cpu() for x in ranks]
    for s in sels[1:]:
        assert torch.equal(s, sels[0])  # every rank selects the same blocks
    return TP.gather_heads([x.out for x in ranks]).cpu(), sels[0]


@pytest.mark.parametrize("name,seq,batch,tp,rows", [
    ("bf16_prefill_s8192", 2112, 1, 2, None),
    ("bf16_prefill_varlen_b8_s16384_leftpad", 1300, 2, 2, None),
    ("bf16_prefill_varlen_b8_s16384_leftpad", 1300, 2, 4, None),
    ("bf16_prefill_s8192", 8192, 1, 2, 256),
])
def test_tp_shards_match_oracle_and_unsharded_path(cuda_lib, name, seq, batch, tp, rows):
    w = W.small_variant(WL[name], seq=seq, batch=batch, pad_max=min(WL[name].pad_max, 200))
    inp = W.make_inputs(w)
    out, sel = run_tp(w, inp, tp)
    if rows is None:
        orc = oracle.run(w, inp)
    else:
        from tests.test_parity_gpu import oracle_rows
        orc = oracle.run(w, inp, rows=oracle_rows(w, inp, rows, 500))
    assert_report(compare(w, inp, out, sel, orc), w)
    out_u, sel_u, _ = run_prefill(cuda_lib, w, inp)
    same = (sel == sel_u).all(-1)
    assert same.float().mean() >= 0.99
    assert torch.equal(out[same].view(torch.int16), out_u[same].view(torch.int16))


def test_select_topk_exact_on_adversarial_scores(cuda_lib):
    """qsa_select_topk on fp32 scores with negatives, zeros of both signs and many
    exact ties: the ids equal the oracle's selection on the same fp32 values."""
    qsa = cuda_lib
    w = W.small_variant(WL["bf16_prefill_s8192"], seq=1500, batch=3, topk=5)
    cfg = qsa.config_for(w)
    n_q, nb = w.seq, w.seq // w.block
    g = torch.Generator().manual_seed(7)
    sc = torch.randint(-3, 4, (w.batch, n_q, nb), generator=g).float() * 0.5  # many exact ties
    sc[sc == 0] = torch.where(torch.rand(int((sc == 0).sum()), generator=g) < 0.5, -0.0, 0.0)
    sc[:, ::7] = torch.randn((w.batch, (n_q + 6) // 7, nb), generator=g)
    kv_len = torch.tensor([1500, 1000, 0], dtype=torch.int32)
    q_first = torch.tensor([0, -500, -1500], dtype=torch.int32)
    sel = torch.empty(w.batch, n_q, w.topk, dtype=torch.int32, device="cuda")
    ws = qsa.alloc_workspace(cfg, qsa.QSA_PREFILL, w.batch, n_q, w.seq)
    qsa.qsa_select_topk(cfg, sc.cuda(), kv_len.cuda(), q_first.cuda(), w.seq, sel, ws)
    torch.cuda.synchronize()
    assert qsa.qsa_read_device_status(ws) == qsa.QSA_OK
    sel = sel.cpu().numpy()
    for b in range(w.batch):
        for r in range(n_q):
            t = int(q_first[b]) + r
            if not (0 <= t < int(kv_len[b])):
                assert np.all(sel[b, r] == -1)
                continue
            n_c = (t + 1) // w.block
            want = oracle.select(sc[b, r, :n_c].double().numpy(), w.topk)
            assert np.array_equal(sel[b, r], want), (b, r)
