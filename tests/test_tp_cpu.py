"""Head-sharded tensor parallelism ("Qwen4-Exp" Usage tips: tp_plan="auto" shards QSA)
on the CPU, with the fp64 oracle.

The reading: ranks hold equal shards of the query, KV and indexer query heads; the
block score is a sum over indexer heads, so the ranks' partial scores summed (an
all-reduce) are the full scores; every rank selects from them and attends its own
heads. Pinned here:
  - the partial scores of the shards add up to the full scores (fp64);
  - the selection from the summed partials is the unsharded selection, and a MAX
    reduction in place of the SUM (a plausible mistake) selects differently;
  - the shards' outputs, concatenated over heads, are the unsharded output;
  - the same, end to end, as two gloo ranks that all-reduce their partial scores.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from block_sparse_long_15_b200 import tp as TP
from block_sparse_long_15_b200 import workloads as W


def _w():
    return W.small_variant(W.WORKLOADS["bf16_prefill_varlen_b8_s16384_leftpad"], seq=700, batch=2, pad_max=120,
                           topk=3)


def _rows(inp, b):
    L, qf = int(inp["kv_len"][b]), int(inp["q_first"][b])
    return list(range(-qf, -qf + L))


def _shard_scores(w, inp, tp, rank, b, rows):
    ws = TP.shard_workload(w, tp)
    return oracle.scores(ws, TP.shard_inputs(inp, w, tp, rank), b, rows)


def _select_rows(w, inp, b, rows, scores):
    qf = int(inp["q_first"][b])
    out = []
    for i, r in enumerate(rows):
        n_c = (qf + r + 1) // w.block
        out.append(oracle.select(scores[i][:n_c], w.topk))
    return np.array(out, dtype=np.int32)


@pytest.mark.parametrize("tp", [2, 4])
def test_partial_scores_add_up_to_the_full_scores(tp):
    w = _w()
    inp = W.make_inputs(w)
    for b in range(w.batch):
        rows = _rows(inp, b)
        full = oracle.scores(w, inp, b, rows)
        parts = sum(_shard_scores(w, inp, tp, r, b, rows) for r in range(tp))
        qf = int(inp["q_first"][b])
        for i, r in enumerate(rows):
            n_c = (qf + r + 1) // w.block
            np.testing.assert_allclose(parts[i][:n_c], full[i][:n_c], rtol=1e-12, atol=1e-15)


def test_selection_from_reduced_scores_is_the_unsharded_selection():
    w, tp = _w(), 2
    inp = W.make_inputs(w)
    orc = oracle.run(w, inp)
    differs = 0
    for b in range(w.batch):
        rows = _rows(inp, b)
        p0, p1 = (_shard_scores(w, inp, tp, r, b, rows) for r in range(tp))
        sel = _select_rows(w, inp, b, rows, p0 + p1)
        assert np.array_equal(sel, orc["sel"][b][rows])
        differs += int(np.any(_select_rows(w, inp, b, rows, np.maximum(p0, p1)) != sel, axis=1).sum())
    assert differs > 0, "a MAX reduction of the partial scores would go unnoticed"


def test_head_shards_concatenate_to_the_unsharded_output():
    w, tp = _w(), 2
    inp = W.make_inputs(w)
    orc = oracle.run(w, inp)
    for b in range(w.batch):
        rows = _rows(inp, b)
        sel = orc["sel"][b][rows]
        outs = [oracle.attend_selection(TP.shard_workload(w, tp), TP.shard_inputs(inp, w, tp, r), b, rows, sel)
                for r in range(tp)]
        assert np.array_equal(np.concatenate(outs, axis=1), orc["o"][b][rows])


def test_sharding_rejects_indivisible_head_counts():
    w = _w()
    with pytest.raises(ValueError):
        TP.shard_workload(w, 3)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    w = _w()
    inp = W.make_inputs(w)
    ws = TP.shard_workload(w, world)
    mine = TP.shard_inputs(inp, w, world, rank)
    res = {}
    for b in range(w.batch):
        rows = _rows(inp, b)
        part = torch.from_numpy(oracle.scores(ws, mine, b, rows))
        dist.all_reduce(part, op=dist.ReduceOp.SUM)  # the score all-reduce before top-k
        sel = _select_rows(w, inp, b, rows, part.numpy())
        out = oracle.attend_selection(ws, mine, b, rows, sel)
        res[b] = (sel, out)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, res))


def test_two_gloo_ranks_all_reduce_partial_scores():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = _w()
    inp = W.make_inputs(w)
    orc = oracle.run(w, inp)
    for b in range(w.batch):
        rows = _rows(inp, b)
        assert np.array_equal(got[0][b][0], got[1][b][0])  # every rank selects the same blocks
        assert np.array_equal(got[0][b][0], orc["sel"][b][rows])
        out = np.concatenate([got[0][b][1], got[1][b][1]], axis=1)
        assert np.array_equal(out, orc["o"][b][rows])
