"""Host logic of bench.py: exact work counting (against the oracle's token sets) and
the multi-rank aggregation (max over ranks, all ranks' tokens), run as two gloo ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import bench
import oracle
from block_sparse_long_15_b200 import workloads as W


def test_attended_pairs_matches_oracle_token_sets():
    w = W.small_variant(W.WORKLOADS["bf16_prefill_varlen_b8_s16384_leftpad"], seq=600, batch=3, pad_max=200)
    inp = W.make_inputs(w)
    pairs, score_pairs = bench.attended_pairs(w, inp)
    want = 0
    want_sc = 0
    for b in range(w.batch):
        L = int(inp["kv_len"][b])
        for t in range(L):
            n_c = (t + 1) // w.block
            sel = np.array(list(range(min(n_c, w.topk))) + [-1] * max(0, w.topk - n_c), dtype=np.int32)
            want += len(oracle.token_set(t, w.block, sel))
            want_sc += n_c
    assert pairs == want and score_pairs == want_sc
    assert bench.real_rows(inp) == int(inp["kv_len"].sum())


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    info = {"rank": rank, "world": world, "backend": "gloo"}
    ms, value = bench.aggregate(10.0 + 5.0 * rank, 8192, info)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ms, value))


def test_aggregate_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, value in res:
        assert ms == 15.0  # the slowest rank's time
        assert value == pytest.approx(2 * 8192 / 15e-3)


def test_ncu_traffic_voided_when_kernel_source_changes(tmp_path, monkeypatch):
    import json
    src = tmp_path / "kern.cu"
    src.write_text("__global__ void k() {}\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    entry = {"kernel": "k", "source": "kern.cu", "source_sha": bench.file_sha("kern.cu"),
             "dram_bytes_per_launch": 1234.0}
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps({"attn_prefill:w": entry}))
    assert bench.ncu_traffic("attn_prefill:w") == 1234.0
    assert bench.ncu_traffic("attn_prefill:other") is None
    src.write_text("__global__ void k() { /* changed */ }\n")
    assert bench.ncu_traffic("attn_prefill:w") is None


def test_decode_kernel_bytes_counts_attended_tokens():
    w = W.small_variant(W.WORKLOADS["bf16_decode_b64_l4k_32k"], seq=4096, batch=5, len_min=40, len_max=4000)
    inp = W.make_inputs(w)
    want = 0
    for b in range(w.batch):
        L = int(inp["kv_len"][b])
        t = L - 1
        n_c = (t + 1) // w.block
        sel = np.array(list(range(min(n_c, w.topk))) + [-1] * max(0, w.topk - n_c), dtype=np.int32)
        toks = len(oracle.token_set(t, w.block, sel))  # attended tokens of the decode row
        want += toks * w.Hkv * w.d * 2 * 2 + 2 * w.Hq * w.d * 2  # K and V, then q and out (bf16)
    assert bench.decode_kernel_bytes(w, inp) == want


def test_executed_tensor_work_model():
    """k_attn_tc's executed work model: with every block selected, tile i (16 rows of
    8 heads) multiplies chunks 0 .. (16 i + 15) // 128 of the keys; tiles whose rows
    select only blocks 1 and 3 (keys 64..127 and 192..255, i.e. chunks 0 and 1) and
    sit in chunk 3 multiply chunks 0, 1 and 3."""
    import torch
    w = W.small_variant(W.WORKLOADS["bf16_prefill_s8192"], seq=512, topk=8)
    inp = W.make_inputs(w)
    sel = torch.from_numpy(oracle.run(w, inp)["sel"][0])[None]
    per = 4 * 128 * 128 * 128 * w.Hkv
    want = sum((16 * i + 15) // 128 + 1 for i in range(32)) * per
    assert bench.tc_executed_flops(w, inp, sel) == want
    w2 = W.small_variant(W.WORKLOADS["bf16_prefill_s8192"], seq=512, topk=2)
    inp2 = W.make_inputs(w2)
    sel2 = torch.full((1, 512, 2), -1, dtype=torch.int32)
    sel2[0, 448:] = torch.tensor([1, 3], dtype=torch.int32)
    ex = bench.tc_executed_flops(w2, inp2, sel2)
    # rows 0..447 (tiles 0..27): only their trailing ranges (every id is -1), one chunk each;
    # tiles 28..31: chunks 0, 1 and the trailing chunk 3
    want2 = 28 + 4 * 3
    assert ex == want2 * per, (ex / per, want2)


def test_cpu_sample_sized_past_the_fixed_cost(monkeypatch):
    """The CPU baseline's sample lasts about the requested seconds even when a call
    has a large fixed part: a fake oracle costs 2 s + 1 ms a row on a fake clock."""
    w = W.small_variant(W.WORKLOADS["bf16_prefill_varlen_b8_s16384_leftpad"], seq=4096, batch=8, pad_max=200)
    inp = W.make_inputs(w)
    clock = [0.0]
    runs = []

    def fake_run(w_, inp_, rows=None, **kw):
        n = sum(len(v) for v in rows.values())
        runs.append(n)
        clock[0] += 2.0 + 1e-3 * n

    monkeypatch.setattr(oracle, "run", fake_run)
    monkeypatch.setattr(bench.time, "perf_counter", lambda: clock[0])
    r = bench.cpu_oracle_rate(w, inp, 15.0)
    n_main = runs[-1]
    assert runs[:2] == [32, 256]
    # 2 s fixed + n_main ms ~= 15 s
    assert abs((2.0 + 1e-3 * n_main) - 15.0) < 0.1, n_main
    assert abs(r["value"] - n_main / (2.0 + 1e-3 * n_main)) < 1e-6
