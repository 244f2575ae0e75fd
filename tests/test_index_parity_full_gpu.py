"""Full index parity on the prefill workloads at full size: the block selection of
EVERY query row against the oracle (scores in fp64, exact top-k).
Output parity on these workloads is checked on sampled rows (test_parity_gpu.py);
the selection is cheap for the oracle, so here it is checked everywhere.

A row may differ from the oracle only where every swapped pair of blocks is a
near-tie under the oracle's fp64 scores (relative gap <= NEAR_TIE_REL): the kernel
scores in fp32 from bf16 inputs. Such rows must stay rare.
"""
import numpy as np
import pytest

import oracle
from block_sparse_long_15_b200 import workloads as W
from tests.parity_util import NEAR_TIE_REL, check_sel_valid
from tests.test_parity_gpu import run_prefill

pytestmark = pytest.mark.gpu

ROWS_PER_CALL = 4096


def _full_index_parity(w, inp, sel):
    exact = near = rows = 0
    failures = []
    k = w.topk
    n_q = inp["q"].shape[1]
    for b in range(w.batch):
        qf, L = int(inp["q_first"][b]), int(inp["kv_len"][b])
        real = [r for r in range(n_q) if 0 <= qf + r < L]
        real_set = set(real)
        for r in range(n_q):  # padding rows select nothing
            if r not in real_set and not np.all(sel[b, r] == -1):
                failures.append(f"b={b} padding row {r} has selections")
        for c0 in range(0, len(real), ROWS_PER_CALL):
            chunk = real[c0:c0 + ROWS_PER_CALL]
            sc = oracle.scores(w, inp, b, chunk)
            for i, r in enumerate(chunk):
                t = qf + r
                n_c = (t + 1) // w.block
                g = sel[b, r]
                msg = check_sel_valid(g, t, w.block, k)
                if msg:
                    failures.append(f"b={b} r={r}: {msg}")
                    continue
                ref = oracle.select(sc[i, :n_c], k)
                rows += 1
                if np.array_equal(g, ref):
                    exact += 1
                    continue
                extra = set(g.tolist()) - set(ref.tolist()) - {-1}
                missing = set(ref.tolist()) - set(g.tolist()) - {-1}
                tie = len(extra) == len(missing) and all(
                    abs(sc[i, a] - sc[i, m]) <= NEAR_TIE_REL * max(abs(sc[i, a]), abs(sc[i, m]))
                    for a in extra for m in missing)
                if tie:
                    near += 1
                else:
                    failures.append(f"b={b} r={r}: gpu {g.tolist()} oracle {ref.tolist()}")
    return rows, exact, near, failures


@pytest.mark.parametrize("name", ["bf16_prefill_s8192", "bf16_prefill_s65536_planted",
                                  "bf16_prefill_varlen_b8_s16384_leftpad"])
def test_full_index_parity(cuda_lib, name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w)
    _, sel, _ = run_prefill(cuda_lib, w, inp)
    rows, exact, near, failures = _full_index_parity(w, inp, sel.numpy())
    print(name, f"rows={rows} exact={exact} near_tie={near} failures={len(failures)}")
    assert not failures, failures[:5]
    assert rows == int(sum(min(int(inp["kv_len"][b]), inp["q"].shape[1]) for b in range(w.batch)))
    assert near <= max(1, 0.01 * rows)
