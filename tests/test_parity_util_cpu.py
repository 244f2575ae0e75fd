"""Host logic of the parity comparison (tests/parity_util.py), on the CPU: a faithful
result passes; a wrong output, an invalid selection or a selection swap that is not
a near-tie fails; a near-tie swap is counted and its output is checked against the
oracle's attention over the swapped selection."""
import numpy as np
import torch

import oracle
from block_sparse_long_15_b200 import workloads as W
from tests.parity_util import compare


def _case():
    w = W.small_variant(W.WORKLOADS["bf16_prefill_s8192"], seq=448, topk=2)
    inp = W.make_inputs(w)
    orc = oracle.run(w, inp)
    out = torch.from_numpy(orc["o"][0]).to(torch.bfloat16)[None]
    sel = torch.from_numpy(orc["sel"][0])[None]
    return w, inp, orc, out, sel


def test_oracle_output_rounded_to_bf16_passes():
    w, inp, orc, out, sel = _case()
    rep = compare(w, inp, out, sel, orc)
    assert rep.ok(), str(rep)
    assert rep.sel_exact == rep.rows == 448 and rep.near_tie_rows == 0


def test_wrong_output_and_invalid_selection_fail():
    w, inp, orc, out, sel = _case()
    bad = out.clone()
    bad[0, 300, 3, 5] += 0.25
    assert not compare(w, inp, bad, sel, orc).ok()
    bad_sel = sel.clone()
    bad_sel[0, 300] = torch.tensor([3, 3], dtype=torch.int32)  # not ascending/unique
    assert compare(w, inp, out, bad_sel, orc).failures


def test_selection_swap_beyond_near_tie_fails():
    w, inp, orc, out, sel = _case()
    r = 400  # n_c = 6 candidates, 2 kept: swap a kept block for the lowest-scoring one
    s = oracle.scores(w, inp, 0, [r])[0][: (r + 1) // w.block]  # the row's candidates
    worst = int(np.argmin(s))
    kept = [int(x) for x in orc["sel"][0][r]]
    assert worst not in kept
    new = sorted([kept[0], worst])
    sel2 = sel.clone()
    sel2[0, r] = torch.tensor(new, dtype=torch.int32)
    rep = compare(w, inp, out, sel2, orc)
    assert any("beyond a near-tie" in f for f in rep.failures), str(rep)


def test_near_tie_swap_is_counted_and_its_output_checked():
    w, inp, orc, out, sel = _case()
    r = 400
    s = oracle.scores(w, inp, 0, [r])[0]
    kept = [int(x) for x in orc["sel"][0][r]]
    other = [j for j in range((r + 1) // w.block) if j not in kept][0]
    # make `other` a near-tie of kept[1] by overriding the oracle's scores for this row
    s_tie = s.copy()
    s_tie[other] = s_tie[kept[1]] * (1 - 1e-4)
    new = sorted([kept[0], other])
    sel2 = sel.clone()
    sel2[0, r] = torch.tensor(new, dtype=torch.int32)
    # the output of that row is the attention over the swapped selection
    o_swap = oracle.attend_selection(w, inp, 0, [r], np.array([new], dtype=np.int32))
    out2 = out.clone()
    out2[0, r] = torch.from_numpy(o_swap[0]).to(torch.bfloat16)
    import tests.parity_util as pu
    real_scores = oracle.scores
    try:
        oracle.scores = lambda *a, **k: np.array([s_tie])
        rep = pu.compare(w, inp, out2, sel2, orc)
        assert rep.ok() and rep.near_tie_rows == 1 and rep.near_tie_checked == 1, str(rep)
        # the same swap with the output of the oracle's own selection left in place fails
        rep = pu.compare(w, inp, out, sel2, orc)
        assert not rep.ok(), str(rep)
    finally:
        oracle.scores = real_scores


def test_attend_selection_on_the_oracle_selection_equals_the_oracle():
    w, inp, orc, _, _ = _case()
    rows = [0, 63, 64, 200, 447]
    o = oracle.attend_selection(w, inp, 0, rows, orc["sel"][0][rows])
    assert np.array_equal(o, orc["o"][0][rows])
