"""Comparison rules between the CUDA path and the fp64 oracle.

Tolerances (written here, used by every parity test):
  fp32 workloads: selected block ids bit-exact; outputs |g - o| <= 1e-4 + 1e-4 |o|.
  bf16 workloads: outputs |g - o| <= 1e-2 + 2e-2 |o| on rows whose selection
  matches; a row whose selection differs is accepted only if every swapped pair
  (a chosen by the GPU, b chosen by the oracle) is a near-tie under the oracle's
  fp64 scores, |s_a - s_b| <= 1e-3 max(|s_a|, |s_b|); such rows are counted, and
  their outputs are compared, within the same tolerance, with the oracle's fp64
  attention over the token set of the GPU's own selection.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Sequence

import numpy as np
import torch

import oracle

TOL = {"fp32": dict(atol=1e-4, rtol=1e-4), "bf16": dict(atol=1e-2, rtol=2e-2)}
NEAR_TIE_REL = 1e-3


@dataclass
class Report:
    rows: int = 0
    sel_exact: int = 0
    near_tie_rows: int = 0
    near_tie_checked: int = 0  # near-tie rows whose output matched the oracle on the GPU's selection
    max_abs_err: float = 0.0
    max_excess: float = -np.inf  # max of |g-o| - (atol + rtol |o|); <= 0 passes
    failures: List[str] = field(default_factory=list)

    def ok(self) -> bool:
        return not self.failures and self.max_excess <= 0.0

    def __str__(self):
        return (f"rows={self.rows} sel_exact={self.sel_exact} near_tie_rows={self.near_tie_rows} "
                f"near_tie_checked={self.near_tie_checked} "
                f"max_abs_err={self.max_abs_err:.3e} max_excess={self.max_excess:.3e} "
                f"failures={self.failures[:5]}")


def check_sel_valid(sel_row: np.ndarray, t: int, block: int, k: int) -> str:
    """Ascending, unique, inside [0, n_c), -1 padding only at the end, count min(n_c, k)."""
    n_c = (t + 1) // block if t >= 0 else 0
    want_n = min(n_c, k)
    valid = sel_row[sel_row >= 0]
    if len(valid) != want_n:
        return f"t={t}: {len(valid)} blocks selected, expected {want_n}"
    if not np.all(sel_row[:want_n] >= 0) or not np.all(sel_row[want_n:] == -1):
        return f"t={t}: -1 padding misplaced {sel_row.tolist()}"
    if want_n and (np.any(np.diff(valid) <= 0) or valid.max() >= n_c):
        return f"t={t}: not ascending / out of range {valid.tolist()}"
    return ""


def compare(w, inp: Dict[str, torch.Tensor], gpu_out: torch.Tensor, gpu_sel: torch.Tensor,
            orc: Dict, decode: bool = False) -> Report:
    """gpu_out [batch][n_q][Hq][d], gpu_sel [batch][n_q][k] (CPU tensors); orc from oracle.run."""
    tol = TOL[w.dtype]
    rep = Report()
    for b, rows in orc["rows"].items():
        q_first = int(inp["q_first"][b])
        o_ref = orc["o"][b]
        s_ref = orc["sel"][b]
        g_out = gpu_out[b].index_select(0, torch.tensor(rows)).double().numpy()
        g_sel = gpu_sel[b].index_select(0, torch.tensor(rows)).numpy()
        mism = []
        for i, r in enumerate(rows):
            t = q_first + r
            msg = check_sel_valid(g_sel[i], t, w.block, w.topk) if 0 <= t < int(inp["kv_len"][b]) else (
                "" if np.all(g_sel[i] == -1) else f"pad row {r} has selections")
            if msg:
                rep.failures.append(f"b={b} {msg}")
                continue
            if np.array_equal(g_sel[i], s_ref[i]):
                rep.sel_exact += 1
            else:
                mism.append(i)
        rep.rows += len(rows)
        if mism:
            if w.dtype == "fp32":
                rep.failures.append(f"b={b}: {len(mism)} fp32 rows with selection mismatch, e.g. row "
                                    f"{rows[mism[0]]}: gpu {g_sel[mism[0]].tolist()} oracle {s_ref[mism[0]].tolist()}")
            else:
                sc = oracle.scores(w, inp, b, [rows[i] for i in mism], decode=decode)
                tie_rows = []
                for j, i in enumerate(mism):
                    a_set = set(g_sel[i].tolist()) - {-1}
                    b_set = set(s_ref[i].tolist()) - {-1}
                    extra, missing = a_set - b_set, b_set - a_set
                    ok = len(extra) == len(missing)
                    for a in extra:
                        for bb in missing:
                            sa, sb = sc[j][a], sc[j][bb]
                            if abs(sa - sb) > NEAR_TIE_REL * max(abs(sa), abs(sb)):
                                ok = False
                    if ok:
                        rep.near_tie_rows += 1
                        tie_rows.append(i)
                    else:
                        rep.failures.append(f"b={b} row {rows[i]}: selection differs beyond a near-tie "
                                            f"(extra {sorted(extra)}, missing {sorted(missing)})")
                if tie_rows:
                    # the GPU's output on a near-tie row against the oracle's attention over
                    # the GPU's own (valid, near-optimal) selection
                    o_tie = oracle.attend_selection(w, inp, b, [rows[i] for i in tie_rows], g_sel[tie_rows],
                                                    decode=decode)
                    g = g_out[tie_rows]
                    if not np.all(np.isfinite(g)):
                        rep.failures.append(f"b={b}: non-finite GPU output on a near-tie row")
                    else:
                        err = np.abs(g - o_tie)
                        exc = (err - (tol["atol"] + tol["rtol"] * np.abs(o_tie))).reshape(len(tie_rows), -1).max(1)
                        rep.max_abs_err = max(rep.max_abs_err, float(err.max()))
                        rep.max_excess = max(rep.max_excess, float(exc.max()))
                        rep.near_tie_checked += int((exc <= 0).sum())
        keep = [i for i in range(len(rows)) if i not in set(mism)]
        if keep:
            g, o = g_out[keep], o_ref[keep]
            if not np.all(np.isfinite(g)):
                rep.failures.append(f"b={b}: non-finite GPU output")
                continue
            err = np.abs(g - o)
            rep.max_abs_err = max(rep.max_abs_err, float(err.max()))
            rep.max_excess = max(rep.max_excess, float((err - (tol["atol"] + tol["rtol"] * np.abs(o))).max()))
    return rep


def sample_rows(n_q: int, q_first: int, kv_len: int, block: int, n_random: int, seed: int) -> List[int]:
    """Query rows: the first and last two blocks of the sequence, block edges, and a seeded sample."""
    lo = max(0, -q_first)
    hi = min(n_q, kv_len - q_first)
    if hi <= lo:
        return []
    rows = set(range(lo, min(hi, lo + 2 * block)))
    rows |= set(range(max(lo, hi - 2 * block), hi))
    g = np.random.default_rng(seed)
    rows |= set(int(x) for x in g.integers(lo, hi, size=n_random))
    for j in g.integers(1, max(2, (hi - lo) // block), size=8):
        for off in (-1, 0, 1):
            r = lo + int(j) * block + off
            if lo <= r < hi:
                rows.add(r)
    if lo > 0:
        rows.add(lo - 1)  # one padding row
    return sorted(rows)
