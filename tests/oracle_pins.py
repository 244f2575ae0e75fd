"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with a
closed form, a brute-force enumeration, a library routine (torch SDPA in fp64),
or an invariant the QSA definition implies.  They are plain functions so that
the mutation test can run them against deliberately broken oracle builds.

Definitions: Hugging Face Transformers model doc "Qwen4-Exp", intro paragraph
on QSA and the Qwen4ExpTextConfig indexer_* / num_key_value_heads parameters.
"""
from __future__ import annotations

import itertools
import json
import math
import os
import types

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _cfg(**kw):
    base = dict(Hq=4, Hkv=2, d=16, Hi=2, di=8, block=4, topk=2, scale=None)
    base.update(kw)
    return types.SimpleNamespace(**base)


def _rand_seq(cfg, S, seed, dtype=torch.float32, std=1.0, batch=1):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s: (torch.randn(*s, generator=g) * std).to(dtype)
    return dict(q=r(batch, S, cfg.Hq, cfg.d), k=r(batch, cfg.Hkv, S, cfg.d),
                v=r(batch, cfg.Hkv, S, cfg.d), qi=r(batch, S, cfg.Hi, cfg.di),
                ki=r(batch, S, cfg.di), kv_start=torch.zeros(batch, dtype=torch.int32),
                kv_len=torch.full((batch,), S, dtype=torch.int32),
                q_first=torch.zeros(batch, dtype=torch.int32))


def _sdpa(q, k, v, scale, mask):
    """Library softmax attention in fp64. q [Hq][T][d], k/v [Hq][S][d], mask [T][S] bool."""
    return torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double(), v.double(), attn_mask=mask, scale=scale)


# --------------------------------------------------------------------------- a1
def pin_compress_closed_form(orc):
    """k̄ of keys ki[u][c] = u/2 + c is the arithmetic-series mean jB/2 + (B-1)/4 + c."""
    for B, n, di in [(4, 19, 3), (8, 64, 5), (1, 3, 2)]:
        u = torch.arange(n, dtype=torch.float32)[:, None]
        c = torch.arange(di, dtype=torch.float32)[None, :]
        kb = orc.compress(u / 2 + c, B)
        assert kb.shape == (n // B, di), kb.shape
        for j in range(n // B):
            want = (j * B) / 2 + (B - 1) / 4 + np.arange(di)
            assert np.allclose(kb[j], want, rtol=0, atol=1e-12), (B, j, kb[j], want)


def pin_compress_constant_and_partial(orc):
    """Constant keys compress to the constant; the partial tail is never compressed."""
    ki = torch.full((10, 4), 0.75)
    kb = orc.compress(ki, 4)
    assert kb.shape == (2, 4) and np.all(kb == 0.75)


# --------------------------------------------------------------------------- a2/a3 hand-worked
def pin_hand_worked(orc):
    with open(os.path.join(GOLDEN, "hand_worked_qsa.json")) as f:
        g = json.load(f)
    B = g["block"]
    ki = torch.tensor(g["ki"], dtype=torch.float32)
    kb = orc.compress(ki, B)
    assert np.array_equal(kb, np.array(g["kbar"], dtype=np.float64)), kb
    for case in g["cases"]:
        qi = torch.tensor(case["qi"], dtype=torch.float32)
        n_c = (case["t"] + 1) // B
        s = orc.block_scores(qi, kb, n_c)
        assert np.array_equal(s, np.array(case["scores"], dtype=np.float64)), (case, s)
        sel = orc.select(s, case["topk"])
        assert sel.tolist() == case["sel"], (case, sel)
        toks = orc.token_set(case["t"], B, sel)
        assert toks.tolist() == case["tokens"], (case, toks)
    a = g["attention"]
    out = orc.attend(torch.tensor(a["q"], dtype=torch.float32),
                     torch.tensor(a["k"], dtype=torch.float32),
                     torch.tensor(a["v"], dtype=torch.float32), 1.0,
                     np.array(a["tokens"], dtype=np.int64))
    assert np.allclose(out, np.array(a["out"]), rtol=0, atol=a["tol"]), out


def pin_scores_single_head_and_homogeneity(orc):
    """Hi=1 with a unit query picks out one coordinate of k̄, clipped at zero;
    scaling all queries by c>0 scales every score by c (positive homogeneity)."""
    kb = np.array([[0.5, -2.0, 1.0], [-0.25, 3.0, 0.0], [2.0, 0.0, -1.0]])
    for c in range(3):
        qi = torch.zeros(1, 3)
        qi[0, c] = 1.0
        s = orc.block_scores(qi, kb, 3)
        assert np.array_equal(s, np.maximum(kb[:, c], 0.0)), (c, s)
    qi = torch.tensor([[0.3, -0.7, 0.2], [1.5, 0.25, -0.5]])
    s1 = orc.block_scores(qi, kb, 3)
    s2 = orc.block_scores(qi * 4, kb, 3)
    assert np.allclose(s2, 4 * s1, rtol=1e-12, atol=0)


# --------------------------------------------------------------------------- a3 brute force
def _brute_select(scores, k):
    n = len(scores)
    if n <= k:
        return list(range(n)) + [-1] * (k - n)
    best, best_sum = None, -math.inf
    for sub in itertools.combinations(range(n), k):  # lexicographic order
        tot = sum(scores[i] for i in sub)
        if tot > best_sum:  # strict: the lexicographically first maximiser is kept
            best, best_sum = sub, tot
    return list(best)


def pin_select_bruteforce(orc):
    """Sort-based top-k equals exhaustive subset search with a lexicographic tie-break."""
    rng = np.random.default_rng(7)
    for trial in range(400):
        n = int(rng.integers(0, 10))
        k = int(rng.integers(1, 8))
        if trial % 2:
            s = rng.integers(0, 3, size=n).astype(np.float64)  # heavy ties
        else:
            s = rng.random(n)
        got = orc.select(s, k).tolist()
        want = _brute_select(s.tolist(), k)
        assert got == want, (s, k, got, want)


# --------------------------------------------------------------------------- trailing block
def pin_token_set_rules(orc):
    """Selected blocks contribute whole; the trailing range [n_c*B, t] is always there."""
    assert orc.token_set(6, 2, np.array([1], np.int32)).tolist() == [2, 3, 6]
    assert orc.token_set(7, 2, np.array([1, 3], np.int32)).tolist() == [2, 3, 6, 7]
    assert orc.token_set(0, 4, np.array([-1, -1], np.int32)).tolist() == [0]
    assert orc.token_set(9, 4, np.array([0, -1], np.int32)).tolist() == [0, 1, 2, 3, 8, 9]


# --------------------------------------------------------------------------- a4 dense equivalence
def _dense_causal(cfg, inp, b=0):
    S = inp["q"].shape[1]
    G = cfg.Hq // cfg.Hkv
    q = inp["q"][b].transpose(0, 1)  # [Hq][S][d]
    k = inp["k"][b].repeat_interleave(G, dim=0)
    v = inp["v"][b].repeat_interleave(G, dim=0)
    mask = torch.ones(S, S, dtype=torch.bool).tril()
    scale = cfg.scale or 1.0 / math.sqrt(cfg.d)
    return _sdpa(q, k, v, scale, mask).transpose(0, 1).numpy()  # [S][Hq][d]


def pin_dense_equivalence(orc):
    """With top-k covering every complete block, QSA is dense causal GQA attention."""
    for dtype, S, B in [(torch.float32, 37, 4), (torch.bfloat16, 50, 8), (torch.float32, 64, 16)]:
        cfg = _cfg(block=B, topk=S // B + 1)
        inp = _rand_seq(cfg, S, seed=S, dtype=dtype)
        res = orc.run(cfg, inp)
        want = _dense_causal(cfg, inp)
        err = np.abs(res["o"][0] - want).max()
        assert err < 1e-12, (dtype, S, err)


def pin_sparse_equals_masked_sdpa(orc):
    """Sparse rows equal library attention under the mask of the selected token set."""
    cfg = _cfg(block=4, topk=2)
    S = 48
    inp = _rand_seq(cfg, S, seed=3)
    res = orc.run(cfg, inp)
    G = cfg.Hq // cfg.Hkv
    mask = torch.zeros(S, S, dtype=torch.bool)
    for t in range(S):
        for u in orc.token_set(t, cfg.block, res["sel"][0][t]).tolist():
            mask[t, u] = True
    q = inp["q"][0].transpose(0, 1)
    k = inp["k"][0].repeat_interleave(G, dim=0)
    v = inp["v"][0].repeat_interleave(G, dim=0)
    want = _sdpa(q, k, v, 1.0 / math.sqrt(cfg.d), mask).transpose(0, 1).numpy()
    assert np.abs(res["o"][0] - want).max() < 1e-12
    # and the selection really is sparse for late rows
    assert (res["sel"][0][S - 1] >= 0).sum() == cfg.topk


# --------------------------------------------------------------------------- invariants
def pin_causality(orc):
    """Perturbing any token after t (K, V, indexer keys) leaves row t bit-identical."""
    cfg = _cfg(block=4, topk=2)
    S, t = 40, 21
    inp = _rand_seq(cfg, S, seed=11)
    base = orc.run(cfg, inp, rows={0: [t]})
    pert = {k_: v_.clone() for k_, v_ in inp.items()}
    g = torch.Generator().manual_seed(5)
    pert["k"][0, :, t + 1:] += torch.randn(pert["k"][0, :, t + 1:].shape, generator=g)
    pert["v"][0, :, t + 1:] += torch.randn(pert["v"][0, :, t + 1:].shape, generator=g)
    pert["ki"][0, t + 1:] += torch.randn(pert["ki"][0, t + 1:].shape, generator=g)
    res = orc.run(cfg, pert, rows={0: [t]})
    assert np.array_equal(base["o"][0], res["o"][0])
    assert np.array_equal(base["sel"][0], res["sel"][0])


def pin_trailing_block(orc):
    """The incomplete trailing block is always attended, uncompressed, never a candidate."""
    cfg = _cfg(block=4, topk=1)
    S = 40
    inp = _rand_seq(cfg, S, seed=12)
    res = orc.run(cfg, inp)
    for t in range(S):
        n_c = (t + 1) // cfg.block
        sel = res["sel"][0][t]
        assert all(j < n_c for j in sel if j >= 0), (t, sel)
        assert (sel >= 0).sum() == min(n_c, cfg.topk)
    t = 22  # L = 23, trailing range [20, 22]
    for u in (20, 21, 22):
        pert = {k_: v_.clone() for k_, v_ in inp.items()}
        pert["v"][0, :, u] += 1.0
        r2 = orc.run(cfg, pert, rows={0: [t]})
        assert not np.array_equal(r2["o"][0][0], res["o"][0][t]), u
    # an unselected complete block does not influence the row
    unsel = [j for j in range((t + 1) // cfg.block) if j not in res["sel"][0][t]]
    pert = {k_: v_.clone() for k_, v_ in inp.items()}
    j = unsel[0]
    pert["v"][0, :, j * cfg.block:(j + 1) * cfg.block] += 1.0
    r3 = orc.run(cfg, pert, rows={0: [t]})
    assert np.array_equal(r3["o"][0][0], res["o"][0][t])


def pin_block_boundary_row(orc):
    """When L is a multiple of B the just-completed block competes in top-k: with a
    zero score and a small budget it drops out, and the row no longer sees itself."""
    cfg = _cfg(Hq=1, Hkv=1, d=4, Hi=1, di=2, block=2, topk=1)
    S = 4
    inp = _rand_seq(cfg, S, seed=1)
    inp["qi"][0, :, 0, :] = torch.tensor([1.0, 0.0])
    inp["ki"][0] = torch.tensor([[2.0, 0.0], [2.0, 0.0], [-1.0, 0.0], [-1.0, 0.0]])
    res = orc.run(cfg, inp, rows={0: [3]})
    assert res["sel"][0][0].tolist() == [0]  # block 1 scores max(0,-1)=0 < 2
    pert = {k_: v_.clone() for k_, v_ in inp.items()}
    pert["v"][0, :, 2:4] += 3.0
    r2 = orc.run(cfg, pert, rows={0: [3]})
    assert np.array_equal(r2["o"][0], res["o"][0])


def pin_gqa_repeat(orc):
    """Repeating each KV head for its query group (MHA) gives an identical result."""
    cfg = _cfg(Hq=6, Hkv=2, block=4, topk=2)
    inp = _rand_seq(cfg, 30, seed=13)
    a = orc.run(cfg, inp)
    G = cfg.Hq // cfg.Hkv
    mha = dict(inp)
    mha["k"] = inp["k"].repeat_interleave(G, dim=1).contiguous()
    mha["v"] = inp["v"].repeat_interleave(G, dim=1).contiguous()
    b = orc.run(_cfg(Hq=6, Hkv=6, block=4, topk=2), mha)
    assert np.array_equal(a["o"][0], b["o"][0])
    assert np.array_equal(a["sel"][0], b["sel"][0])


def pin_left_padding(orc):
    """A left-padded batch equals each sequence run alone; pad rows are zero / -1."""
    cfg = _cfg(block=4, topk=2)
    S = 36
    pads = [0, 5, 13]
    parts = [_rand_seq(cfg, S - p, seed=20 + i) for i, p in enumerate(pads)]
    batch = {}
    for key in ("q", "qi"):
        batch[key] = torch.stack([torch.cat([torch.full((p,) + parts[i][key].shape[2:], float("nan")),
                                             parts[i][key][0]]) for i, p in enumerate(pads)])
    for key in ("k", "v"):
        batch[key] = torch.stack([torch.cat([torch.full((cfg.Hkv, p, cfg.d), float("nan")),
                                             parts[i][key][0]], dim=1) for i, p in enumerate(pads)])
    batch["ki"] = torch.stack([torch.cat([torch.full((p, cfg.di), float("nan")), parts[i]["ki"][0]])
                               for i, p in enumerate(pads)])
    batch["kv_start"] = torch.tensor(pads, dtype=torch.int32)
    batch["kv_len"] = torch.tensor([S - p for p in pads], dtype=torch.int32)
    batch["q_first"] = -batch["kv_start"]
    res = orc.run(cfg, batch)
    for i, p in enumerate(pads):
        alone = orc.run(cfg, parts[i])
        assert np.array_equal(res["o"][i][p:], alone["o"][0])
        assert np.array_equal(res["sel"][i][p:], alone["sel"][0])
        assert np.all(res["o"][i][:p] == 0) and np.all(res["sel"][i][:p] == -1)


def pin_decode_equals_prefill_row(orc):
    """A decode step at length L equals prefill row L-1 of the same sequence."""
    cfg = _cfg(block=4, topk=2)
    S = 45
    inp = _rand_seq(cfg, S, seed=14)
    pre = orc.run(cfg, inp)
    for L in (1, 4, 17, 45):
        dec = dict(q=inp["q"][:, L - 1:L], qi=inp["qi"][:, L - 1:L],
                   k=inp["k"].clone(), v=inp["v"].clone(), ki=inp["ki"].clone(),
                   k_new=inp["k"][:, :, L - 1], v_new=inp["v"][:, :, L - 1],
                   ki_new=inp["ki"][:, L - 1], kv_start=torch.zeros(1, dtype=torch.int32),
                   kv_len=torch.tensor([L], dtype=torch.int32),
                   q_first=torch.tensor([L - 1], dtype=torch.int32))
        dec["k"][:, :, L - 1:] = float("nan")
        dec["v"][:, :, L - 1:] = float("nan")
        dec["ki"][:, L - 1:] = float("nan")
        r = orc.run(cfg, dec)
        assert np.array_equal(r["o"][0][0], pre["o"][0][L - 1]), L
        assert np.array_equal(r["sel"][0][0], pre["sel"][0][L - 1]), L


def pin_selection_scale_invariance(orc):
    """Scaling indexer queries or keys by a positive power of two leaves the selection unchanged."""
    cfg = _cfg(block=4, topk=3)
    inp = _rand_seq(cfg, 60, seed=15)
    a = orc.run(cfg, inp)
    for key in ("qi", "ki"):
        p = dict(inp)
        p[key] = inp[key] * 4.0
        b = orc.run(cfg, p)
        assert np.array_equal(a["sel"][0], b["sel"][0]), key


# --------------------------------------------------------------------------- projections + RoPE
def _pc(**kw):
    base = dict(Hq=4, Hkv=2, d=8, Hi=2, di=4, rope_theta=100.0, rd_attn=8, rd_idx=4)
    base.update(kw)
    return types.SimpleNamespace(**base)


def _proj_inputs(pc, n, D, seed):
    g = torch.Generator().manual_seed(seed)
    n_out = pc.Hq * pc.d + 2 * pc.Hkv * pc.d + pc.Hi * pc.di + pc.di
    return torch.randn(n, D, generator=g), torch.randn(n_out, D, generator=g) * 0.3


def pin_projection_is_the_matmul_at_position_zero(orc):
    """At position 0 every rotation is the identity: the stage is x W^T (library matmul
    in fp64), split into q, k, v, qi, ki by the stacked-row layout."""
    pc = _pc()
    x, w = _proj_inputs(pc, 5, 12, 0)
    out = orc.project_rope(pc, x, w, [0] * 5)
    y = (x.double() @ w.double().T).numpy()
    flat = np.concatenate([out["q"].reshape(5, -1), out["k"].reshape(5, -1), out["v"].reshape(5, -1),
                           out["qi"].reshape(5, -1), out["ki"]], axis=1)
    assert np.allclose(flat, y, rtol=1e-12, atol=1e-12)


def pin_rope_hand_worked(orc):
    """Head [1, 0, 0, 0], rd 4, theta 100: dim 0 pairs with dim 2 at frequency 1, dim 1
    with dim 3 at frequency 100^(-1/2) = 0.1. At pos pi/2 the first pair turns a
    quarter: [0, 0, 1, 0]; [0, 1, 0, 0] at pos 5 turns by 0.5 rad: [0, cos .5, 0, sin .5]."""
    a = orc.rope_head([1, 0, 0, 0], math.pi / 2, 100.0, 4)
    assert np.allclose(a, [0, 0, 1, 0], atol=1e-15), a
    b = orc.rope_head([0, 1, 0, 0], 5.0, 100.0, 4)
    assert np.allclose(b, [0, math.cos(0.5), 0, math.sin(0.5)], atol=1e-15), b
    c = orc.rope_head([0, 0, 2, 0], 1.0, 100.0, 4)  # the second half rotates the other way
    assert np.allclose(c, [-2 * math.sin(1.0), 0, 2 * math.cos(1.0), 0], atol=1e-15), c


def pin_rope_norm_and_relative_position(orc):
    """A rotation keeps each head's norm, and q . k after RoPE depends only on the
    distance between the two positions."""
    g = np.random.default_rng(3)
    q, k = g.standard_normal(16), g.standard_normal(16)
    for p in (0, 1, 7, 1000):
        assert abs(np.linalg.norm(orc.rope_head(q, p, 1e4, 16)) - np.linalg.norm(q)) < 1e-12
    d1 = orc.rope_head(q, 9, 1e4, 16) @ orc.rope_head(k, 4, 1e4, 16)
    d2 = orc.rope_head(q, 1009, 1e4, 16) @ orc.rope_head(k, 1004, 1e4, 16)
    d3 = orc.rope_head(q, 9, 1e4, 16) @ orc.rope_head(k, 5, 1e4, 16)
    assert abs(d1 - d2) < 1e-10 and abs(d1 - d3) > 1e-3, (d1, d2, d3)


def pin_rope_partial_and_which_heads(orc):
    """With rotary dims rd < d only the first rd dims of a head move; v is never
    rotated; the indexer heads rotate with rd_idx and stay put with rd_idx = 0."""
    pc = _pc(rd_attn=4, rd_idx=2)
    x, w = _proj_inputs(pc, 3, 10, 1)
    at0 = orc.project_rope(pc, x, w, [0, 0, 0])
    at5 = orc.project_rope(pc, x, w, [5, 5, 5])
    for name in ("q", "k"):
        assert np.allclose(at5[name][..., 4:], at0[name][..., 4:], atol=1e-12)
        assert not np.allclose(at5[name][..., :4], at0[name][..., :4])
    assert np.allclose(at5["v"], at0["v"], atol=1e-12)
    assert np.allclose(at5["qi"][..., 2:], at0["qi"][..., 2:], atol=1e-12)
    assert not np.allclose(at5["qi"][..., :2], at0["qi"][..., :2])
    assert not np.allclose(at5["ki"][..., :2], at0["ki"][..., :2])
    off = orc.project_rope(_pc(rd_attn=4, rd_idx=0), x, w, [5, 5, 5])
    assert np.allclose(off["qi"], at0["qi"], atol=1e-12) and np.allclose(off["ki"], at0["ki"], atol=1e-12)
    # each row rotates at its own position: row 1 of a mixed call equals row 1 at its position alone
    mixed = orc.project_rope(pc, x, w, [0, 5, 0])
    assert np.allclose(mixed["q"][1], at5["q"][1], atol=1e-12) and np.allclose(mixed["q"][0], at0["q"][0])


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
