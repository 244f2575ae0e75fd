"""fp64 CPU oracle for the QSA hot path -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may
import this package.  It wraps ``qsa_oracle.c`` (plain C, double precision) with
ctypes.  The wrapper only slices and reorders inputs (per-sequence views, the
decode token appended to its cache); every arithmetic step of the method lives
in the C file, which shares nothing with the CUDA library.

Definitions follow the Hugging Face Transformers model doc "Qwen4-Exp": the
intro paragraph on QSA and the Qwen4ExpTextConfig indexer_* parameters; the
readings of open points are documented in qsa_oracle.c.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Dict, Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libqsa_oracle.so")
_lib = None
_lock = threading.Lock()

_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)
_I64 = ctypes.POINTER(ctypes.c_int64)
_V = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (OpenMP) if it is missing or stale."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            L.qsa_oracle_compress.argtypes = [_V, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                              ctypes.c_int, _D]
            L.qsa_oracle_block_scores.argtypes = [_V, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                  _D, ctypes.c_int64, _D]
            L.qsa_oracle_select.argtypes = [_D, ctypes.c_int64, ctypes.c_int, _I32]
            L.qsa_oracle_select.restype = ctypes.c_int
            L.qsa_oracle_token_set.argtypes = [ctypes.c_int64, ctypes.c_int, _I32, ctypes.c_int,
                                               _I64]
            L.qsa_oracle_token_set.restype = ctypes.c_int64
            L.qsa_oracle_attend.argtypes = [_V, _V, _V, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int64, ctypes.c_double, _I64,
                                            ctypes.c_int64, _D]
            L.qsa_oracle_sequence.argtypes = [_V, _V, _I64, ctypes.c_int64, _V, _V, _V,
                                              ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_double, _D, _I32, _D,
                                              ctypes.c_int]
            L.qsa_oracle_sequence_scores.argtypes = [_V, _I64, ctypes.c_int64, _V, ctypes.c_int64,
                                                     ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                     ctypes.c_int, _D, ctypes.c_int]
            L.qsa_oracle_max_threads.restype = ctypes.c_int
            L.qsa_oracle_rope_head.argtypes = [_D, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double]
            L.qsa_oracle_project_rope.argtypes = [_V, _V, ctypes.c_int, ctypes.c_int64, ctypes.c_int, _I64,
                                                  ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _D,
                                                  ctypes.c_int]
            _lib = L
    return _lib


def max_threads() -> int:
    return int(lib().qsa_oracle_max_threads())


# ----------------------------------------------------------------------------
# marshalling: torch/numpy -> raw element arrays the C oracle reads exactly
# ----------------------------------------------------------------------------

def _raw(x) -> tuple:
    """Return (contiguous numpy array of raw elements, dtype code)."""
    if isinstance(x, np.ndarray):
        x = torch.from_numpy(x)
    x = x.detach().cpu().contiguous()
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).numpy(), 1
    if x.dtype == torch.float32:
        return x.numpy(), 0
    raise TypeError(f"oracle inputs must be fp32 or bf16, got {x.dtype}")


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dptr(a: np.ndarray):
    return a.ctypes.data_as(_D)


# ----------------------------------------------------------------------------
# stage functions (each a thin call into the C oracle)
# ----------------------------------------------------------------------------

def compress(ki, block: int) -> np.ndarray:
    """k̄ for the complete blocks of one sequence's indexer keys ki [n_keys][di]."""
    a, dt = _raw(ki)
    n, di = a.shape
    out = np.zeros((n // block, di), dtype=np.float64)
    lib().qsa_oracle_compress(_ptr(a), dt, n, di, block, _dptr(out))
    return out


def block_scores(qi_row, kbar: np.ndarray, n_c: int) -> np.ndarray:
    """Scores of the first n_c compressed blocks for one query's indexer heads [Hi][di]."""
    a, dt = _raw(qi_row)
    Hi, di = a.shape
    kb = np.ascontiguousarray(kbar, dtype=np.float64)
    out = np.zeros(max(n_c, 1), dtype=np.float64)
    lib().qsa_oracle_block_scores(_ptr(a), dt, Hi, di, _dptr(kb), n_c, _dptr(out))
    return out[:n_c]


def select(scores: Sequence[float], k: int) -> np.ndarray:
    s = np.ascontiguousarray(np.asarray(scores, dtype=np.float64).reshape(-1))
    sel = np.zeros(k, dtype=np.int32)
    lib().qsa_oracle_select(_dptr(s), s.shape[0], k, sel.ctypes.data_as(_I32))
    return sel


def token_set(t: int, block: int, sel: np.ndarray) -> np.ndarray:
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    k = sel.shape[0]
    toks = np.zeros(k * block + block, dtype=np.int64)
    n = lib().qsa_oracle_token_set(t, block, sel.ctypes.data_as(_I32), k, toks.ctypes.data_as(_I64))
    return toks[:n].copy()


def attend(q_row, k_seq, v_seq, scale: float, toks: np.ndarray) -> np.ndarray:
    """q_row [Hq][d]; k_seq, v_seq [Hkv][L][d]; returns fp64 [Hq][d]."""
    qa, dt = _raw(q_row)
    ka, dt2 = _raw(k_seq)
    va, dt3 = _raw(v_seq)
    assert dt == dt2 == dt3
    Hq, d = qa.shape
    Hkv, L, _ = ka.shape
    toks = np.ascontiguousarray(toks, dtype=np.int64)
    out = np.zeros((Hq, d), dtype=np.float64)
    lib().qsa_oracle_attend(_ptr(qa), _ptr(ka), _ptr(va), dt, Hq, Hkv, d, L, scale,
                            toks.ctypes.data_as(_I64), toks.shape[0], _dptr(out))
    return out


# ----------------------------------------------------------------------------
# whole path over a batch (prefill with left padding, or one decode step)
# ----------------------------------------------------------------------------

def _sequence_views(inp: Dict[str, torch.Tensor], b: int, decode: bool):
    """Per-sequence key planes at relative positions 0..L-1 (slicing only)."""
    s0 = int(inp["kv_start"][b])
    L = int(inp["kv_len"][b])
    if decode:
        k = torch.cat([inp["k"][b, :, s0:s0 + L - 1], inp["k_new"][b][:, None]], dim=1)
        v = torch.cat([inp["v"][b, :, s0:s0 + L - 1], inp["v_new"][b][:, None]], dim=1)
        ki = torch.cat([inp["ki"][b, s0:s0 + L - 1], inp["ki_new"][b][None]], dim=0)
    else:
        k = inp["k"][b, :, s0:s0 + L]
        v = inp["v"][b, :, s0:s0 + L]
        ki = inp["ki"][b, s0:s0 + L]
    return k, v, ki, L


def run(cfg, inp: Dict[str, torch.Tensor], rows: Optional[Dict[int, Sequence[int]]] = None,
        decode: Optional[bool] = None, n_threads: int = 0, want_kbar: bool = False):
    """Run the oracle over a batch.

    cfg: object with Hq, Hkv, d, Hi, di, block, topk and (optionally) scale.
    inp: tensors laid out as in the workload generator.
    rows: optional {b: [query row indices]} to compute only a sample.
    Returns dict(o={b: fp64 [n_rows][Hq][d]}, sel={b: int32 [n_rows][k]},
    rows={b: row indices}, kbar={b: fp64} if want_kbar).
    """
    if decode is None:
        decode = "k_new" in inp
    scale = getattr(cfg, "scale", None) or 1.0 / float(np.sqrt(cfg.d))
    n_q = inp["q"].shape[1]
    out_o, out_sel, out_rows, out_kbar = {}, {}, {}, {}
    for b in range(inp["q"].shape[0]):
        k, v, ki, L = _sequence_views(inp, b, decode)
        r_idx = list(range(n_q)) if rows is None else list(rows.get(b, []))
        if not r_idx:
            continue
        r_t = torch.tensor(r_idx, dtype=torch.long)
        q = inp["q"][b].index_select(0, r_t)
        qi = inp["qi"][b].index_select(0, r_t)
        t_pos = np.ascontiguousarray(np.asarray(r_idx, dtype=np.int64) + int(inp["q_first"][b]))
        qa, dt = _raw(q)
        qia, _ = _raw(qi)
        ka, _ = _raw(k)
        va, _ = _raw(v)
        kia, _ = _raw(ki)
        o = np.zeros((len(r_idx), cfg.Hq, cfg.d), dtype=np.float64)
        sel = np.zeros((len(r_idx), cfg.topk), dtype=np.int32)
        kbar = np.zeros((max(L // cfg.block, 1), cfg.di), dtype=np.float64)
        lib().qsa_oracle_sequence(_ptr(qa), _ptr(qia), t_pos.ctypes.data_as(_I64), len(r_idx),
                                  _ptr(ka), _ptr(va), _ptr(kia), L, L, dt, cfg.Hq, cfg.Hkv, cfg.d,
                                  cfg.Hi, cfg.di, cfg.block, cfg.topk, scale, _dptr(o),
                                  sel.ctypes.data_as(_I32), _dptr(kbar), n_threads)
        out_o[b], out_sel[b], out_rows[b] = o, sel, r_idx
        if want_kbar:
            out_kbar[b] = kbar[: L // cfg.block]
    res = dict(o=out_o, sel=out_sel, rows=out_rows)
    if want_kbar:
        res["kbar"] = out_kbar
    return res


def scores(cfg, inp: Dict[str, torch.Tensor], b: int, r_idx: Sequence[int],
           decode: Optional[bool] = None, n_threads: int = 0) -> np.ndarray:
    """fp64 scores [len(r_idx)][n_blocks] of sequence b (non-candidates are -1)."""
    if decode is None:
        decode = "k_new" in inp
    _, _, ki, L = _sequence_views(inp, b, decode)
    r_t = torch.tensor(list(r_idx), dtype=torch.long)
    qia, dt = _raw(inp["qi"][b].index_select(0, r_t))
    kia, _ = _raw(ki)
    t_pos = np.ascontiguousarray(np.asarray(r_idx, dtype=np.int64) + int(inp["q_first"][b]))
    nb = L // cfg.block
    out = np.zeros((len(r_idx), max(nb, 1)), dtype=np.float64)
    lib().qsa_oracle_sequence_scores(_ptr(qia), t_pos.ctypes.data_as(_I64), len(r_idx), _ptr(kia),
                                     L, dt, cfg.Hi, cfg.di, cfg.block, _dptr(out), n_threads)
    return out[:, :nb]


def rope_head(h, pos: float, theta: float, rd: int) -> np.ndarray:
    """One head vector rotated at position pos (rotate-half form, first rd dims)."""
    out = np.ascontiguousarray(np.asarray(h, dtype=np.float64).copy())
    lib().qsa_oracle_rope_head(_dptr(out), out.shape[0], rd, float(pos), float(theta))
    return out


def project_rope(pc, x, w, pos, n_threads: int = 0) -> Dict[str, np.ndarray]:
    """Projections of the rows x [n][D] by the stacked weights w [n_out][D] and RoPE at
    positions pos [n]. pc: Hq, Hkv, d, Hi, di, rope_theta, rd_attn, rd_idx.
    Returns fp64 q [n][Hq][d], k [n][Hkv][d], v [n][Hkv][d], qi [n][Hi][di], ki [n][di]."""
    xa, dt = _raw(x)
    wa, dt2 = _raw(w)
    assert dt == dt2
    n, D = xa.shape
    n_out = pc.Hq * pc.d + 2 * pc.Hkv * pc.d + pc.Hi * pc.di + pc.di
    assert wa.shape == (n_out, D), (wa.shape, n_out, D)
    p = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    y = np.zeros((n, n_out), dtype=np.float64)
    lib().qsa_oracle_project_rope(_ptr(xa), _ptr(wa), dt, n, D, p.ctypes.data_as(_I64), float(pc.rope_theta),
                                  pc.Hq, pc.Hkv, pc.d, pc.Hi, pc.di, pc.rd_attn, pc.rd_idx, _dptr(y), n_threads)
    a, b = 0, pc.Hq * pc.d
    out = {"q": y[:, a:b].reshape(n, pc.Hq, pc.d)}
    a, b = b, b + pc.Hkv * pc.d
    out["k"] = y[:, a:b].reshape(n, pc.Hkv, pc.d)
    a, b = b, b + pc.Hkv * pc.d
    out["v"] = y[:, a:b].reshape(n, pc.Hkv, pc.d)
    a, b = b, b + pc.Hi * pc.di
    out["qi"] = y[:, a:b].reshape(n, pc.Hi, pc.di)
    out["ki"] = y[:, b:b + pc.di]
    return out


def attend_selection(cfg, inp: Dict[str, torch.Tensor], b: int, r_idx: Sequence[int],
                     sel_rows: np.ndarray, decode: Optional[bool] = None) -> np.ndarray:
    """fp64 attention outputs [len(r_idx)][Hq][d] of sequence b's query rows r_idx over
    the token sets that the given selections (sel_rows [len(r_idx)][k], e.g. another
    implementation's) define, together with each row's trailing range."""
    if decode is None:
        decode = "k_new" in inp
    scale = getattr(cfg, "scale", None) or 1.0 / float(np.sqrt(cfg.d))
    k, v, _, L = _sequence_views(inp, b, decode)
    ka, dt = _raw(k)
    va, _ = _raw(v)
    out = np.zeros((len(r_idx), cfg.Hq, cfg.d), dtype=np.float64)
    for i, r in enumerate(r_idx):
        t = int(r) + int(inp["q_first"][b])
        toks = token_set(t, cfg.block, np.asarray(sel_rows[i], dtype=np.int32))
        qa, _ = _raw(inp["q"][b, r])
        o = np.zeros((cfg.Hq, cfg.d), dtype=np.float64)
        lib().qsa_oracle_attend(_ptr(qa), _ptr(ka), _ptr(va), dt, cfg.Hq, cfg.Hkv, cfg.d, L, scale,
                                toks.ctypes.data_as(_I64), toks.shape[0], _dptr(o))
        out[i] = o
    return out


class use_library:
    """Context manager: route oracle calls to another build of qsa_oracle.c (used by
    the mutation test, which plants mistakes in a copy of the oracle on the CPU)."""

    def __init__(self, path: str):
        self.path = path
        self.saved = None

    def __enter__(self):
        global _lib
        lib()  # make sure the default library and its signatures are set up
        saved = _lib
        other = ctypes.CDLL(self.path)
        for name in ("qsa_oracle_compress", "qsa_oracle_block_scores", "qsa_oracle_select",
                     "qsa_oracle_token_set", "qsa_oracle_attend", "qsa_oracle_sequence",
                     "qsa_oracle_sequence_scores", "qsa_oracle_max_threads", "qsa_oracle_rope_head",
                     "qsa_oracle_project_rope"):
            f, g = getattr(saved, name), getattr(other, name)
            g.argtypes, g.restype = f.argtypes, f.restype
        self.saved = saved
        with _lock:
            _lib = other
        return self

    def __exit__(self, *exc):
        global _lib
        with _lock:
            _lib = self.saved
        return False
