"""Python binding of the QSA C ABI (include/qsa.h) -- argument marshalling only.

Each function has the name of the C entry point it calls and takes torch CUDA
tensors; it checks shapes and dtypes, passes raw device pointers and the
current CUDA stream, and raises QSAError on a non-OK status. Every step of the
path runs in libqsa.so; there is no fallback: if the library is missing or
fails to load, the import of this module raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# QSA_LIBRARY may name another in-tree build of the library (libqsa_debug.so: the
# same entry points with device-side checks of every selection list read).
LIB_PATH = os.path.join(_PKG, os.environ.get("QSA_LIBRARY", "libqsa.so"))

QSA_OK, QSA_ERR_INVALID_ARG, QSA_ERR_UNSUPPORTED, QSA_ERR_CUDA, QSA_ERR_TIMEOUT, QSA_ERR_DEVICE_CHECK = range(6)
QSA_DTYPE_BF16, QSA_DTYPE_FP32 = 0, 1
QSA_PREFILL, QSA_DECODE = 0, 1


class QSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = f" [{qsa_last_error()}]" if status == QSA_ERR_CUDA else ""
        super().__init__(f"{where}: {status_string(status)} (status {status}){detail}")


class qsa_config_t(ctypes.Structure):
    _fields_ = [("num_attention_heads", ctypes.c_int32), ("num_key_value_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("indexer_n_heads", ctypes.c_int32),
                ("indexer_kv_heads", ctypes.c_int32), ("indexer_head_dim", ctypes.c_int32),
                ("indexer_budget", ctypes.c_int32), ("indexer_compress_ratio", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("dtype", ctypes.c_int32)]


class qsa_proj_config_t(ctypes.Structure):
    _fields_ = [("hidden_size", ctypes.c_int32), ("rope_theta", ctypes.c_float), ("rotary_dim", ctypes.c_int32),
                ("indexer_rotary_dim", ctypes.c_int32)]


class qsa_tensors_t(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q", ctypes.c_int32), ("kv_cap", ctypes.c_int32),
                ("q", ctypes.c_void_p), ("qi", ctypes.c_void_p), ("k_cache", ctypes.c_void_p),
                ("v_cache", ctypes.c_void_p), ("ki_cache", ctypes.c_void_p),
                ("kbar_cache", ctypes.c_void_p), ("kbar_blocks", ctypes.c_void_p),
                ("k_new", ctypes.c_void_p), ("v_new", ctypes.c_void_p), ("ki_new", ctypes.c_void_p),
                ("kv_start", ctypes.c_void_p), ("kv_len", ctypes.c_void_p), ("q_first", ctypes.c_void_p),
                ("sel", ctypes.c_void_p), ("out", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"QSA CUDA library not built: {LIB_PATH} is missing "
                          "(run block_sparse_long_15_b200.build.build())")
    L = ctypes.CDLL(LIB_PATH)
    P, V, I, S = ctypes.POINTER, ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    cfgp = P(qsa_config_t)
    sig = {
        "qsa_config_validate": ([cfgp], I),
        "qsa_topk_blocks": ([cfgp], I),
        "qsa_status_string": ([I], ctypes.c_char_p),
        "qsa_workspace_size": ([cfgp, I, I, I, I, P(S)], I),
        "qsa_compress_blocks": ([cfgp, V, V, V, V, I, I, V, V, V], I),
        "qsa_index_score_topk": ([cfgp, V, V, V, V, I, I, I, V, V, S, V], I),
        "qsa_sparse_attn": ([cfgp, V, V, V, V, V, V, V, I, I, I, V, V, S, V], I),
        "qsa_index_scores": ([cfgp, V, V, V, V, I, I, I, V, V, S, V], I),
        "qsa_project": ([cfgp, P(qsa_proj_config_t), V, V, V, I, I, V, V, V, V, V, I, I, V, S, V], I),
        "qsa_select_topk": ([cfgp, V, V, V, I, I, I, V, V, S, V], I),
        "qsa_forward": ([cfgp, I, P(qsa_tensors_t), V, S, V], I),
        "qsa_read_device_status": ([V, V, P(I)], I),
        "qsa_abi_version": ([], I),
        "qsa_attn_kernel_name": ([cfgp, I], ctypes.c_char_p),
        "qsa_kernel_launch_count": ([], ctypes.c_uint64),
        "qsa_last_error": ([], ctypes.c_char_p),
        "qsa_sparse_attn_decode_noalloc": ([cfgp, V, V, V, V, V, V, I, I, V, V], I),
        "qsa_selftest_wait_timeout": ([V, ctypes.c_int64, V], I),
        "qsa_offload_staging_size": ([cfgp, I, P(S)], I),
        "qsa_decode_offload": ([cfgp, P(qsa_tensors_t), V, S, V, S, V], I),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes, f.restype = args, res
    return L


_lib = _load()

EXPORTED = ("qsa_config_validate", "qsa_topk_blocks", "qsa_status_string", "qsa_workspace_size",
            "qsa_compress_blocks", "qsa_index_score_topk", "qsa_sparse_attn", "qsa_forward",
            "qsa_read_device_status", "qsa_abi_version", "qsa_attn_kernel_name",
            "qsa_kernel_launch_count", "qsa_last_error", "qsa_sparse_attn_decode_noalloc",
            "qsa_selftest_wait_timeout", "qsa_offload_staging_size", "qsa_decode_offload",
            "qsa_index_scores", "qsa_select_topk", "qsa_project")

# Size of the library's fixed decode scratch (QSA_NOALLOC_SCRATCH_BYTES in qsa.h).
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


def library() -> ctypes.CDLL:
    return _lib


def status_string(status: int) -> str:
    return _lib.qsa_status_string(status).decode()


def _check(status: int, where: str):
    if status != QSA_OK:
        raise QSAError(status, where)


def make_config(Hq: int, Hkv: int, d: int, Hi: int, di: int, block: int, topk: int,
                dtype: str = "bf16", scale: float = 0.0, indexer_kv_heads: int = 1,
                budget: Optional[int] = None) -> qsa_config_t:
    return qsa_config_t(Hq, Hkv, d, Hi, indexer_kv_heads, di,
                        budget if budget is not None else topk * block, block, scale,
                        QSA_DTYPE_BF16 if dtype == "bf16" else QSA_DTYPE_FP32)


def config_for(w) -> qsa_config_t:
    """Config of a workload description (fields Hq, Hkv, d, Hi, di, block, topk, dtype)."""
    return make_config(w.Hq, w.Hkv, w.d, w.Hi, w.di, w.block, w.topk, w.dtype)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _p(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("QSA tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("QSA tensors must be contiguous")
    return t.data_ptr()


def _elem(cfg: qsa_config_t) -> torch.dtype:
    return torch.bfloat16 if cfg.dtype == QSA_DTYPE_BF16 else torch.float32


def _want(t: torch.Tensor, dtype: torch.dtype, shape, name: str):
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


def _want_lengths(batch: int, **named):
    """Per-sequence int32 vectors of `batch` entries (kv_start, kv_len, q_first, ...)."""
    for name, t in named.items():
        if t is None:
            raise ValueError(f"{name}: required")
        _want(t, torch.int32, (batch,), name)


# --------------------------------------------------------------------------- entry points
def qsa_config_validate(cfg: qsa_config_t) -> int:
    return _lib.qsa_config_validate(ctypes.byref(cfg))


def qsa_topk_blocks(cfg: qsa_config_t) -> int:
    return _lib.qsa_topk_blocks(ctypes.byref(cfg))


def qsa_abi_version() -> int:
    return _lib.qsa_abi_version()


def qsa_attn_kernel_name(cfg: qsa_config_t, mode: int = QSA_PREFILL) -> str:
    return _lib.qsa_attn_kernel_name(ctypes.byref(cfg), mode).decode()


def qsa_last_error() -> str:
    return _lib.qsa_last_error().decode()


def qsa_kernel_launch_count() -> int:
    return _lib.qsa_kernel_launch_count()


def qsa_workspace_size(cfg: qsa_config_t, mode: int, batch: int, n_q: int, kv_cap: int) -> int:
    out = ctypes.c_size_t(0)
    _check(_lib.qsa_workspace_size(ctypes.byref(cfg), mode, batch, n_q, kv_cap, ctypes.byref(out)),
           "qsa_workspace_size")
    return out.value


def alloc_workspace(cfg: qsa_config_t, mode: int, batch: int, n_q: int, kv_cap: int,
                    device=None) -> torch.Tensor:
    """Zeroed workspace bytes (the status word must start at zero)."""
    n = qsa_workspace_size(cfg, mode, batch, n_q, kv_cap)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def qsa_compress_blocks(cfg, ki, kv_start, kv_len, kbar, blocks_done=None, kbar_blocks=None, stream=None):
    """k̄ of the complete blocks; kbar_blocks (optional, int32 [batch]) receives kv_len // B."""
    batch, kv_cap = ki.shape[0], ki.shape[1]
    _want(ki, _elem(cfg), (batch, kv_cap, cfg.indexer_head_dim), "ki")
    _want(kbar, torch.float32, (batch, kv_cap // cfg.indexer_compress_ratio, cfg.indexer_head_dim), "kbar")
    _want_lengths(batch, kv_start=kv_start, kv_len=kv_len)
    if blocks_done is not None:
        _want_lengths(batch, blocks_done=blocks_done)
    if kbar_blocks is not None:
        _want_lengths(batch, kbar_blocks=kbar_blocks)
    _check(_lib.qsa_compress_blocks(ctypes.byref(cfg), _p(ki), _p(kv_start), _p(kv_len), _p(blocks_done),
                                    batch, kv_cap, _p(kbar), _p(kbar_blocks), _stream(stream)),
           "qsa_compress_blocks")


def qsa_index_score_topk(cfg, qi, kbar, kv_len, q_first, kv_cap, sel, workspace, stream=None):
    batch, n_q = qi.shape[0], qi.shape[1]
    _want(qi, _elem(cfg), (batch, n_q, cfg.indexer_n_heads, cfg.indexer_head_dim), "qi")
    _want(sel, torch.int32, (batch, n_q, qsa_topk_blocks(cfg)), "sel")
    _want(kbar, torch.float32, (batch, kv_cap // cfg.indexer_compress_ratio, cfg.indexer_head_dim), "kbar")
    _want_lengths(batch, kv_len=kv_len, q_first=q_first)
    _check(_lib.qsa_index_score_topk(ctypes.byref(cfg), _p(qi), _p(kbar), _p(kv_len), _p(q_first), batch,
                                     n_q, kv_cap, _p(sel), _p(workspace), workspace.numel(),
                                     _stream(stream)), "qsa_index_score_topk")


def qsa_project(cfg, pc: qsa_proj_config_t, x, w, q_first, q, qi, k, v, ki, kv_row0: int = 0, workspace=None,
                stream=None):
    """Projections of x [batch][n_tok][D] by the stacked weights w and RoPE, written to
    q [batch][n_tok][Hq][d], qi [batch][n_tok][Hi][di], k / v [batch][Hkv][kv_cap][d] and
    ki [batch][kv_cap][di] (rows kv_row0 + r)."""
    batch, n_tok, D = x.shape
    kv_cap = k.shape[2]
    n_out = (cfg.num_attention_heads * cfg.head_dim + 2 * cfg.num_key_value_heads * cfg.head_dim
             + cfg.indexer_n_heads * cfg.indexer_head_dim + cfg.indexer_head_dim)
    dt = _elem(cfg)
    _want(x, dt, (batch, n_tok, pc.hidden_size), "x")
    _want(w, dt, (n_out, pc.hidden_size), "w")
    _want(q, dt, (batch, n_tok, cfg.num_attention_heads, cfg.head_dim), "q")
    _want(qi, dt, (batch, n_tok, cfg.indexer_n_heads, cfg.indexer_head_dim), "qi")
    _want(k, dt, (batch, cfg.num_key_value_heads, kv_cap, cfg.head_dim), "k")
    _want(v, dt, (batch, cfg.num_key_value_heads, kv_cap, cfg.head_dim), "v")
    _want(ki, dt, (batch, kv_cap, cfg.indexer_head_dim), "ki")
    _want_lengths(batch, q_first=q_first)
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=x.device)
    _check(_lib.qsa_project(ctypes.byref(cfg), ctypes.byref(pc), _p(x), _p(w), _p(q_first), batch, n_tok, _p(q),
                            _p(qi), _p(k), _p(v), _p(ki), kv_cap, kv_row0, _p(workspace), workspace.numel(),
                            _stream(stream)), "qsa_project")
    return workspace


def qsa_index_scores(cfg, qi, kbar, kv_len, q_first, kv_cap, scores, workspace, stream=None):
    """Scores over the heads in qi (a shard of the indexer query heads), written to
    scores [batch][n_q][kv_cap // B] fp32 for each real row's candidate blocks."""
    batch, n_q = qi.shape[0], qi.shape[1]
    nb = kv_cap // cfg.indexer_compress_ratio
    _want(qi, _elem(cfg), (batch, n_q, cfg.indexer_n_heads, cfg.indexer_head_dim), "qi")
    _want(kbar, torch.float32, (batch, nb, cfg.indexer_head_dim), "kbar")
    _want(scores, torch.float32, (batch, n_q, nb), "scores")
    _want_lengths(batch, kv_len=kv_len, q_first=q_first)
    _check(_lib.qsa_index_scores(ctypes.byref(cfg), _p(qi), _p(kbar), _p(kv_len), _p(q_first), batch, n_q, kv_cap,
                                 _p(scores), _p(workspace), workspace.numel(), _stream(stream)), "qsa_index_scores")


def qsa_select_topk(cfg, scores, kv_len, q_first, kv_cap, sel, workspace, stream=None):
    """Top-k blocks of each real row from a score matrix [batch][n_q][kv_cap // B] fp32."""
    batch, n_q = scores.shape[0], scores.shape[1]
    _want(scores, torch.float32, (batch, n_q, kv_cap // cfg.indexer_compress_ratio), "scores")
    _want(sel, torch.int32, (batch, n_q, qsa_topk_blocks(cfg)), "sel")
    _want_lengths(batch, kv_len=kv_len, q_first=q_first)
    _check(_lib.qsa_select_topk(ctypes.byref(cfg), _p(scores), _p(kv_len), _p(q_first), batch, n_q, kv_cap, _p(sel),
                                _p(workspace), workspace.numel(), _stream(stream)), "qsa_select_topk")


def qsa_sparse_attn(cfg, q, k, v, sel, kv_start, kv_len, q_first, out, workspace, stream=None):
    batch, n_q = q.shape[0], q.shape[1]
    kv_cap = k.shape[2]
    dt = _elem(cfg)
    _want(q, dt, (batch, n_q, cfg.num_attention_heads, cfg.head_dim), "q")
    _want(k, dt, (batch, cfg.num_key_value_heads, kv_cap, cfg.head_dim), "k")
    _want(v, dt, (batch, cfg.num_key_value_heads, kv_cap, cfg.head_dim), "v")
    _want(out, dt, (batch, n_q, cfg.num_attention_heads, cfg.head_dim), "out")
    _want(sel, torch.int32, (batch, n_q, qsa_topk_blocks(cfg)), "sel")
    _want_lengths(batch, kv_start=kv_start, kv_len=kv_len, q_first=q_first)
    _check(_lib.qsa_sparse_attn(ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(sel), _p(kv_start), _p(kv_len),
                                _p(q_first), batch, n_q, kv_cap, _p(out), _p(workspace),
                                workspace.numel(), _stream(stream)), "qsa_sparse_attn")


def qsa_forward(cfg, mode: int, t: Dict[str, torch.Tensor], workspace, stream=None):
    """t: q, qi, k_cache, v_cache, ki_cache, kbar_cache, kbar_blocks, kv_start, kv_len,
    q_first (prefill), k_new / v_new / ki_new (decode), sel, out."""
    q = t["q"]
    batch, n_q = q.shape[0], q.shape[1]
    kv_cap = t["k_cache"].shape[2]
    dt = _elem(cfg)
    for name in ("q", "qi", "k_cache", "v_cache", "ki_cache", "out"):
        if t[name].dtype != dt:
            raise ValueError(f"{name}: dtype {t[name].dtype}, expected {dt}")
    T = qsa_tensors_t(batch, n_q, kv_cap, _p(q), _p(t["qi"]), _p(t["k_cache"]), _p(t["v_cache"]),
                      _p(t["ki_cache"]), _p(t["kbar_cache"]), _p(t["kbar_blocks"]),
                      _p(t.get("k_new")), _p(t.get("v_new")), _p(t.get("ki_new")),
                      _p(t["kv_start"]), _p(t["kv_len"]), _p(t.get("q_first")), _p(t["sel"]),
                      _p(t["out"]))
    _check(_lib.qsa_forward(ctypes.byref(cfg), mode, ctypes.byref(T), _p(workspace), workspace.numel(),
                            _stream(stream)), "qsa_forward")


def qsa_sparse_attn_decode_noalloc(cfg, q, k, v, sel, kv_start, kv_len, out, stream=None):
    """Decode attention with no workspace: for callers that cannot allocate device
    memory of their own (a plugin given only its inputs and outputs, a server whose
    memory is all in its own pool). The partials live in a fixed array inside the
    library; calls that overlap on the GPU race on it."""
    batch = q.shape[0]
    kv_cap = k.shape[2]
    dt = _elem(cfg)
    _want(q, dt, (batch, 1, cfg.num_attention_heads, cfg.head_dim), "q")
    _want(k, dt, (batch, cfg.num_key_value_heads, kv_cap, cfg.head_dim), "k")
    _want(v, dt, (batch, cfg.num_key_value_heads, kv_cap, cfg.head_dim), "v")
    _want(sel, torch.int32, (batch, 1, qsa_topk_blocks(cfg)), "sel")
    _want_lengths(batch, kv_start=kv_start, kv_len=kv_len)
    _want(out, dt, (batch, 1, cfg.num_attention_heads, cfg.head_dim), "out")
    _check(_lib.qsa_sparse_attn_decode_noalloc(ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(sel), _p(kv_start),
                                               _p(kv_len), batch, kv_cap, _p(out), _stream(stream)),
           "qsa_sparse_attn_decode_noalloc")


def qsa_offload_staging_size(cfg, batch: int) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.qsa_offload_staging_size(ctypes.byref(cfg), batch, ctypes.byref(n)), "qsa_offload_staging_size")
    return n.value


def alloc_offload_staging(cfg, batch: int, device=None) -> torch.Tensor:
    """Device staging buffer for qsa_decode_offload (no initialisation needed)."""
    return torch.empty(qsa_offload_staging_size(cfg, batch), dtype=torch.uint8, device=device or "cuda")


def _p_host_or_device(t: torch.Tensor) -> int:
    """Address of a contiguous tensor in host or device memory. Whether the device can
    reach it (page-locked host memory or device memory) is the library's check."""
    if not t.is_contiguous():
        raise ValueError("QSA tensors must be contiguous")
    return t.data_ptr()


def qsa_decode_offload(cfg, t: Dict[str, torch.Tensor], staging, workspace, stream=None):
    """The decode step of qsa_forward with t["k_cache"] and t["v_cache"] in page-locked
    host memory (e.g. tensor.pin_memory()); everything else on the device. Only the
    attended blocks are copied to the device, into `staging`."""
    q = t["q"]
    batch, n_q = q.shape[0], q.shape[1]
    kv_cap = t["k_cache"].shape[2]
    dt = _elem(cfg)
    for name in ("q", "qi", "k_cache", "v_cache", "ki_cache", "out"):
        if t[name].dtype != dt:
            raise ValueError(f"{name}: dtype {t[name].dtype}, expected {dt}")
    T = qsa_tensors_t(batch, n_q, kv_cap, _p(q), _p(t["qi"]), _p_host_or_device(t["k_cache"]),
                      _p_host_or_device(t["v_cache"]), _p(t["ki_cache"]), _p(t["kbar_cache"]),
                      _p(t["kbar_blocks"]), _p(t["k_new"]), _p(t["v_new"]), _p(t["ki_new"]),
                      _p(t["kv_start"]), _p(t["kv_len"]), None, _p(t["sel"]), _p(t["out"]))
    _check(_lib.qsa_decode_offload(ctypes.byref(cfg), ctypes.byref(T), _p(staging), staging.numel(),
                                   _p(workspace), workspace.numel(), _stream(stream)), "qsa_decode_offload")


def qsa_selftest_wait_timeout(workspace, limit_ns: int = 50_000_000, stream=None):
    """Enqueue a wait that nothing completes; it gives up after limit_ns and records
    QSA_ERR_TIMEOUT in the workspace status word (read it with qsa_read_device_status)."""
    _check(_lib.qsa_selftest_wait_timeout(_p(workspace), int(limit_ns), _stream(stream)),
           "qsa_selftest_wait_timeout")


def qsa_read_device_status(workspace: torch.Tensor, stream=None) -> int:
    out = ctypes.c_int32(0)
    _check(_lib.qsa_read_device_status(_p(workspace), _stream(stream), ctypes.byref(out)),
           "qsa_read_device_status")
    return out.value
