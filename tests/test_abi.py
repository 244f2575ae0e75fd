"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before touching the GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest

from block_sparse_long_15_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def qsa():
    build.build()
    from block_sparse_long_15_b200 import qsa as q
    return q


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "qsa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(qsa_[a-z_]+)\s*\(", txt)))


def test_exports_every_declared_symbol(qsa):
    syms = declared_symbols()
    assert len(syms) >= 10, syms
    lib = ctypes.CDLL(qsa.LIB_PATH)
    for s in syms:
        assert hasattr(lib, s), f"libqsa.so does not export {s}"
    assert set(qsa.EXPORTED) == set(syms)


def test_abi_version_and_status_strings(qsa):
    assert qsa.qsa_abi_version() == 2
    for s in range(6):
        assert qsa.status_string(s)
    assert qsa.status_string(99) == "unknown status"


def _cfg(qsa, **kw):
    base = dict(Hq=16, Hkv=2, d=128, Hi=4, di=64, block=64, topk=32)
    base.update(kw)
    return qsa.make_config(**base)


def test_config_validation(qsa):
    assert qsa.qsa_config_validate(_cfg(qsa)) == qsa.QSA_OK
    assert qsa.qsa_topk_blocks(_cfg(qsa)) == 32
    assert qsa.qsa_topk_blocks(_cfg(qsa, budget=100, block=64)) == 1
    # one indexer key head only (Qwen4ExpTextConfig.indexer_kv_heads)
    assert qsa.qsa_config_validate(_cfg(qsa, indexer_kv_heads=2)) == qsa.QSA_ERR_UNSUPPORTED
    # incomplete indexer field set
    assert qsa.qsa_config_validate(_cfg(qsa, Hi=0)) == qsa.QSA_ERR_INVALID_ARG
    assert qsa.qsa_config_validate(_cfg(qsa, indexer_kv_heads=0)) == qsa.QSA_ERR_INVALID_ARG
    # budget smaller than one block
    assert qsa.qsa_config_validate(_cfg(qsa, budget=63)) == qsa.QSA_ERR_INVALID_ARG
    # GQA needs Hq % Hkv == 0; dims multiple of 8
    assert qsa.qsa_config_validate(_cfg(qsa, Hq=15)) == qsa.QSA_ERR_INVALID_ARG
    assert qsa.qsa_config_validate(_cfg(qsa, d=100)) == qsa.QSA_ERR_INVALID_ARG
    assert qsa.qsa_config_validate(_cfg(qsa, di=12)) == qsa.QSA_ERR_INVALID_ARG
    assert qsa.qsa_config_validate(_cfg(qsa, d=512)) == qsa.QSA_ERR_UNSUPPORTED
    c = _cfg(qsa)
    c.dtype = 7
    assert qsa.qsa_config_validate(c) == qsa.QSA_ERR_INVALID_ARG
    assert qsa.library().qsa_config_validate(None) == qsa.QSA_ERR_INVALID_ARG


def test_workspace_size(qsa):
    c = _cfg(qsa)
    n = qsa.qsa_workspace_size(c, qsa.QSA_PREFILL, 1, 8192, 8192)
    assert n >= 256 and n % 256 == 0
    n = qsa.qsa_workspace_size(c, qsa.QSA_DECODE, 64, 1, 32768)
    assert n >= 256
    with pytest.raises(qsa.QSAError):
        qsa.qsa_workspace_size(c, 7, 1, 1, 1)
    with pytest.raises(qsa.QSAError):
        qsa.qsa_workspace_size(c, qsa.QSA_PREFILL, -1, 1, 1)


def test_null_and_misaligned_pointers_rejected_on_host(qsa):
    L = qsa.library()
    c = _cfg(qsa)
    cp = ctypes.byref(c)
    P = ctypes.c_void_p
    # null pointers
    assert L.qsa_sparse_attn(cp, None, None, None, None, None, None, None, 1, 16, 16, None, None, 1 << 20,
                             None) == qsa.QSA_ERR_INVALID_ARG
    assert L.qsa_index_score_topk(cp, None, None, None, None, 1, 16, 16, None, None, 1 << 20,
                                  None) == qsa.QSA_ERR_INVALID_ARG
    assert L.qsa_compress_blocks(cp, None, None, None, None, 1, 64, None, None, None) == qsa.QSA_ERR_INVALID_ARG
    assert L.qsa_forward(cp, qsa.QSA_PREFILL, None, None, 0, None) == qsa.QSA_ERR_INVALID_ARG
    # misaligned (never dereferenced: rejected before any launch)
    bad = P(0x1001)
    good = P(0x10000)
    assert L.qsa_sparse_attn(cp, bad, good, good, good, good, good, good, 1, 16, 16, good, good, 1 << 20,
                             None) == qsa.QSA_ERR_INVALID_ARG
    # empty batches are a no-op that succeeds without touching memory
    assert L.qsa_sparse_attn(cp, None, None, None, None, None, None, None, 0, 16, 16, None, None, 0,
                             None) == qsa.QSA_OK
    # decode requires n_q == 1 and the new-token tensors
    t = qsa.qsa_tensors_t(1, 2, 64, *([0x10000] * 15))
    assert L.qsa_forward(cp, qsa.QSA_DECODE, ctypes.byref(t), good, 1 << 20, None) == qsa.QSA_ERR_INVALID_ARG
    # a workspace too small for the status word
    t = qsa.qsa_tensors_t(1, 1, 64, *([0x10000] * 15))
    assert L.qsa_forward(cp, qsa.QSA_DECODE, ctypes.byref(t), good, 16, None) == qsa.QSA_ERR_INVALID_ARG


def test_sizes_beyond_limits(qsa):
    c = _cfg(qsa, block=1, budget=4)
    with pytest.raises(qsa.QSAError) as e:
        qsa.qsa_workspace_size(c, qsa.QSA_PREFILL, 1, 1 << 20, 1 << 20)
    assert e.value.status == qsa.QSA_ERR_UNSUPPORTED


def test_kernel_names(qsa):
    assert qsa.qsa_attn_kernel_name(_cfg(qsa, dtype="fp32", Hq=4, Hkv=1, d=64)) == "simt"


def test_kernel_names_by_shape(qsa):
    # head_dim 128: the two-tile tcgen05 prefill kernel and the streaming decode kernel
    assert qsa.qsa_attn_kernel_name(_cfg(qsa)) == "tcgen05"
    assert qsa.qsa_attn_kernel_name(_cfg(qsa), qsa.QSA_DECODE) == "split-kv decode"
    # head_dim 256 (the config default): the one-tile kernel for prefill and decode
    assert qsa.qsa_attn_kernel_name(_cfg(qsa, d=256)) == "tcgen05 one-tile"
    assert qsa.qsa_attn_kernel_name(_cfg(qsa, d=256), qsa.QSA_DECODE) == "tcgen05 one-tile"


def test_prefill_tensor_core_routing(qsa):
    # a group size that divides the 128-row tile (up to 32, the config limit) and a block
    # size that is a multiple of the 64-key half take the persistent tcgen05 kernel
    for hq, hkv in [(2, 2), (4, 2), (8, 2), (16, 2), (32, 4), (32, 1), (64, 2)]:
        for block in (64, 128, 192, 256):
            c = _cfg(qsa, Hq=hq, Hkv=hkv, block=block, topk=4)
            assert qsa.qsa_attn_kernel_name(c) == "tcgen05", (hq, hkv, block)
    # a group of 12 (does not divide 128), a block of 32 keys, head_dim 64, fp32: CUDA cores
    assert qsa.qsa_attn_kernel_name(_cfg(qsa, Hq=24, Hkv=2)) == "simt"
    assert qsa.qsa_attn_kernel_name(_cfg(qsa, block=32)) == "simt"
    assert qsa.qsa_attn_kernel_name(_cfg(qsa, d=64)) == "simt"
    assert qsa.qsa_attn_kernel_name(_cfg(qsa, dtype="fp32")) == "simt"


def test_offload_staging_size(qsa):
    # K and V of (k + 1) * B tokens per (sequence, KV head), then the remapped
    # selection and lengths, each section rounded up to 256 bytes
    def r256(x):
        return (x + 255) // 256 * 256
    for kw, batch in ((dict(), 64), (dict(d=256), 3), (dict(Hq=32, Hkv=4, Hi=8, block=128, topk=16), 7)):
        c = _cfg(qsa, **kw)
        cfg = dict(Hq=16, Hkv=2, d=128, Hi=4, di=64, block=64, topk=32)
        cfg.update(kw)
        kv = r256(batch * cfg["Hkv"] * (cfg["topk"] + 1) * cfg["block"] * cfg["d"] * 2)
        want = 2 * kv + r256(batch * cfg["topk"] * 4) + r256(batch * 4)
        assert qsa.qsa_offload_staging_size(c, batch) == want
    assert qsa.qsa_offload_staging_size(_cfg(qsa), 0) == 3 * 0
    with pytest.raises(qsa.QSAError):
        qsa.qsa_offload_staging_size(_cfg(qsa, indexer_kv_heads=2), 4)


def test_offload_rejects_null_arguments_on_host(qsa):
    lib = qsa.library()
    c = _cfg(qsa)
    assert lib.qsa_decode_offload(ctypes.byref(c), None, None, 0, None, 0, None) == qsa.QSA_ERR_INVALID_ARG
    t = qsa.qsa_tensors_t()
    t.batch, t.n_q, t.kv_cap = 2, 1, 4096  # pointers all NULL
    assert lib.qsa_decode_offload(ctypes.byref(c), ctypes.byref(t), None, 0, None, 0, None) == \
        qsa.QSA_ERR_INVALID_ARG


def test_project_rejects_bad_arguments_on_host(qsa):
    L = qsa.library()
    c = _cfg(qsa)
    cp = ctypes.byref(c)
    P = ctypes.c_void_p
    good = P(0x10000)
    pc = qsa.qsa_proj_config_t(2048, 1e6, 128, 64)
    args = lambda pcx, kv_cap=16, row0=0, x=good: (cp, ctypes.byref(pcx), x, good, good, 1, 16, good, good, good,
                                                   good, good, kv_cap, row0, good, 256, None)
    assert L.qsa_project(*args(pc, x=P(0x10001))) == qsa.QSA_ERR_INVALID_ARG        # misaligned
    assert L.qsa_project(*args(pc, kv_cap=8)) == qsa.QSA_ERR_INVALID_ARG             # rows past kv_cap
    bad_theta = qsa.qsa_proj_config_t(2048, 0.0, 128, 64)
    assert L.qsa_project(*args(bad_theta)) == qsa.QSA_ERR_INVALID_ARG
    for bad in (qsa.qsa_proj_config_t(2048, 1e6, 48, 64),    # rotary dim not a multiple of 32
                qsa.qsa_proj_config_t(2000, 1e6, 128, 64),   # hidden size not a multiple of 64
                qsa.qsa_proj_config_t(2048, 1e6, 256, 64)):  # more rotary dims than head dims
        if c.head_dim == 128:
            assert L.qsa_project(*args(bad)) == qsa.QSA_ERR_UNSUPPORTED
