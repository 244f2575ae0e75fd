"""The QSA_DEBUG build (libqsa_debug.so): before every attention launch a device-side
check reads the selection list and records QSA_ERR_DEVICE_CHECK for any row whose
ids are not the row's min(n_c, k) complete blocks in strictly ascending order
followed by -1 padding (padding rows: -1 only). The attention kernels skip ids
outside [0, n_c) by themselves, so every list used here stays in bounds.

Runs in a child process, since the binding picks the library (QSA_LIBRARY) at import."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import torch
from block_sparse_long_15_b200 import qsa, workloads as W
from block_sparse_long_15_b200.runner import QSAPrefill
assert qsa.LIB_PATH.endswith("libqsa_debug.so"), qsa.LIB_PATH
w = W.small_variant(W.WORKLOADS["bf16_prefill_varlen_b8_s16384_leftpad"], seq=700, batch=2, pad_max=100,
                    block=64, topk=3, Hq=16, Hkv=2)
inp = W.make_inputs(w)
p = QSAPrefill(w, inp)
p()
torch.cuda.synchronize()
assert p.status() == qsa.QSA_OK, "a valid selection was flagged"
t = p.t
good = t["sel"].clone()
pad = int(inp["kv_start"][1])
assert pad > 0
r = 600  # a real row of sequence 0 with n_c = 9 > k = 3
def check(mut, want):
    s = good.clone()
    mut(s)
    qsa.qsa_sparse_attn(p.cfg, t["q"], t["k_cache"], t["v_cache"], s, t["kv_start"], t["kv_len"], t["q_first"],
                        t["out"], p.ws)
    torch.cuda.synchronize()
    got = qsa.qsa_read_device_status(p.ws)
    assert got == want, (want, got)
def out_of_range(s): s[0, r, 2] = (r + 1) // 64 + 3
def descending(s): s[0, r, 0], s[0, r, 1] = good[0, r, 1], good[0, r, 0]
def duplicate(s): s[0, r, 1] = good[0, r, 0]
def minus_one_first(s): s[0, r, 0] = -1
def padding_row_with_an_id(s): s[1, pad - 1, 0] = 0
check(lambda s: None, qsa.QSA_OK)
for m in (out_of_range, descending, duplicate, minus_one_first, padding_row_with_an_id):
    check(m, qsa.QSA_ERR_DEVICE_CHECK)
check(lambda s: None, qsa.QSA_OK)
print("DEBUG_CHECKS_OK")
'''


@pytest.mark.gpu
def test_debug_build_flags_bad_selection_lists(cuda_lib):
    env = dict(os.environ, QSA_LIBRARY="libqsa_debug.so", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "DEBUG_CHECKS_OK" in r.stdout, r.stdout + r.stderr


def test_debug_library_exports_the_same_entry_points():
    import ctypes

    from block_sparse_long_15_b200 import build, qsa
    build.build()
    dbg = ctypes.CDLL(build.LIB_DEBUG)
    for name in qsa.EXPORTED:
        assert hasattr(dbg, name), name
