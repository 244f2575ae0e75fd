"""Failure detection on the GPU without a GPU fault: a device wait that nothing
completes runs out after a short limit, the kernel records QSA_ERR_TIMEOUT and
returns, the host reads the status, and the context keeps working."""
import time

import pytest
import torch

from block_sparse_long_15_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_context_survives(cuda_lib):
    qsa = cuda_lib
    w = W.small_variant(W.WORKLOADS["bf16_prefill_s8192"], seq=256)
    from block_sparse_long_15_b200.runner import QSAPrefill
    p = QSAPrefill(w, W.make_inputs(w))
    assert p.status() == qsa.QSA_OK
    t0 = time.perf_counter()
    qsa.qsa_selftest_wait_timeout(p.ws, 50_000_000)
    assert qsa.qsa_read_device_status(p.ws) == qsa.QSA_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    # reading cleared the word; the context still runs the real path
    out, sel = p()
    torch.cuda.synchronize()
    assert p.status() == qsa.QSA_OK
    assert torch.isfinite(out.float()).all()


def test_selftest_rejects_bad_limits(cuda_lib):
    qsa = cuda_lib
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(qsa.QSAError):
        qsa.qsa_selftest_wait_timeout(ws, 10)
