"""A bounded wait that runs out is reported, and the device stays usable.

Every wait in the kernels is bounded: after its limit (2 s) the waiting
thread records SA_ERR_TIMEOUT in the workspace error word and the kernel
returns; nothing traps or hangs.  sa_debug_wait_timeout runs one kernel that
waits, through the same helper, on a barrier nothing completes.  The test
checks that sa_check reports the timeout, that the wait took about its limit,
and that the next calls on the same device still compute correct results.
Runs last among the GPU tests (it spends about two seconds waiting).
"""
import time

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_util import check_attention, dev_bf16, host_f64
from workloads import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import prompt_aware_head_b200 as sa
    return sa


def test_wait_timeout_is_reported_and_the_device_stays_usable(sa):
    w = WORKLOADS["tiny"]
    ws_bytes = sa.sa_workspace_size(w.B, w.H, w.N, w.d)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    sa.sa_workspace_init(ws, ws_bytes)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    sa.sa_debug_wait_timeout(ws, ws_bytes)
    assert sa.sa_check(ws) == sa.SA_ERR_TIMEOUT
    waited = time.perf_counter() - t0
    assert 1.5 < waited < 60.0, waited
    assert sa.sa_check(ws) == sa.SA_OK  # sa_check cleared the word
    # the same device and workspace still work: dense attention against the oracle
    Q, K, V = make_qkv(w, seed=31)
    O = torch.full((w.B, w.H, w.N, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    sa.sa_dense_attention(dev_bf16(Q), dev_bf16(K), dev_bf16(V), w.B, w.H, w.N, w.d, 0.0, O, ws, ws_bytes)
    assert sa.sa_check(ws) == sa.SA_OK
    idx, counts = oracle.select(np.zeros((w.B * w.H, w.nB, w.nB)), oracle.layout([], w.N), w.H, 1.0)
    ref = oracle.attention(Q, K, V, w.H, idx, counts).reshape(-1, w.d)
    check_attention(host_f64(O).reshape(-1, w.d), ref, np.ones(ref.shape[0], bool))
