"""sa_select_blocks_noalloc: the selection for callers that cannot allocate
device memory (hosts that own all device memory and give plugins no
allocator, or latency-critical code that must not call cudaMalloc).  Its
scratch is a fixed array inside the library; this test checks, through the C
ABI, that two calls in a row give exactly what sa_select_blocks gives for the
same inputs (lists bit-exact, scores identical), also with the scores kept in
the array, that its device-side errors are reported by sa_check_noalloc and
then cleared, and that a call beyond its size cap is refused before anything
runs."""
import numpy as np
import pytest
import torch

from tests.gpu_util import Buffers, compare_lists, dev_bf16
from workloads import WORKLOADS, head_mask_for_layer, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import prompt_aware_head_b200 as sa
    return sa


def _both(sa, w, seed, rho):
    Q, K, _ = make_qkv(w, seed=seed)
    q, k = dev_bf16(Q), dev_bf16(K)
    mask = head_mask_for_layer(w)
    L = sa.Layout(list(w.segments), w.N)
    ref = Buffers(sa, w.B, w.H, w.N, w.d, L.cap)
    ref_scores = torch.zeros((w.B, w.H, w.nB, w.nB), dtype=torch.float32, device="cuda")
    sa.sa_select_blocks(L, q, k, w.B, w.H, w.d, rho, mask, w.min_active, ref.idx, ref.counts, ref_scores,
                        ref.ws, ref.ws_bytes)
    idx = torch.full_like(ref.idx, -7)
    counts = torch.full_like(ref.counts, -7)
    scores = torch.zeros_like(ref_scores)
    sa.sa_select_blocks_noalloc(L, q, k, w.B, w.H, w.d, rho, mask, w.min_active, idx, counts, scores)
    assert sa.sa_check_noalloc() == sa.SA_OK
    return ref, ref_scores, idx, counts, scores, mask


def test_noalloc_matches_workspace_selection_twice(sa):
    for name, seed, rho in (("joint", 0, 0.3), ("sdxl", 1, 0.3)):   # two calls in a row, different sizes
        w = WORKLOADS[name]
        ref, ref_scores, idx, counts, scores, mask = _both(sa, w, seed, rho)
        compare_lists(*ref.lists(), idx.cpu().numpy(), counts.cpu().numpy())
        for h in np.flatnonzero(mask):
            assert torch.equal(scores[:, h], ref_scores[:, h])


def test_noalloc_lists_only_heads_in_groups(sa):
    # no scores_out: the scores stay in the fixed array too, so the joint workload's 24 heads go through it in
    # two groups (15 heads, then 9) -- the plain multi-head pooling path with scores in scratch
    w = WORKLOADS["joint"]
    Q, K, _ = make_qkv(w, seed=4)
    q, k = dev_bf16(Q), dev_bf16(K)
    L = sa.Layout(list(w.segments), w.N)
    ref = Buffers(sa, w.B, w.H, w.N, w.d, L.cap)
    sa.sa_select_blocks(L, q, k, w.B, w.H, w.d, 0.3, None, 0, ref.idx, ref.counts, None, ref.ws, ref.ws_bytes)
    for _ in range(2):
        idx = torch.full_like(ref.idx, -7)
        counts = torch.full_like(ref.counts, -7)
        sa.sa_select_blocks_noalloc(L, q, k, w.B, w.H, w.d, 0.3, None, 0, idx, counts, None)
        assert sa.sa_check_noalloc() == sa.SA_OK
        compare_lists(*ref.lists(), idx.cpu().numpy(), counts.cpu().numpy())


def test_noalloc_device_errors_are_reported_then_cleared(sa):
    # the path records device faults in an error word inside its fixed array; sa_check_noalloc reads and
    # clears it (the word is set here by a one-thread kernel, as a faulting kernel would set it)
    assert sa.sa_check_noalloc() == sa.SA_OK
    sa.sa_debug_noalloc_error(sa.SA_ERR_TIMEOUT)
    assert sa.sa_check_noalloc() == sa.SA_ERR_TIMEOUT
    assert sa.sa_check_noalloc() == sa.SA_OK
    sa.sa_debug_noalloc_error(sa.SA_ERR_BAD_INDEX)
    assert sa.sa_check_noalloc() == sa.SA_ERR_BAD_INDEX
    assert sa.sa_check_noalloc() == sa.SA_OK
    with pytest.raises(sa.SAError) as e:
        sa.sa_debug_noalloc_error(sa.SA_ERR_SHAPE)
    assert e.value.status == sa.SA_ERR_INVALID_ARG


def test_noalloc_refuses_sizes_beyond_its_scratch(sa):
    w = WORKLOADS["video"]
    L = sa.Layout(list(w.segments), w.N)
    q = torch.zeros(1024, dtype=torch.bfloat16, device="cuda")   # never read: the size check comes first
    idx = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(sa.SAError) as e:
        sa.sa_select_blocks_noalloc(L, q, q, 8, w.H, w.d, 0.2, None, 0, idx, idx, None)
    assert e.value.status == sa.SA_ERR_WORKSPACE
