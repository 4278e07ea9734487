"""The largest sequence the library takes: 1024 blocks (N = 65536), GPU.

Sorts last among the GPU tests.

This size runs the 32-chunk rank kernel, 8 row tiles of the score kernel
and union lists of up to 1024 entries (25 MB of union-list workspace for
its two heads; 301 MB at 24 heads).  The selection must match the oracle
as everywhere else; attention is checked on sampled rows and on every row
of the pinned text block.  One block more is refused before any launch.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_util import Buffers, check_attention, compare_lists, dev_bf16, host_f64, sample_rows
from workloads import SEG_IMAGE, SEG_PAD, SEG_TEXT, make_qkv, make_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import prompt_aware_head_b200 as sa
    return sa


def test_largest_block_count(sa):
    N = 65536
    w = make_workload("joint", N=N, H=2, segments=((SEG_TEXT, 0, 20), (SEG_PAD, 20, 492), (SEG_IMAGE, 512, N - 512)),
                      grid=(254, 256))
    assert w.nB == 1024
    Q, K, V = make_qkv(w, seed=41)
    L = sa.Layout(list(w.segments), N)
    buf = Buffers(sa, w.B, w.H, N, w.d, L.cap)
    scores = torch.zeros((w.B, w.H, w.nB, w.nB), dtype=torch.float32, device="cuda")
    sa.sa_select_blocks(L, dev_bf16(Q), dev_bf16(K), w.B, w.H, w.d, 0.3, None, 0, buf.idx, buf.counts, scores,
                        buf.ws, buf.ws_bytes)
    assert sa.sa_check(buf.ws) == sa.SA_OK
    sc = scores.cpu().numpy()
    ref = oracle.scores(oracle.pool(Q), oracle.pool(K))
    qn = np.linalg.norm(oracle.pool(Q), axis=-1)
    kn = np.linalg.norm(oracle.pool(K), axis=-1)
    assert np.all(np.abs(sc - ref) <= 1e-5 * qn[..., :, None] * kn[..., None, :] + 1e-7)
    cls = oracle.layout(list(w.segments), N)
    ref_idx, ref_cnt = oracle.select(sc.reshape(-1, w.nB, w.nB).astype(np.float64), cls, w.H, 0.3,
                                     np.ones(w.H, np.uint8), cap=L.cap)
    idx, cnt = buf.lists()
    compare_lists(idx, cnt, ref_idx, ref_cnt)
    O = torch.full((w.B, w.H, N, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    sa.sa_block_sparse_attention(dev_bf16(Q), dev_bf16(K), dev_bf16(V), w.B, w.H, N, w.d, buf.idx, buf.counts,
                                 L.cap, None, 0, 0.0, O, buf.ws, buf.ws_bytes)
    assert sa.sa_check(buf.ws) == sa.SA_OK
    rows = sample_rows(w.B, w.H, N, 0.001, seed=6, must=list(range(64)) + [N + r for r in range(64)])
    live = np.repeat(cnt.reshape(-1, w.nB) > 0, 64, axis=1).reshape(-1)
    check_attention(host_f64(O).reshape(-1, w.d)[rows], oracle.attention(Q, K, V, w.H, idx, cnt, rows=rows),
                    live[rows])


def test_one_block_more_is_refused(sa):
    with pytest.raises(sa.SAError) as e:
        sa.sa_workspace_size(1, 2, 65536 + 64, 128)
    assert e.value.status == sa.SA_ERR_SHAPE
