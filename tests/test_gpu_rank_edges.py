"""Selection when a row's scores are degenerate, through the C ABI.

The rank kernel keeps the top k - 1 candidates of a row with a histogram of
the linear map (s - min) * 256 / (max - min) and ranks only the bucket that
holds the k-th score.  Two inputs take its other paths:
- every score equal: there is no range, and the radix select ranks the row;
- two distinct values: the boundary bucket holds more than 32 equal scores,
  and the radix select ranks that bucket.
In both, equal scores go to the lower block index, and the lists must equal
the oracle's for the scores the GPU dumped."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_util import Buffers, compare_lists, dev_bf16
from workloads import bf16_bits_from_f32, make_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import prompt_aware_head_b200 as sa
    return sa


def _select_and_compare(sa, w, Q, K, rho):
    L = sa.Layout(list(w.segments), w.N)
    buf = Buffers(sa, w.B, w.H, w.N, w.d, L.cap)
    scores = torch.zeros((w.B, w.H, w.nB, w.nB), dtype=torch.float32, device="cuda")
    sa.sa_select_blocks(L, dev_bf16(Q), dev_bf16(K), w.B, w.H, w.d, rho, None, 0, buf.idx, buf.counts, scores,
                        buf.ws, buf.ws_bytes)
    assert sa.sa_check(buf.ws) == sa.SA_OK
    sc = scores.cpu().numpy()
    cls = oracle.layout(list(w.segments), w.N)
    ref_idx, ref_cnt = oracle.select(sc.reshape(-1, w.nB, w.nB).astype(np.float64), cls, w.H, rho,
                                     np.ones(w.H, np.uint8), cap=L.cap)
    idx, cnt = buf.lists()
    compare_lists(idx, cnt, ref_idx, ref_cnt)
    return sc, idx, cnt


def test_all_scores_equal(sa):
    w = make_workload("sdxl", B=1, H=2)  # N 4096, 64 blocks, no segments
    shape = (w.B, w.H, w.N, w.d)
    Q = bf16_bits_from_f32(np.full(shape, 0.5, np.float32))
    K = bf16_bits_from_f32(np.full(shape, 0.25, np.float32))
    sc, idx, cnt = _select_and_compare(sa, w, Q, K, 0.3)
    assert np.all(sc == sc.flat[0])
    # the diagonal, then the lowest other indices
    k = sa.sa_budget(0.3, w.nB)
    for i in (0, 5, w.nB - 1):
        row = sorted([i] + [j for j in range(w.nB) if j != i][:k - 1])
        assert list(idx[0, 0, i, :cnt[0, 0, i]]) == row


def test_two_score_values_fill_the_boundary_bucket(sa):
    w = make_workload("joint", B=1, H=2)  # 264 blocks: 1 pinned, 7 dropped, 256 candidates
    rng = np.random.default_rng(5)
    Qf = (1.0 + 0.1 * rng.standard_normal((w.B, w.H, w.N, w.d))).astype(np.float32)  # q-bar . 1 > 0
    c = np.where(np.arange(w.nB) % 3 == 0, 2.0, 1.0).astype(np.float32)  # key block j holds c_j everywhere
    Kf = np.broadcast_to(np.repeat(c, 64)[:, None], (w.B, w.H, w.N, w.d)).astype(np.float32)
    sc, idx, cnt = _select_and_compare(sa, w, bf16_bits_from_f32(Qf), bf16_bits_from_f32(Kf), 0.3)
    # every sparse row holds exactly two score values, the larger on ~86 blocks
    cls = oracle.layout(list(w.segments), w.N)
    sparse = np.flatnonzero(cls == 1)
    row = sc[0, 0, sparse[10], sparse]
    assert len(np.unique(row)) == 2
