"""The random-block control pattern on the GPU (SplitMix64 draws on both sides).

sa_pattern_mask with SA_PAT_RANDOM keeps, per sparse row, its diagonal and
k - 1 other sparse blocks ranked by 21 bits of a SplitMix64 output per
(row, column), plus the pins; the lists must equal the oracle's exactly.
This file sorts after the other parity files.
"""
import pytest
import torch

import oracle
from tests.gpu_util import Buffers, compare_lists
from workloads import WORKLOADS, head_mask_for_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import prompt_aware_head_b200 as sa
    return sa


@pytest.mark.parametrize("name,seed", [("tiny", 0), ("sdxl", 1), ("joint", 2), ("video", 3), ("video", 2 ** 63 + 5)])
def test_random_pattern_parity(sa, name, seed):
    # SplitMix64 draws on both sides: the lists must be identical
    w = WORKLOADS[name]
    rho = w.densities[0]
    mask = head_mask_for_layer(w)
    L = sa.Layout(list(w.segments), w.N)
    buf = Buffers(sa, w.B, w.H, w.N, w.d, L.cap)
    sa.sa_pattern_mask(L, sa.SA_PAT_RANDOM, w.B, w.H, rho, mask, w.min_active, buf.idx, buf.counts, seed=seed)
    cls = oracle.layout(list(w.segments), w.N)
    ref_idx, ref_cnt = oracle.pattern(cls, oracle.PAT_RANDOM, w.B * w.H, w.H, density=rho, head_mask=mask,
                                      cap=L.cap, seed=seed)
    compare_lists(*buf.lists(), ref_idx, ref_cnt)
