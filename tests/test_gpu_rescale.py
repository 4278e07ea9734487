"""The online softmax's rescale path, forced.

The kernel keeps a row's running max until a later key block's max exceeds
it by more than 2^8 (in base-2 exponent), then rescales that row's partial
O in TMEM (after the previous PV completes) and continues with the new max.
The synthetic workloads rarely trigger it, so these inputs do: every query
row is a_r * u and key block j is c_j * u plus noise, with u a unit vector
and c_j rising by 8 per block, so a row's logits grow by 8 a_r (11.5 to 35
in base 2) from one key block to the next.  A row's walk (its union list in
ascending order from a rotated start) then raises its max at nearly every
step; rows differ in a_r, so the rows of a warp rescale by different factors
at the same step.  Outputs within max-abs 1e-2 / mean-abs 1e-3 of the fp64
oracle at the same softmax scale, on every row, for d = 64 and 128, with
content-selected lists and with full lists.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_util import Buffers, check_attention, dev_bf16, host_f64
from workloads import bf16_bits_from_f32

pytestmark = pytest.mark.gpu

B, H, N = 1, 4, 2048
NB = N // 64
SCALE = 1.0  # logits are q . k itself


@pytest.fixture(scope="module")
def sa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import prompt_aware_head_b200 as sa
    return sa


def _inputs(d, seed):
    rng = np.random.default_rng([seed, d])
    u = np.ones(d, np.float32) / np.sqrt(d)
    a = 1.0 + 2.0 * rng.random((B, H, N, 1), dtype=np.float32)          # a_r in [1, 3)
    Q = a * u + 0.05 * rng.standard_normal((B, H, N, d), dtype=np.float32)
    c = (8.0 * np.repeat(np.arange(NB, dtype=np.float32), 64))[None, None, :, None]
    K = c * u + 0.5 * rng.standard_normal((B, H, N, d), dtype=np.float32)
    V = rng.standard_normal((B, H, N, d), dtype=np.float32)
    return tuple(bf16_bits_from_f32(x) for x in (Q, K, V))


def _run(sa, d, Q, K, V, idx_t, cnt_t, buf):
    O = torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    sa.sa_block_sparse_attention(dev_bf16(Q), dev_bf16(K), dev_bf16(V), B, H, N, d, idx_t, cnt_t, buf.cap, None,
                                 0, SCALE, O, buf.ws, buf.ws_bytes)
    assert sa.sa_check(buf.ws) == sa.SA_OK
    return host_f64(O).reshape(-1, d)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("lists", ["content", "full"])
def test_growing_logits_force_rescales(sa, d, lists):
    Q, K, V = _inputs(d, seed=11)
    L = sa.Layout([], N)
    buf = Buffers(sa, B, H, N, d, L.cap)
    if lists == "content":
        sa.sa_select_blocks(L, dev_bf16(Q), dev_bf16(K), B, H, d, 0.3, None, 0, buf.idx, buf.counts, None, buf.ws,
                            buf.ws_bytes)
        assert sa.sa_check(buf.ws) == sa.SA_OK
    else:
        full = np.broadcast_to(np.arange(NB, dtype=np.int32), (B, H, NB, NB))
        buf.idx[..., :NB] = torch.from_numpy(full.copy()).cuda()
        buf.counts.fill_(NB)
    idx, cnt = buf.lists()
    # the walk really climbs: every row's list spans key blocks whose logits differ by far more than 2^8
    assert np.all(cnt >= 2)
    got = _run(sa, d, Q, K, V, buf.idx, buf.counts, buf)
    ref = oracle.attention(Q, K, V, H, idx, cnt, scale=SCALE).reshape(-1, d)
    mx, mean = check_attention(got, ref, np.ones(B * H * N, bool))
    print("d=%d %s lists: max-abs %.3g mean-abs %.3g" % (d, lists, mx, mean))
    L.release()
