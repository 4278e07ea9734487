"""Token-level key mask inside the kept tiles, through the C ABI.

sa_block_sparse_attention_masked attends to a key only when its block is
kept for the row and the key's mask byte is set; a row left with no key gets
O = 0.  Checked against the fp64 oracle with the same mask (max-abs 1e-2,
mean-abs 1e-3, exact zeros for rows with no key), and a mask of ones must
give exactly the unmasked result.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_util import Buffers, check_attention, dev_bf16, host_f64, sample_rows
from workloads import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import prompt_aware_head_b200 as sa
    return sa


def _select(sa, w, Q, K, rho, H_kv=None):
    L = sa.Layout(list(w.segments), w.N)
    buf = Buffers(sa, w.B, w.H, w.N, w.d, L.cap)
    sa.sa_select_blocks_gqa(L, dev_bf16(Q), dev_bf16(K), w.B, w.H, H_kv or w.H, w.d, rho, None, 0, buf.idx,
                            buf.counts, None, buf.ws, buf.ws_bytes)
    assert sa.sa_check(buf.ws) == sa.SA_OK
    return L, buf


def _masked(sa, w, Q, K, V, buf, km, H_kv=None):
    O = torch.full((w.B, w.H, w.N, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    kmd = None if km is None else torch.from_numpy(np.ascontiguousarray(km, dtype=np.uint8)).cuda()
    sa.sa_block_sparse_attention_masked(dev_bf16(Q), dev_bf16(K), dev_bf16(V), w.B, w.H, H_kv or w.H, w.N, w.d,
                                        buf.idx, buf.counts, buf.cap, kmd, None, 0, 0.0, O, buf.ws, buf.ws_bytes)
    assert sa.sa_check(buf.ws) == sa.SA_OK
    return O


def _live(idx, cnt, km, H, N):
    """Rows with at least one key both kept and unmasked: [B*H*N] bool."""
    nB = cnt.shape[-1]
    BH = cnt.size // nB
    idx = idx.reshape(BH, nB, -1)
    cnt = cnt.reshape(BH, nB)
    blk_any = (km.reshape(km.shape[0], nB, 64) != 0).any(-1)  # [B, nB]
    live = np.zeros((BH, nB), bool)
    for bh in range(BH):
        b = bh // H
        for i in range(nB):
            live[bh, i] = bool(blk_any[b, idx[bh, i, :cnt[bh, i]]].any())
    return np.repeat(live, 64, axis=1).reshape(-1)


def _sdxl_mask(w):
    km = np.ones((w.B, w.N), np.uint8)
    km[0, 100:300] = 0      # partial blocks 1 and 4, full blocks 2 and 3
    km[0, 4000:] = 0        # the tail of the last block
    km[1, :37] = 0          # the head of block 0
    km[1, 2048 + 5::7] = 0  # a scatter over the second half
    return km


def test_key_mask_parity_sdxl_all_rows(sa):
    w = WORKLOADS["sdxl"]
    Q, K, V = make_qkv(w, seed=21)
    km = _sdxl_mask(w)
    L, buf = _select(sa, w, Q, K, 0.3)
    O = host_f64(_masked(sa, w, Q, K, V, buf, km)).reshape(-1, w.d)
    idx, cnt = buf.lists()
    ref = oracle.attention(Q, K, V, w.H, idx, cnt, key_mask=km).reshape(-1, w.d)
    check_attention(O, ref, _live(idx, cnt, km, w.H, w.N))


def test_key_mask_joint_padding(sa):
    # the joint layout with its padding masked: the pinned block 0 holds 20 live text keys and 44 padding keys
    w = WORKLOADS["joint"]
    Q, K, V = make_qkv(w, seed=22)
    km = np.ones((w.B, w.N), np.uint8)
    km[:, 20:512] = 0
    L, buf = _select(sa, w, Q, K, 0.3)
    O = host_f64(_masked(sa, w, Q, K, V, buf, km)).reshape(-1, w.d)
    idx, cnt = buf.lists()
    rows = sample_rows(w.B, w.H, w.N, 0.002, seed=3, must=range(0, 64))
    ref = oracle.attention(Q, K, V, w.H, idx, cnt, rows=rows, key_mask=km)
    check_attention(O[rows], ref, _live(idx, cnt, km, w.H, w.N)[rows])


def test_mask_of_ones_is_the_unmasked_result(sa):
    w = WORKLOADS["sdxl"]
    Q, K, V = make_qkv(w, seed=23)
    L, buf = _select(sa, w, Q, K, 0.5)
    O1 = _masked(sa, w, Q, K, V, buf, np.ones((w.B, w.N), np.uint8))
    O0 = _masked(sa, w, Q, K, V, buf, None)
    assert torch.equal(O1.view(torch.int16), O0.view(torch.int16))


def test_fully_masked_batch_gives_zeros(sa):
    w = WORKLOADS["sdxl"]
    Q, K, V = make_qkv(w, seed=24)
    km = np.ones((w.B, w.N), np.uint8)
    km[1] = 0
    L, buf = _select(sa, w, Q, K, 0.3)
    O = host_f64(_masked(sa, w, Q, K, V, buf, km))
    assert np.all(O[1] == 0.0)
    idx, cnt = buf.lists()
    rows = sample_rows(1, w.H, w.N, 0.05, seed=4)  # batch 0 is as without the mask
    ref = oracle.attention(Q, K, V, w.H, idx, cnt, rows=rows, key_mask=km)
    check_attention(O.reshape(-1, w.d)[rows], ref, np.ones(len(rows), bool))


def test_key_mask_with_grouped_heads(sa):
    w = WORKLOADS["sdxl"]
    g = 2
    Q, K, V = make_qkv(w, seed=25)
    K, V = np.ascontiguousarray(K[:, ::g]), np.ascontiguousarray(V[:, ::g])
    km = _sdxl_mask(w)
    L, buf = _select(sa, w, Q, K, 0.3, H_kv=w.H // g)
    O = host_f64(_masked(sa, w, Q, K, V, buf, km, H_kv=w.H // g)).reshape(-1, w.d)
    idx, cnt = buf.lists()
    rows = sample_rows(w.B, w.H, w.N, 0.05, seed=5)
    ref = oracle.attention(Q, K, V, w.H, idx, cnt, rows=rows, key_mask=km)
    check_attention(O[rows], ref, _live(idx, cnt, km, w.H, w.N)[rows])


def test_row_whose_only_tile_is_masked_gives_zeros(sa):
    # hand-built lists: row 0 keeps only block 1, whose 64 keys are all masked (exact zeros); row 2 keeps
    # blocks 1 and 3 (block 1 is skipped, block 3 is partly masked); row 5 keeps only block 4 (untouched)
    w = WORKLOADS["tiny"]
    Q, K, V = make_qkv(w, seed=26)
    B, H, N, d, nB = w.B, w.H, w.N, w.d, w.nB
    buf = Buffers(sa, B, H, N, d, nB)
    idx = np.tile(np.arange(nB, dtype=np.int32), (B, H, nB, 1))
    cnt = np.full((B, H, nB), nB, np.int32)
    idx[:, :, 0, 0] = 1
    cnt[:, :, 0] = 1
    idx[:, :, 2, :2] = (1, 3)
    cnt[:, :, 2] = 2
    idx[:, :, 5, 0] = 4
    cnt[:, :, 5] = 1
    buf.idx.copy_(torch.from_numpy(idx))
    buf.counts.copy_(torch.from_numpy(cnt))
    km = np.ones((B, N), np.uint8)
    km[:, 64:128] = 0          # block 1: every key masked
    km[:, 192:200] = 0         # block 3: a few keys masked
    O = host_f64(_masked(sa, w, Q, K, V, buf, km))
    assert np.all(O[:, :, 0:64] == 0.0), "a row whose only kept tile is fully masked must be exactly zero"
    ref = oracle.attention(Q, K, V, H, idx, cnt, key_mask=km)
    check_attention(O.reshape(-1, d), ref.reshape(-1, d), _live(idx, cnt, km, H, N))
