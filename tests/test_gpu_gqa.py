"""Grouped key/value heads through the C ABI (the _gqa entry points).

K and V hold H_kv heads; query head h reads key/value head h // (H / H_kv).
Scores are held to the fp64 oracle's grouped scores, block lists bit-exactly
to the oracle's ranking of the GPU's own scores, attention within max-abs
1e-2 / mean-abs 1e-3 of the fp64 oracle.  Sharing a key/value head must give
exactly what the plain calls give on K and V repeated per group.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_util import Buffers, check_attention, compare_lists, dev_bf16, host_f64, sample_rows
from workloads import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import prompt_aware_head_b200 as sa
    return sa


@functools.lru_cache(maxsize=4)
def _grouped(name, g, seed=0):
    """Q with the workload's H heads; K, V with the first head of each group of g."""
    Q, K, V = make_qkv(WORKLOADS[name], seed=seed)
    return Q, np.ascontiguousarray(K[:, ::g]), np.ascontiguousarray(V[:, ::g])


def _select_gqa(sa, w, Q, K, H_kv, rho, mask, min_active):
    L = sa.Layout(list(w.segments), w.N)
    buf = Buffers(sa, w.B, w.H, w.N, w.d, L.cap)
    scores = torch.zeros((w.B, w.H, w.nB, w.nB), dtype=torch.float32, device="cuda")
    sa.sa_select_blocks_gqa(L, dev_bf16(Q), dev_bf16(K), w.B, w.H, H_kv, w.d, rho, mask, min_active, buf.idx,
                            buf.counts, scores, buf.ws, buf.ws_bytes)
    assert sa.sa_check(buf.ws) == sa.SA_OK
    return L, buf, scores.cpu().numpy()


def _attention_gqa(sa, w, Q, K, V, H_kv, buf, mask, min_active):
    O = torch.full((w.B, w.H, w.N, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    sa.sa_block_sparse_attention_gqa(dev_bf16(Q), dev_bf16(K), dev_bf16(V), w.B, w.H, H_kv, w.N, w.d, buf.idx,
                                     buf.counts, buf.cap, mask, min_active, 0.0, O, buf.ws, buf.ws_bytes)
    assert sa.sa_check(buf.ws) == sa.SA_OK
    return O


def _live(cnt, mask, H, N):
    live = np.repeat(cnt.reshape(-1, cnt.shape[-1]) > 0, 64, axis=1)
    if mask is not None:
        live &= np.tile(np.asarray(mask, bool), live.shape[0] // H)[:, None]
    return live.reshape(-1)


CASES = [
    # (workload, group size, head mask, min_active, density, fraction of rows checked against the oracle)
    ("tiny", 2, (0, 1, 1, 0), 2, 0.5, 1.0),   # each group's first head skipped: the second pools the key head
    ("tiny", 4, (0, 0, 1, 1), 2, 0.5, 1.0),   # one key head for all four query heads
    ("sdxl", 5, None, 0, 0.3, 0.05),
    ("joint", 4, None, 0, 0.3, 0.002),
]


@pytest.mark.parametrize("name,g,hm,min_active,rho,frac", CASES)
def test_gqa_select_and_attention_parity(sa, name, g, hm, min_active, rho, frac):
    w = WORKLOADS[name]  # its own head mask is not used: the case passes one (or none)
    mask = None if hm is None else np.array(hm, np.uint8)
    H_kv = w.H // g
    Q, K, V = _grouped(name, g, seed=g)
    L, buf, sc = _select_gqa(sa, w, Q, K, H_kv, rho, mask, min_active)
    ref = oracle.scores(oracle.pool(Q), oracle.pool(K))
    qn = np.linalg.norm(oracle.pool(Q), axis=-1)
    kn = np.repeat(np.linalg.norm(oracle.pool(K), axis=-1), g, axis=1)
    tol = 1e-5 * qn[..., :, None] * kn[..., None, :] + 1e-7
    for h in range(w.H):
        if mask is None or mask[h]:
            assert np.all(np.abs(sc[:, h] - ref[:, h]) <= tol[:, h]), "scores off for head %d" % h
    cls = oracle.layout(list(w.segments), w.N)
    om = np.ones(w.H, np.uint8) if mask is None else mask
    ref_idx, ref_cnt = oracle.select(sc.reshape(-1, w.nB, w.nB).astype(np.float64), cls, w.H, rho, om, cap=L.cap)
    idx, cnt = buf.lists()
    compare_lists(idx, cnt, ref_idx, ref_cnt)
    O = host_f64(_attention_gqa(sa, w, Q, K, V, H_kv, buf, mask, min_active)).reshape(-1, w.d)
    live = _live(cnt, om, w.H, w.N)
    if frac >= 1.0:
        out_ref = oracle.attention(Q, K, V, w.H, idx, cnt, om).reshape(-1, w.d)
        check_attention(O, out_ref, live)
    else:
        rows = sample_rows(w.B, w.H, w.N, frac, seed=7)
        check_attention(O[rows], oracle.attention(Q, K, V, w.H, idx, cnt, om, rows=rows), live[rows])


def test_gqa_equals_plain_calls_on_repeated_kv(sa):
    w = WORKLOADS["sdxl"]
    g, rho = 2, 0.3
    Q, K, V = _grouped("sdxl", g, seed=3)
    Kr, Vr = (np.ascontiguousarray(np.repeat(x, g, axis=1)) for x in (K, V))
    L, buf, _ = _select_gqa(sa, w, Q, K, w.H // g, rho, None, 0)
    O = _attention_gqa(sa, w, Q, K, V, w.H // g, buf, None, 0)
    buf2 = Buffers(sa, w.B, w.H, w.N, w.d, L.cap)
    sa.sa_select_blocks(L, dev_bf16(Q), dev_bf16(Kr), w.B, w.H, w.d, rho, None, 0, buf2.idx, buf2.counts, None,
                        buf2.ws, buf2.ws_bytes)
    O2 = torch.empty_like(O)
    sa.sa_block_sparse_attention(dev_bf16(Q), dev_bf16(Kr), dev_bf16(Vr), w.B, w.H, w.N, w.d, buf2.idx, buf2.counts,
                                 L.cap, None, 0, 0.0, O2, buf2.ws, buf2.ws_bytes)
    assert sa.sa_check(buf2.ws) == sa.SA_OK
    idx, cnt = buf.lists()
    idx2, cnt2 = buf2.lists()
    compare_lists(idx, cnt, idx2, cnt2)
    assert torch.equal(O.view(torch.int16), O2.view(torch.int16))
    # the dense kernel likewise
    Od, Od2 = torch.empty_like(O), torch.empty_like(O)
    sa.sa_dense_attention_gqa(dev_bf16(Q), dev_bf16(K), dev_bf16(V), w.B, w.H, w.H // g, w.N, w.d, 0.0, Od, buf.ws,
                              buf.ws_bytes)
    sa.sa_dense_attention(dev_bf16(Q), dev_bf16(Kr), dev_bf16(Vr), w.B, w.H, w.N, w.d, 0.0, Od2, buf.ws,
                          buf.ws_bytes)
    assert sa.sa_check(buf.ws) == sa.SA_OK
    assert torch.equal(Od.view(torch.int16), Od2.view(torch.int16))


def test_gqa_noalloc_matches_workspace_path(sa):
    # joint, 24 query heads over 6 key heads: the fixed scratch takes 15 heads at a time (no scores
    # requested), so the second group of heads starts inside a group sharing a key head
    w = WORKLOADS["joint"]
    g = 4
    Q, K, _ = _grouped("joint", g, seed=g)
    L, buf, _ = _select_gqa(sa, w, Q, K, w.H // g, 0.3, None, 0)
    idx2 = torch.full_like(buf.idx, -7)
    cnt2 = torch.full_like(buf.counts, -7)
    sa.sa_select_blocks_noalloc_gqa(L, dev_bf16(Q), dev_bf16(K), w.B, w.H, w.H // g, w.d, 0.3, None, 0, idx2, cnt2,
                                    None)
    torch.cuda.synchronize()
    idx, cnt = buf.lists()
    compare_lists(idx, cnt, idx2.cpu().numpy(), cnt2.cpu().numpy())


def test_gqa_shape_errors(sa):
    w = WORKLOADS["sdxl"]  # 10 query heads
    Q, K, _ = _grouped("sdxl", 5, seed=5)
    L = sa.Layout([], w.N)
    buf = Buffers(sa, w.B, w.H, w.N, w.d, L.cap)
    for H_kv in (0, 3, 20):
        with pytest.raises(sa.SAError) as e:
            sa.sa_select_blocks_gqa(L, dev_bf16(Q), dev_bf16(K), w.B, w.H, H_kv, w.d, 0.3, None, 0, buf.idx,
                                    buf.counts, None, buf.ws, buf.ws_bytes)
        assert e.value.status == sa.SA_ERR_SHAPE
