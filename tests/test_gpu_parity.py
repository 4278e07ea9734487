"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Block lists are compared bit-exactly given identical fp32 block scores (the
oracle ranks the scores the GPU dumped); scores themselves are compared with
the oracle's fp64 scores; attention output within max-abs 1e-2 / mean-abs
1e-3 of the fp64 oracle, exact zeros for rows without tiles and skipped heads.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_util import Buffers, check_attention, compare_lists, dev_bf16, host_f64, sample_rows
from workloads import (SEG_IMAGE, SEG_OTHER, SEG_PAD, SEG_TEXT, WORKLOADS, bf16_bits_from_f32, bf16_bits_to_f32,
                       head_mask_for_layer, make_qkv, make_workload)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import prompt_aware_head_b200 as sa
    return sa


def _select(sa, w, Q, K, rho, mask, min_active, want_scores=True, layout=None):
    L = layout or sa.Layout(list(w.segments), w.N)
    buf = Buffers(sa, w.B, w.H, w.N, w.d, L.cap)
    scores = torch.zeros((w.B, w.H, w.nB, w.nB), dtype=torch.float32, device="cuda") if want_scores else None
    sa.sa_select_blocks(L, dev_bf16(Q), dev_bf16(K), w.B, w.H, w.d, rho, mask, min_active, buf.idx, buf.counts,
                        scores, buf.ws, buf.ws_bytes)
    assert sa.sa_check(buf.ws) == sa.SA_OK
    return L, buf, (scores.cpu().numpy() if want_scores else None)


def _check_scores(w, Q, K, gpu_scores, mask):
    ref = oracle.scores(oracle.pool(Q), oracle.pool(K))          # fp64 [B, H, nB, nB]
    qn = np.linalg.norm(oracle.pool(Q), axis=-1)
    kn = np.linalg.norm(oracle.pool(K), axis=-1)
    tol = 1e-5 * qn[..., :, None] * kn[..., None, :] + 1e-7
    for h in range(w.H):
        if mask is None or mask[h]:
            assert np.all(np.abs(gpu_scores[:, h] - ref[:, h]) <= tol[:, h]), "scores off for head %d" % h


# ------------------------------------------------------------------ layout

def test_layout_classes_match_oracle(sa):
    rng = np.random.default_rng(11)
    cases = [(list(w.segments), w.N) for w in WORKLOADS.values()]
    cases.append(([(SEG_TEXT, 0, 100), (SEG_PAD, 100, 412), (SEG_IMAGE, 512, 16384)], 16896))
    for _ in range(30):
        N = 64 * int(rng.integers(1, 40))
        cuts = np.sort(rng.choice(np.arange(1, N), size=int(rng.integers(0, 6)), replace=False))
        b = [0] + list(cuts) + [N]
        cases.append(([(int(rng.integers(0, 4)), b[i], b[i + 1] - b[i]) for i in range(len(b) - 1)], N))
    for segs, N in cases:
        L = sa.Layout(segs, N)
        ref = oracle.layout(segs, N)
        assert np.array_equal(L.classes(), ref)
        assert L.cap == oracle.cap_of(ref)
        L.release()
    with pytest.raises(sa.SAError) as e:
        sa.Layout([(SEG_TEXT, 0, 64), (SEG_IMAGE, 100, 28)], 128)
    assert e.value.status == sa.SA_ERR_LAYOUT


# ------------------------------------------------------------------ selection

SELECT_CASES = [("tiny", 0.5), ("sdxl", 0.3), ("sdxl", 0.5), ("sdxl", 1.0), ("joint", 0.3), ("video", 0.2)]


@pytest.mark.parametrize("name,rho", SELECT_CASES)
def test_select_parity(sa, name, rho):
    w = WORKLOADS[name]
    Q, K, _ = make_qkv(w)
    mask = head_mask_for_layer(w)
    L, buf, sc = _select(sa, w, Q, K, rho, mask, w.min_active)
    _check_scores(w, Q, K, sc, mask)
    cls = oracle.layout(list(w.segments), w.N)
    ref_idx, ref_cnt = oracle.select(sc.reshape(-1, w.nB, w.nB).astype(np.float64), cls, w.H, rho, mask, cap=L.cap)
    idx, cnt = buf.lists()
    compare_lists(idx, cnt, ref_idx, ref_cnt)
    # informational: rows whose fp64 ranking differs from the fp32 one
    if rho < 1.0:
        f64_idx, f64_cnt = oracle.select(oracle.scores(oracle.pool(Q), oracle.pool(K)).reshape(-1, w.nB, w.nB),
                                         cls, w.H, rho, mask, cap=L.cap)
        diff = sum(not np.array_equal(f64_idx[r, i, :f64_cnt[r, i]], ref_idx[r, i, :ref_cnt[r, i]])
                   for r in range(f64_cnt.shape[0]) for i in range(w.nB))
        print("%s rho=%.1f: %d rows rank differently under fp64 scores" % (name, rho, diff))


@pytest.mark.parametrize("nB", [131, 132, 262])
def test_select_parity_ragged_block_count(sa, nB):
    # a multiple of 4 blocks: scores leave in 128 x 32 tensor-store boxes clipped at nB; otherwise as row stores
    N = 64 * nB
    w = make_workload("tiny", N=N, d=128, H=2, head_mask=None, min_active=0,
                      segments=((SEG_TEXT, 0, 64), (SEG_PAD, 64, 64), (SEG_IMAGE, 128, N - 128)))
    Q, K, _ = make_qkv(w, seed=nB)
    L, buf, sc = _select(sa, w, Q, K, 0.3, None, 0)
    _check_scores(w, Q, K, sc, None)
    cls = oracle.layout(list(w.segments), w.N)
    ref_idx, ref_cnt = oracle.select(sc.reshape(-1, w.nB, w.nB).astype(np.float64), cls, w.H, 0.3,
                                     np.ones(w.H, np.uint8), cap=L.cap)
    idx, cnt = buf.lists()
    compare_lists(idx, cnt, ref_idx, ref_cnt)


@pytest.mark.parametrize("layer", [0, 1, 63])
@pytest.mark.parametrize("rho", [1.0, 0.5])
def test_select_parity_stack(sa, layer, rho):
    w = WORKLOADS["stack"]
    Q, K, _ = make_qkv(w, layer=layer)
    mask = head_mask_for_layer(w, layer)
    L, buf, sc = _select(sa, w, Q, K, rho, mask, w.min_active)
    cls = oracle.layout([], w.N)
    ref_idx, ref_cnt = oracle.select(sc.reshape(-1, w.nB, w.nB).astype(np.float64), cls, w.H, rho, mask, cap=L.cap)
    compare_lists(*buf.lists(), ref_idx, ref_cnt)
    assert np.all(buf.counts.cpu().numpy()[0][mask == 0] == 0)


def test_select_dense_short_circuit_and_scale_invariance(sa):
    w = WORKLOADS["sdxl"]
    Q, K, _ = make_qkv(w)
    L = sa.Layout([], w.N)
    buf = Buffers(sa, w.B, w.H, w.N, w.d, L.cap)
    sa.sa_select_blocks(L, dev_bf16(Q), dev_bf16(K), w.B, w.H, w.d, 1.0, None, 0, buf.idx, buf.counts, None,
                        buf.ws, buf.ws_bytes)
    idx, cnt = buf.lists()
    assert np.all(cnt == w.nB) and np.all(idx[..., :w.nB] == np.arange(w.nB))
    # doubling Q scales every score by exactly 2: identical lists
    _, b1, _ = _select(sa, w, Q, K, 0.3, None, 0, want_scores=False, layout=L)
    Q2 = bf16_bits_from_f32(2 * bf16_bits_to_f32(Q))
    _, b2, _ = _select(sa, w, Q2, K, 0.3, None, 0, want_scores=False, layout=L)
    compare_lists(*b1.lists(), *b2.lists())


def test_select_head_mask_errors(sa):
    w = WORKLOADS["stack"]
    L = sa.Layout([], w.N)
    buf = Buffers(sa, 1, 32, w.N, 128, L.cap)
    q = torch.zeros((1, 32, w.N, 128), dtype=torch.bfloat16, device="cuda")
    three = np.zeros(32, np.uint8)
    three[:3] = 1
    with pytest.raises(sa.SAError) as e:
        sa.sa_select_blocks(L, q, q, 1, 32, 128, 0.5, three, sa.MIN_ACTIVE_HEADS, buf.idx, buf.counts, None,
                            buf.ws, buf.ws_bytes)
    assert e.value.status == sa.SA_ERR_HEAD_MASK


# ------------------------------------------------------------------ patterns

PATTERN_CASES = [("tiny", sa_kind, W, G, r) for sa_kind, W, G, r in [(0, 0, 0, 1), (1, 64, 1, 1), (2, 96, 0, 3)]] + [
    ("joint", 0, 0, 0, 1), ("joint", 1, 512, 8, 1), ("video", 0, 0, 0, 1), ("video", 1, 512, 8, 1),
    ("video", 2, 1024, 2, 80), ("sdxl", 2, 200, 0, 3)]


@pytest.mark.parametrize("name,kind,W,G,r", PATTERN_CASES)
def test_pattern_parity(sa, name, kind, W, G, r):
    w = WORKLOADS[name]
    rho = w.densities[0]
    mask = head_mask_for_layer(w)
    L = sa.Layout(list(w.segments), w.N)
    buf = Buffers(sa, w.B, w.H, w.N, w.d, L.cap)
    sa.sa_pattern_mask(L, kind, w.B, w.H, rho, mask, w.min_active, buf.idx, buf.counts, window_tokens=W,
                       n_global_blocks=G, dilation=r)
    cls = oracle.layout(list(w.segments), w.N)
    ref_idx, ref_cnt = oracle.pattern(cls, kind, w.B * w.H, w.H, window=W, n_global=G, dilation=r, density=rho,
                                      head_mask=mask, cap=L.cap)
    compare_lists(*buf.lists(), ref_idx, ref_cnt)


# ------------------------------------------------------------------ attention

def _attention(sa, w, Q, K, V, buf, mask, min_active):
    O = torch.full((w.B, w.H, w.N, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    sa.sa_block_sparse_attention(dev_bf16(Q), dev_bf16(K), dev_bf16(V), w.B, w.H, w.N, w.d, buf.idx, buf.counts,
                                 buf.cap, mask, min_active, 0.0, O, buf.ws, buf.ws_bytes)
    assert sa.sa_check(buf.ws) == sa.SA_OK
    return O


def _live_rows(cnt, mask, H, N):
    live = np.repeat(cnt.reshape(-1, cnt.shape[-1]) > 0, 64, axis=1)  # [BH, N]
    if mask is not None:
        live &= np.tile(np.asarray(mask, bool), live.shape[0] // H)[:, None]
    return live.reshape(-1)


ATTN_FULL = [("tiny", 0.5), ("sdxl", 0.3), ("sdxl", 1.0)]


@pytest.mark.parametrize("name,rho", ATTN_FULL)
def test_attention_parity_full(sa, name, rho):
    w = WORKLOADS[name]
    Q, K, V = make_qkv(w)
    mask = head_mask_for_layer(w)
    L, buf, _ = _select(sa, w, Q, K, rho, mask, w.min_active, want_scores=False)
    O = _attention(sa, w, Q, K, V, buf, mask, w.min_active)
    idx, cnt = buf.lists()
    ref = oracle.attention(Q, K, V, w.H, idx, cnt, mask).reshape(-1, w.d)
    mx, mean = check_attention(host_f64(O).reshape(-1, w.d), ref, _live_rows(cnt, mask, w.H, w.N))
    print("%s rho=%.1f attention max-abs %.3g mean-abs %.3g" % (name, rho, mx, mean))


def test_attention_parity_joint_every_row(sa):
    # the headline workload, every row of every head against the fp64 oracle (about 20 s of oracle time on 16
    # host cores: 47 us per row)
    w = WORKLOADS["joint"]
    Q, K, V = make_qkv(w)
    mask = head_mask_for_layer(w)
    L, buf, _ = _select(sa, w, Q, K, 0.3, mask, w.min_active, want_scores=False)
    O = _attention(sa, w, Q, K, V, buf, mask, w.min_active)
    idx, cnt = buf.lists()
    ref = oracle.attention(Q, K, V, w.H, idx, cnt, mask).reshape(-1, w.d)
    mx, mean = check_attention(host_f64(O).reshape(-1, w.d), ref, _live_rows(cnt, mask, w.H, w.N))
    print("joint rho=0.3 every row: max-abs %.3g mean-abs %.3g" % (mx, mean))


def test_attention_parity_d64_work_queue(sa):
    # d = 64 with enough items for the work queue (4 x 10 heads x 32 pairs = 1280 items, at least 8 per CTA
    # on 148 SMs; SDXL itself has 640 and takes the static deal): 5 % of the rows, seeded, plus the first and
    # last row of every head
    w = make_workload("sdxl", B=4)
    Q, K, V = make_qkv(w, seed=21)
    L, buf, _ = _select(sa, w, Q, K, 0.3, None, 0, want_scores=False)
    O = _attention(sa, w, Q, K, V, buf, None, 0)
    idx, cnt = buf.lists()
    edges = [bh * w.N + n for bh in range(w.B * w.H) for n in (0, w.N - 1)]
    rows = sample_rows(w.B, w.H, w.N, 0.05, seed=4, must=edges)
    ref = oracle.attention(Q, K, V, w.H, idx, cnt, rows=rows)
    mx, mean = check_attention(host_f64(O).reshape(-1, w.d)[rows], ref, _live_rows(cnt, None, w.H, w.N)[rows])
    print("sdxl x4 batches (work queue): max-abs %.3g mean-abs %.3g" % (mx, mean))


def _pin_rows(w):
    """Flat row ids of every query row in a pinned block, over every head."""
    cls = oracle.layout(list(w.segments), w.N)
    pins = np.flatnonzero(cls == oracle.PIN)
    toks = (pins[:, None] * 64 + np.arange(64)[None, :]).reshape(-1)
    return ((np.arange(w.B * w.H)[:, None] * w.N) + toks[None, :]).reshape(-1)


def test_attention_parity_video_sampled_and_pinned_rows(sa):
    # 5 % of the rows, seeded, plus every row of the pinned text block of every head (dense over 513 blocks)
    w = WORKLOADS["video"]
    Q, K, V = make_qkv(w)
    mask = head_mask_for_layer(w)
    L, buf, _ = _select(sa, w, Q, K, 0.2, mask, w.min_active, want_scores=False)
    O = _attention(sa, w, Q, K, V, buf, mask, w.min_active)
    idx, cnt = buf.lists()
    rows = sample_rows(w.B, w.H, w.N, 0.05, seed=3, must=_pin_rows(w).tolist() + [w.N - 1])
    ref = oracle.attention(Q, K, V, w.H, idx, cnt, mask, rows=rows)
    live = _live_rows(cnt, mask, w.H, w.N)[rows]
    mx, mean = check_attention(host_f64(O).reshape(-1, w.d)[rows], ref, live)
    print("video rho=0.2 %d rows (5 %% + pinned): max-abs %.3g mean-abs %.3g" % (len(rows), mx, mean))


@pytest.mark.parametrize("layer,rho", [(0, 0.5), (5, 1.0), (31, 0.5), (63, 0.5)])
def test_attention_stack_layer_head_mask(sa, layer, rho):
    # four of the 64 layers, every row: skipped heads exactly zero, active heads against the oracle
    w = WORKLOADS["stack"]
    Q, K, V = make_qkv(w, layer=layer)
    mask = head_mask_for_layer(w, layer)
    L, buf, _ = _select(sa, w, Q, K, rho, mask, w.min_active, want_scores=False)
    O = _attention(sa, w, Q, K, V, buf, mask, w.min_active)
    idx, cnt = buf.lists()
    o = host_f64(O)
    assert np.all(o[0][mask == 0] == 0.0)
    ref = oracle.attention(Q, K, V, w.H, idx, cnt, mask).reshape(-1, w.d)
    check_attention(o.reshape(-1, w.d), ref, _live_rows(cnt, mask, w.H, w.N))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [64, 320, 1152])
def test_attention_ragged_and_edge_layouts(sa, d, N):
    # odd block counts (a pair with no partner), dropped rows, pinned rows, empty heads
    w = make_workload("tiny", N=N, d=d, H=3, head_mask=(1, 0, 1), min_active=2,
                      segments=((SEG_OTHER, 0, 30), (SEG_PAD, 30, 98), (SEG_IMAGE, 128, N - 128)) if N > 128 else ())
    Q, K, V = make_qkv(w, seed=N + d)
    mask = head_mask_for_layer(w)
    for rho in (0.4, 1.0):
        L, buf, _ = _select(sa, w, Q, K, rho, mask, w.min_active, want_scores=False)
        O = _attention(sa, w, Q, K, V, buf, mask, w.min_active)
        idx, cnt = buf.lists()
        ref = oracle.attention(Q, K, V, w.H, idx, cnt, mask).reshape(-1, w.d)
        check_attention(host_f64(O).reshape(-1, w.d), ref, _live_rows(cnt, mask, w.H, w.N))


@pytest.mark.parametrize("name", ["sdxl", "joint"])
def test_dense_attention_parity(sa, name):
    w = WORKLOADS[name]
    Q, K, V = make_qkv(w)
    ws_bytes = sa.sa_workspace_size(w.B, w.H, w.N, w.d)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    O = torch.full((w.B, w.H, w.N, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    sa.sa_dense_attention(dev_bf16(Q), dev_bf16(K), dev_bf16(V), w.B, w.H, w.N, w.d, 0.0, O, ws, ws_bytes)
    assert sa.sa_check(ws) == sa.SA_OK
    nB = w.nB
    idx = np.broadcast_to(np.arange(nB, dtype=np.int32), (w.B * w.H, nB, nB)).copy()
    cnt = np.full((w.B * w.H, nB), nB, np.int32)
    rows = sample_rows(w.B, w.H, w.N, 0.002, seed=9, must=[0, w.N - 1])
    ref = oracle.attention(Q, K, V, w.H, idx, cnt, rows=rows)
    check_attention(host_f64(O).reshape(-1, w.d)[rows], ref, np.ones(len(rows), bool))


def test_selection_changes_the_output(sa):
    # fails if a block-only mask is silently attended densely
    w = WORKLOADS["sdxl"]
    Q, K, V = make_qkv(w)
    L, buf, _ = _select(sa, w, Q, K, 0.3, None, 0, want_scores=False)
    O_sparse = host_f64(_attention(sa, w, Q, K, V, buf, None, 0))
    L1, buf1, _ = _select(sa, w, Q, K, 1.0, None, 0, want_scores=False)
    O_dense = host_f64(_attention(sa, w, Q, K, V, buf1, None, 0))
    rows = sample_rows(w.B, w.H, w.N, 0.002, seed=2)
    idx1, cnt1 = buf1.lists()
    floor = np.abs(O_dense.reshape(-1, w.d)[rows] - oracle.attention(Q, K, V, w.H, idx1, cnt1, rows=rows)).mean()
    change = np.abs(O_sparse - O_dense).mean()
    assert change > 100 * floor, "selection changes the output by %.3g, floor %.3g" % (change, floor)


def test_determinism(sa):
    w = WORKLOADS["joint"]
    Q, K, V = make_qkv(w)
    outs = []
    for _ in range(2):
        L, buf, _ = _select(sa, w, Q, K, 0.3, None, 0, want_scores=False)
        O = _attention(sa, w, Q, K, V, buf, None, 0)
        outs.append((buf.lists(), O.view(torch.int16).cpu().numpy()))
    compare_lists(*outs[0][0], *outs[1][0])
    assert np.array_equal(outs[0][1], outs[1][1])


def test_bad_index_is_reported(sa):
    w = make_workload("tiny", N=512, H=2, head_mask=None, min_active=0)
    Q, K, V = make_qkv(w)
    buf = Buffers(sa, 1, 2, 512, 64, 8)
    idx = np.tile(np.arange(8, dtype=np.int32), (1, 2, 8, 1))
    idx[0, 1, 3, 2] = 99           # out of range: skipped and reported
    buf.idx.copy_(torch.from_numpy(idx))
    buf.counts.fill_(8)
    O = torch.zeros((1, 2, 512, 64), dtype=torch.bfloat16, device="cuda")
    sa.sa_block_sparse_attention(dev_bf16(Q), dev_bf16(K), dev_bf16(V), 1, 2, 512, 64, buf.idx, buf.counts, 8, None,
                                 0, 0.0, O, buf.ws, buf.ws_bytes)
    assert sa.sa_check(buf.ws) == sa.SA_ERR_BAD_INDEX
    assert sa.sa_check(buf.ws) == sa.SA_OK   # the error word was cleared
    assert torch.isfinite(O.float()).all()


def test_density_readback(sa):
    w = WORKLOADS["joint"]
    Q, K, _ = make_qkv(w)
    mask = np.ones(w.H, np.uint8)
    mask[5:9] = 0
    L, buf, _ = _select(sa, w, Q, K, 0.3, mask, 4, want_scores=False)
    da, dall, st = sa.sa_density(buf.counts, w.B, w.H, w.nB, mask, buf.ws, buf.ws_bytes)
    idx, cnt = buf.lists()
    ra, rall = oracle.density(cnt, w.H, w.nB, mask)
    assert da == pytest.approx(ra) and dall == pytest.approx(rall)
    assert st.tiles == 19969 * (w.H - 4) and st.heads_active == w.H - 4
    assert da == pytest.approx(19969 / 264 ** 2)


def test_polynomial_exp2_against_cuda(sa):
    # the softmax's software exponential vs CUDA's exp2 (fp32), relative error bound 1e-4
    y = torch.cat([torch.linspace(-125.0, 8.0, 1 << 20, device="cuda"),
                   torch.rand(1 << 20, device="cuda") * 16 - 12]).contiguous()
    out = torch.empty_like(y)
    sa.sa_debug_exp2(y, out, y.numel())
    torch.cuda.synchronize()
    ref = torch.exp2(y.double())
    rel = ((out.double() - ref) / ref).abs().max().item()
    assert rel < 1e-4, rel
    low = torch.tensor([-200.0, -126.0, -1e30], device="cuda")
    o2 = torch.empty_like(low)
    sa.sa_debug_exp2(low, o2, 3)
    torch.cuda.synchronize()
    assert torch.all(torch.isfinite(o2)) and torch.all(o2 <= 2.0 ** -124)
