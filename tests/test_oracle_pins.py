"""Pins of the CPU oracle to things other than itself (CPU only).

Each test checks the oracle against the pages' worked numbers, a library
routine (numpy, torch SDPA in fp64), a closed form, or brute force on tiny
inputs, chosen so that a dropped term, a wrong sign or index, or a transposed
operand fails at least one of them.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.conftest import read_golden
from workloads import (SEG_IMAGE, SEG_OTHER, SEG_PAD, SEG_TEXT, WORKLOADS, bf16_bits_from_f32,
                       bf16_bits_to_f32, head_mask_for_layer, make_qkv)


def _bits(x):
    return bf16_bits_from_f32(np.asarray(x, dtype=np.float32))


def _f64(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


# ---------------------------------------------------------------- layout

def test_layout_worked_example_2048():
    g = read_golden("layout_2048_short_prompt.txt")
    N, block, text = int(g["N"]), int(g["block"]), int(g["text_stream_tokens"])
    whole_text = oracle.layout([(SEG_TEXT, 0, text), (SEG_IMAGE, text, N - text)], N, block)
    assert whole_text.shape[0] == int(g["key_blocks_per_row"])
    for live in (65, 100, 128):  # a short prompt: its live tokens fill two blocks
        runs = oracle.layout([(SEG_TEXT, 0, live), (SEG_PAD, live, text - live),
                              (SEG_IMAGE, text, N - text)], N, block)
        moved = int(np.sum((whole_text == oracle.PIN) & (runs == oracle.DROP)))
        assert moved == int(g["moved_pinned_to_dropped"])
        assert np.all(runs[text // block:] == oracle.SPARSE)


def test_layout_configs_block_counts():
    # pinned / dropped / candidate blocks of the five workloads
    expect = {"tiny": (1, 1, 6), "sdxl": (0, 0, 64), "joint": (1, 7, 256), "stack": (0, 0, 64),
              "video": (1, 7, 512)}
    for name, (p, d, c) in expect.items():
        w = WORKLOADS[name]
        cls = oracle.layout(list(w.segments), w.N)
        assert (np.sum(cls == oracle.PIN), np.sum(cls == oracle.DROP), np.sum(cls == oracle.SPARSE)) == (p, d, c)


def test_layout_straddle_and_kinds_brute_force():
    rng = np.random.default_rng(7)
    for _ in range(200):
        N = 64 * int(rng.integers(1, 9))
        cuts = np.sort(rng.choice(np.arange(1, N), size=int(rng.integers(0, 5)), replace=False))
        bounds = [0] + list(cuts) + [N]
        segs = [(int(rng.integers(0, 4)), bounds[i], bounds[i + 1] - bounds[i]) for i in range(len(bounds) - 1)]
        cls = oracle.layout(segs, N)
        tok = np.concatenate([np.full(l, k) for k, s, l in segs])
        for b in range(N // 64):
            kinds = set(tok[64 * b:64 * b + 64].tolist())
            if kinds == {SEG_IMAGE}:
                assert cls[b] == oracle.SPARSE
            elif kinds == {SEG_PAD}:
                assert cls[b] == oracle.DROP
            else:
                assert cls[b] == oracle.PIN


def test_layout_rejects_bad_segments():
    with pytest.raises(ValueError):
        oracle.layout([(SEG_TEXT, 0, 64), (SEG_IMAGE, 65, 63)], 128)   # gap
    with pytest.raises(ValueError):
        oracle.layout([(SEG_TEXT, 0, 64)], 128)                         # short
    with pytest.raises(ValueError):
        oracle.layout([(7, 0, 128)], 128)                               # unknown kind
    assert np.all(oracle.layout([], 256) == oracle.SPARSE)              # no layout: all sparse
    assert np.all(oracle.layout([(SEG_OTHER, 0, 128)], 128) == oracle.PIN)


# ---------------------------------------------------------------- pool / scores

def test_pool_matches_numpy_block_mean():
    rng = np.random.default_rng(1)
    X = _bits(rng.standard_normal((3, 256, 64)))
    got = oracle.pool(X)
    ref = _f64(X).reshape(3, 4, 64, 64).mean(axis=2)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-15)
    const = oracle.pool(_bits(np.full((1, 128, 64), 0.375)))
    assert np.all(const == 0.375)


def test_scores_match_numpy_matmul_and_orientation():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((2, 5, 16))
    k = rng.standard_normal((2, 5, 16))
    s = oracle.scores(q, k)
    np.testing.assert_allclose(s, q @ np.swapaxes(k, -1, -2), rtol=1e-14, atol=1e-14)
    assert not np.allclose(s, np.swapaxes(s, -1, -2))   # q/k roles are not symmetric


# ---------------------------------------------------------------- budget / selection

def test_budget_properties():
    for C in (1, 6, 64, 256, 512):
        for rho in (0.01, 0.2, 0.3, 0.5, 0.7, 0.999, 1.0):
            k = oracle.budget(rho, C)
            assert 1 <= k <= C
            assert k <= np.float32(rho) * C + 1e-4 + 1e-9 or k == 1
            assert k == C or (k + 1) > np.float32(rho) * C + 1e-4
    assert oracle.budget(np.float32(0.7), 10) == 7     # 0.7f * 10 = 6.99999988
    assert oracle.budget(1.0, 256) == 256


def _check_selection(sc, cls, H, rho, hm, idx, counts):
    nB = cls.shape[0]
    P = int(np.sum(cls == oracle.PIN))
    C = int(np.sum(cls == oracle.SPARSE))
    k = oracle.budget(rho, C)
    for bh in range(sc.shape[0]):
        active = hm is None or hm[bh % H]
        for i in range(nB):
            lst = idx[bh, i, :counts[bh, i]]
            if not active or cls[i] == oracle.DROP:
                assert counts[bh, i] == 0
                continue
            assert np.all(np.diff(lst) > 0)
            assert not np.any(cls[lst] == oracle.DROP)
            if cls[i] == oracle.PIN:
                assert counts[bh, i] == P + C
                continue
            assert counts[bh, i] == P + k
            assert i in lst
            assert set(np.flatnonzero(cls == oracle.PIN)) <= set(lst.tolist())
            kept = [j for j in lst if cls[j] == oracle.SPARSE and j != i]
            unkept = [j for j in np.flatnonzero(cls == oracle.SPARSE) if j not in lst]
            for a in kept:           # every kept candidate beats every dropped one
                for b in unkept:
                    sa, sb = sc[bh, i, a] + 0.0, sc[bh, i, b] + 0.0
                    assert sa > sb or (sa == sb and a < b)


def test_select_invariants_random_scores():
    rng = np.random.default_rng(3)
    segs = [(SEG_TEXT, 0, 40), (SEG_PAD, 40, 88), (SEG_IMAGE, 128, 640)]
    cls = oracle.layout(segs, 768)
    H = 3
    sc = rng.standard_normal((2 * H, 12, 12))
    sc[0, 5, :] = 0.25           # ties resolve to the lower index
    sc[1, 6, ::2] = -0.0         # -0 ranks as +0
    sc[1, 6, 1::2] = 0.0
    hm = np.array([1, 0, 1], dtype=np.uint8)
    for rho in (0.1, 0.3, 0.5, 1.0):
        idx, counts = oracle.select(sc, cls, H, rho, hm)
        _check_selection(sc, cls, H, rho, hm, idx, counts)
    idx, counts = oracle.select(sc, cls, H, 0.5, hm)
    # all-equal scores keep the diagonal plus the lowest-index candidates
    assert idx[0, 5, :counts[0, 5]].tolist() == [0, 2, 3, 4, 5, 6]   # k = 5 of C = 10, pin 0


def test_select_scale_invariance_and_dense_budget():
    w = WORKLOADS["tiny"]
    Q, K, _ = make_qkv(w)
    cls = oracle.layout(list(w.segments), w.N)
    s1 = oracle.scores(oracle.pool(Q), oracle.pool(K)).reshape(-1, w.nB, w.nB)
    s2 = oracle.scores(oracle.pool(_bits(2 * bf16_bits_to_f32(Q))), oracle.pool(K)).reshape(-1, w.nB, w.nB)
    a = oracle.select(s1, cls, w.H, 0.5)
    b = oracle.select(s2, cls, w.H, 0.5)
    assert np.array_equal(a[1], b[1])
    for bh in range(w.H):
        for i in range(w.nB):
            assert np.array_equal(a[0][bh, i, :a[1][bh, i]], b[0][bh, i, :b[1][bh, i]])
    # a budget covering every candidate is the dense (non-drop) list
    idx, counts = oracle.select(s1, cls, w.H, 1.0)
    nd = np.flatnonzero(cls != oracle.DROP)
    for i in np.flatnonzero(cls != oracle.DROP):
        assert idx[0, i, :counts[0, i]].tolist() == nd.tolist()


def test_realized_density_closed_form():
    # tiles per head = P*(P+C) + C*(P+k); density = tiles / nB^2
    for name, rho, tiles in (("tiny", 0.5, 31), ("joint", 0.3, 19969), ("video", 0.2, 53249),
                             ("sdxl", 0.3, 1216)):
        w = WORKLOADS[name]
        cls = oracle.layout(list(w.segments), w.N)
        sc = np.random.default_rng(0).standard_normal((1, w.nB, w.nB))
        idx, counts = oracle.select(sc, cls, 1, rho)
        assert int(counts.sum()) == tiles
        da, dall = oracle.density(counts, 1, w.nB)
        assert da == pytest.approx(tiles / w.nB ** 2)


def test_density_over_active_and_over_all_with_skipped_heads():
    # joint layout, two batches of 24 heads with heads 5-8 skipped: every active head keeps 19969 tiles
    # (P(P+C) + C(P+k)) and a skipped head none, so over the active heads the density is 19969 / nB^2 and over
    # all heads 19969 * 20 / (24 nB^2) -- dividing either by the other head count fails one of the two
    w = WORKLOADS["joint"]
    H, B = 24, 2
    cls = oracle.layout(list(w.segments), w.N)
    hm = np.ones(H, np.uint8)
    hm[5:9] = 0
    sc = np.random.default_rng(5).standard_normal((B * H, w.nB, w.nB))
    idx, counts = oracle.select(sc, cls, H, 0.3, hm)
    assert int(counts.sum()) == 19969 * B * 20
    da, dall = oracle.density(counts, H, w.nB, hm)
    assert da == pytest.approx(19969 / w.nB ** 2, rel=1e-12)
    assert dall == pytest.approx(19969 * 20 / (24 * w.nB ** 2), rel=1e-12)
    # no mask: both are the same; every head skipped but one: over_all is 1/24 of over_active
    da1, dall1 = oracle.density(counts, H, w.nB, None)
    assert da1 == pytest.approx(dall1, rel=1e-12) and dall1 == pytest.approx(dall, rel=1e-12)
    one = np.zeros(H, np.uint8)
    one[3] = 1
    _, c1 = oracle.select(sc, cls, H, 0.3, one)
    a1, b1 = oracle.density(c1, H, w.nB, one)
    assert a1 == pytest.approx(19969 / w.nB ** 2, rel=1e-12) and b1 == pytest.approx(a1 / 24, rel=1e-12)


def test_min_active_heads_in_stack_masks():
    g = read_golden("crate_constants.txt")
    min_active = int(g["MIN_ACTIVE_HEADS"])
    w = WORKLOADS["stack"]
    for layer in range(w.layers):
        m = head_mask_for_layer(w, layer)
        assert int(m.sum()) >= min_active
        assert int(m.sum()) == int(w.H * (1 - float(g["DEFAULT_SPARSITY"])))
        runs = m.reshape(8, 4)
        assert np.all((runs.sum(1) == 0) | (runs.sum(1) == 4))   # contiguous runs of 4


# ---------------------------------------------------------------- patterns

def _token_keysets(N, kind, W, r):
    q = np.arange(N)[:, None]
    k = np.arange(N)[None, :]
    rel = np.abs(q - k) <= W
    if kind == oracle.PAT_DILATED:
        rel &= ((q - k) % r) == 0
    return rel


def _block_cover(rel, block=64):
    nB = rel.shape[0] // block
    return rel.reshape(nB, block, nB, block).any(axis=(1, 3))


@pytest.mark.parametrize("kind,W,r", [(oracle.PAT_WINDOW_GLOBAL, 64, 1), (oracle.PAT_WINDOW_GLOBAL, 96, 1),
                                      (oracle.PAT_WINDOW_GLOBAL, 512, 1), (oracle.PAT_DILATED, 96, 3),
                                      (oracle.PAT_DILATED, 200, 80), (oracle.PAT_DILATED, 64, 3)])
def test_patterns_match_brute_force_token_sets(kind, W, r):
    N = 512 + 256
    cover = _block_cover(_token_keysets(N, kind, W, r))
    for segs in ([], [(SEG_TEXT, 0, 40), (SEG_PAD, 40, 88), (SEG_IMAGE, 128, N - 128)]):
        cls = oracle.layout(segs, N)
        idx, counts = oracle.pattern(cls, kind, 1, 1, window=W, n_global=0, dilation=r)
        for i in range(N // 64):
            got = set(idx[0, i, :counts[0, i]].tolist())
            if cls[i] == oracle.DROP:
                assert not got
            elif cls[i] == oracle.PIN:
                assert got == set(np.flatnonzero(cls != oracle.DROP).tolist())
            else:
                want = {j for j in range(N // 64) if cls[j] == oracle.PIN or (cls[j] == oracle.SPARSE and cover[i, j])}
                assert got == want


def test_window_global_blocks():
    w = WORKLOADS["video"]
    cls = oracle.layout(list(w.segments), w.N)
    idx, counts = oracle.pattern(cls, oracle.PAT_WINDOW_GLOBAL, 1, 1, window=512, n_global=8)
    glob = np.flatnonzero(cls == oracle.SPARSE)[:8]
    nd = np.flatnonzero(cls != oracle.DROP)
    for i in range(w.nB):
        lst = idx[0, i, :counts[0, i]]
        if cls[i] == oracle.DROP:
            continue
        if i in glob:
            assert lst.tolist() == nd.tolist()
        assert set(glob.tolist()) <= set(lst.tolist())
    i = 300   # a row far from the globals: 17 window blocks + 8 globals + 1 pin
    assert counts[0, i] == 17 + 8 + 1


def test_radial_is_nearest_band_with_pins():
    w = WORKLOADS["joint"]
    cls = oracle.layout(list(w.segments), w.N)
    rho = 0.3
    k = oracle.budget(rho, int(np.sum(cls == oracle.SPARSE)))
    idx, counts = oracle.pattern(cls, oracle.PAT_RADIAL, 1, 1, density=rho)
    for i in np.flatnonzero(cls == oracle.SPARSE):
        lst = idx[0, i, :counts[0, i]]
        assert 0 in lst                                    # the pinned text column
        band = [j for j in lst if cls[j] == oracle.SPARSE]
        assert len(band) == k and i in band
        rest = [j for j in np.flatnonzero(cls == oracle.SPARSE) if j not in band]
        dmax = max(abs(i - j) for j in band)
        assert all(abs(i - j) > dmax or (abs(i - j) == dmax and j > max(b for b in band if abs(i - b) == dmax))
                   for j in rest)


# ---------------------------------------------------------------- attention

def _torch_masked_attention(Q, K, V, mask):
    q = torch.from_numpy(_f64(Q))
    k = torch.from_numpy(_f64(K))
    v = torch.from_numpy(_f64(V))
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=torch.from_numpy(mask)).numpy()


def _token_mask(idx, counts, N, block=64):
    BH, nB = counts.shape
    m = np.zeros((BH, N, N), dtype=bool)
    for bh in range(BH):
        for i in range(nB):
            for j in idx[bh, i, :counts[bh, i]]:
                m[bh, block * i:block * (i + 1), block * j:block * (j + 1)] = True
    return m


def test_attention_dense_equals_sdpa():
    rng = np.random.default_rng(4)
    Q, K, V = (_bits(rng.standard_normal((1, 2, 256, 64))) for _ in range(3))
    cls = oracle.layout([], 256)
    idx, counts = oracle.select(np.zeros((2, 4, 4)), cls, 2, 1.0)
    got = oracle.attention(Q, K, V, 2, idx, counts)
    ref = torch.nn.functional.scaled_dot_product_attention(*(torch.from_numpy(_f64(x)) for x in (Q, K, V))).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_attention_sparse_equals_masked_sdpa():
    w = WORKLOADS["tiny"]
    Q, K, V = make_qkv(w)
    cls = oracle.layout(list(w.segments), w.N)
    hm = head_mask_for_layer(w)
    sc = oracle.scores(oracle.pool(Q), oracle.pool(K)).reshape(-1, w.nB, w.nB)
    idx, counts = oracle.select(sc, cls, w.H, 0.5, hm)
    got = oracle.attention(Q, K, V, w.H, idx, counts, hm)
    mask = _token_mask(idx.reshape(-1, w.nB, idx.shape[-1]), counts.reshape(-1, w.nB), w.N)
    ref = _torch_masked_attention(Q[0], K[0], V[0], mask)
    for h in range(w.H):
        rows_live = np.repeat(counts[h] > 0, 64)
        if hm[h]:
            np.testing.assert_allclose(got[0, h][rows_live], ref[h][rows_live], rtol=1e-12, atol=1e-12)
            assert np.all(got[0, h][~rows_live] == 0)
        else:
            assert np.all(got[0, h] == 0)


def test_attention_closed_forms():
    rng = np.random.default_rng(5)
    N, d = 512, 64
    K = _bits(rng.standard_normal((1, 1, N, d)))
    V = _bits(rng.standard_normal((1, 1, N, d)))
    cls = oracle.layout([], N)
    sc = rng.standard_normal((1, 8, 8))
    idx, counts = oracle.select(sc, cls, 1, 0.4)
    # Q = 0: uniform weights -> mean of V over the kept keys
    out = oracle.attention(np.zeros((1, 1, N, d), np.uint16), K, V, 1, idx, counts)
    Vf = _f64(V)[0, 0]
    for i in range(8):
        keys = np.concatenate([np.arange(64 * j, 64 * j + 64) for j in idx[0, i, :counts[0, i]]])
        np.testing.assert_allclose(out[0, 0, 64 * i:64 * i + 64], np.broadcast_to(Vf[keys].mean(0), (64, d)),
                                   rtol=1e-12, atol=1e-12)
    # V = c: output c on every live row
    Q = _bits(rng.standard_normal((1, 1, N, d)))
    out = oracle.attention(Q, K, _bits(np.full((1, 1, N, d), -1.5)), 1, idx, counts)
    np.testing.assert_allclose(out, -1.5, rtol=0, atol=1e-12)
    # a single kept tile: a 64-key softmax by brute force
    one_idx = np.full((1, 8, 1), 3, np.int32)
    one_cnt = np.ones((1, 8), np.int32)
    out = oracle.attention(Q, K, V, 1, one_idx, one_cnt, rows=np.array([5, 300]))
    for t, row in enumerate((5, 300)):
        s = _f64(K)[0, 0, 192:256] @ _f64(Q)[0, 0, row] / np.sqrt(d)
        p = np.exp(s - s.max())
        np.testing.assert_allclose(out[t], (p / p.sum()) @ Vf[192:256], rtol=1e-12, atol=1e-12)


def test_attention_rows_subset_matches_full():
    w = WORKLOADS["tiny"]
    Q, K, V = make_qkv(w)
    cls = oracle.layout(list(w.segments), w.N)
    idx, counts = oracle.pattern(cls, oracle.PAT_RADIAL, w.H, w.H, density=0.5)
    full = oracle.attention(Q, K, V, w.H, idx, counts).reshape(-1, w.d)
    rows = np.array([0, 77, 130, 511, 512 + 200, 3 * 512 + 511])
    np.testing.assert_array_equal(oracle.attention(Q, K, V, w.H, idx, counts, rows=rows), full[rows])


# ---------------------------------------------------------------- grouped key/value heads

def test_grouped_attention_dense_equals_sdpa_gqa():
    # 6 query heads over 2 key/value heads, two batches: torch SDPA's grouped mode in fp64
    rng = np.random.default_rng(8)
    Q = _bits(rng.standard_normal((2, 6, 256, 64)))
    K, V = (_bits(rng.standard_normal((2, 2, 256, 64))) for _ in range(2))
    cls = oracle.layout([], 256)
    idx, counts = oracle.select(np.zeros((12, 4, 4)), cls, 6, 1.0)
    got = oracle.attention(Q, K, V, 6, idx, counts)
    ref = torch.nn.functional.scaled_dot_product_attention(*(torch.from_numpy(_f64(x)) for x in (Q, K, V)),
                                                           enable_gqa=True).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_grouped_heads_equal_multi_head_on_repeated_keys():
    # sharing a key/value head is multi-head attention on keys and values repeated per group
    w = WORKLOADS["tiny"]
    rng = np.random.default_rng(9)
    B, H, Hkv, N, d = 2, 4, 2, w.N, 64
    Q = _bits(rng.standard_normal((B, H, N, d)))
    K, V = (_bits(rng.standard_normal((B, Hkv, N, d))) for _ in range(2))
    Kr, Vr = (np.repeat(x, H // Hkv, axis=1) for x in (K, V))
    qbar, kbar = oracle.pool(Q), oracle.pool(K)
    s = oracle.scores(qbar, kbar)
    np.testing.assert_array_equal(s, oracle.scores(qbar, oracle.pool(Kr)))
    assert not np.array_equal(s[0, 1], s[0, 2])  # heads 1 and 2 read different key heads
    cls = oracle.layout(list(w.segments), N)
    idx, counts = oracle.select(s.reshape(-1, w.nB, w.nB), cls, H, 0.5)
    np.testing.assert_array_equal(oracle.attention(Q, K, V, H, idx, counts),
                                  oracle.attention(Q, Kr, Vr, H, idx, counts))


def test_grouped_heads_reject_a_partial_group():
    q = np.zeros((1, 6, 2, 8))
    with pytest.raises(ValueError):
        oracle.scores(q, np.zeros((1, 4, 2, 8)))


# ---------------------------------------------------------------- token-level key mask inside kept tiles

def _key_mask_case(seed=12):
    """Two batches of the tiny layout, each with its own live prompt length:
    keys past the live text (inside the straddling pinned block) and the
    padding are masked."""
    w = WORKLOADS["tiny"]
    rng = np.random.default_rng(seed)
    B, H, N, d = 2, 2, w.N, w.d
    Q, K, V = (_bits(rng.standard_normal((B, H, N, d))) for _ in range(3))
    km = np.ones((B, N), np.uint8)
    km[0, 25:128] = 0   # batch 0: 25 live text tokens
    km[1, 40:128] = 0   # batch 1: 40
    cls = oracle.layout(list(w.segments), N)
    sc = oracle.scores(oracle.pool(Q), oracle.pool(K)).reshape(-1, w.nB, w.nB)
    idx, counts = oracle.select(sc, cls, H, 0.5)
    return w, Q, K, V, km, idx, counts


def test_key_mask_equals_masked_sdpa():
    w, Q, K, V, km, idx, counts = _key_mask_case()
    B, H, N = Q.shape[0], Q.shape[1], w.N
    got = oracle.attention(Q, K, V, H, idx, counts, key_mask=km)
    tiles = _token_mask(idx.reshape(-1, w.nB, idx.shape[-1]), counts.reshape(-1, w.nB), N).reshape(B, H, N, N)
    mask = tiles & (km[:, None, None, :] != 0)
    live = mask.any(-1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(_f64(x)) for x in (Q, K, V)), attn_mask=torch.from_numpy(mask)).numpy()
    np.testing.assert_allclose(got[live], ref[live], rtol=1e-12, atol=1e-12)
    assert np.all(got[~live] == 0)
    # the two batches' masks differ: the result depends on each batch's own mask
    swapped = oracle.attention(Q, K, V, H, idx, counts, key_mask=km[::-1].copy())
    assert not np.allclose(swapped[0], got[0])


def test_key_mask_of_ones_changes_nothing():
    w, Q, K, V, _, idx, counts = _key_mask_case()
    np.testing.assert_array_equal(oracle.attention(Q, K, V, 2, idx, counts, key_mask=np.ones((2, w.N), np.uint8)),
                                  oracle.attention(Q, K, V, 2, idx, counts))


def test_key_mask_closed_forms():
    w, _, K, V, km, idx, counts = _key_mask_case()
    B, H, N = K.shape[0], K.shape[1], w.N
    out = oracle.attention(np.zeros_like(K), K, V, H, idx, counts, key_mask=km)
    Vf = _f64(V)
    for b, h, i in ((0, 0, 0), (1, 1, 0), (0, 1, 5), (1, 0, 7)):
        keys = np.concatenate([np.arange(64 * j, 64 * j + 64) for j in idx[b * H + h, i, :counts[b * H + h, i]]])
        keys = keys[km[b, keys] != 0]
        np.testing.assert_allclose(out[b, h, 64 * i:64 * i + 64], np.broadcast_to(Vf[b, h, keys].mean(0), (64, w.d)),
                                   rtol=1e-12, atol=1e-12)
    # a row whose only kept tile is fully masked gives exact zeros
    one_idx = np.full((B * H, w.nB, 1), 1, np.int32)
    one_cnt = np.ones((B * H, w.nB), np.int32)
    out = oracle.attention(_bits(np.ones((B, H, N, w.d))), K, V, H, one_idx, one_cnt, key_mask=km)
    assert np.all(out == 0)


# ---------------------------------------------------------------- random-block control pattern

@pytest.mark.parametrize("name", ["tiny", "joint"])
def test_random_pattern_invariants(name):
    w = WORKLOADS[name]
    cls = oracle.layout(list(w.segments), w.N)
    rho = w.densities[0]
    C, P = int(np.sum(cls == oracle.SPARSE)), int(np.sum(cls == oracle.PIN))
    k = oracle.budget(rho, C)
    idx, counts = oracle.pattern(cls, oracle.PAT_RANDOM, 1, 1, density=rho, seed=7)
    pins = set(np.flatnonzero(cls == oracle.PIN).tolist())
    for i in range(w.nB):
        row = idx[0, i, :counts[0, i]].tolist()
        if cls[i] == oracle.DROP:
            assert counts[0, i] == 0
        elif cls[i] == oracle.PIN:
            assert row == np.flatnonzero(cls != oracle.DROP).tolist()
        else:
            assert len(row) == P + k and i in row and pins <= set(row)
            assert all(cls[j] != oracle.DROP for j in row) and row == sorted(set(row))
    again, _ = oracle.pattern(cls, oracle.PAT_RANDOM, 1, 1, density=rho, seed=7)
    other, _ = oracle.pattern(cls, oracle.PAT_RANDOM, 1, 1, density=rho, seed=8)
    assert np.array_equal(again, idx) and not np.array_equal(other, idx)


def test_random_pattern_draws_uniform_subsets():
    # 6 sparsifiable blocks, k = 3: the diagonal plus 2 of the other 5, each of the 10 pairs equally likely
    cls = np.full(6, oracle.SPARSE, np.uint8)
    n = 20000
    for i in (0, 3):
        tally = {}
        for seed in range(n):
            idx, counts = oracle.pattern(cls, oracle.PAT_RANDOM, 1, 1, density=0.5, seed=seed)
            row = idx[0, i, :counts[0, i]].tolist()
            assert len(row) == 3 and i in row
            key = tuple(j for j in row if j != i)
            tally[key] = tally.get(key, 0) + 1
        assert len(tally) == 10
        # each count is Binomial(20000, 0.1): mean 2000, sd 42.4; 250 is about 6 sd
        assert all(abs(c - n / 10) < 250 for c in tally.values()), tally
