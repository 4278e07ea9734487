"""The seeded input generator (CPU): rounding, shapes, structure and seeding.

The generator is shared by the CUDA path's tests and bench and by the oracle,
so what it states (bf16 round-to-nearest-even, the rank-8 position term on
image tokens only, independent seeded streams) is checked here against
torch's own conversion and plain properties.
"""
import numpy as np
import torch

from workloads import (SEG_IMAGE, WORKLOADS, bf16_bits_from_f32, bf16_bits_to_f32, head_mask_for_layer, make_qkv,
                       make_workload)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 100000),
                        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-40, np.inf, -np.inf], np.float32)])
    ours = bf16_bits_from_f32(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_ties_go_to_even():
    # 1 + 2^-8 lies halfway between the bf16 neighbours 1 and 1 + 2^-7: the even one (1) wins;
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6: 1 + 2^-6 (even mantissa) wins
    x = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8], np.float32)
    assert bf16_bits_to_f32(bf16_bits_from_f32(x)).tolist() == [1.0, 1 + 2.0 ** -6]


def test_shapes_and_seeding():
    w = WORKLOADS["tiny"]
    Q, K, V = make_qkv(w, seed=3)
    assert Q.shape == K.shape == V.shape == (w.B, w.H, w.N, w.d) and Q.dtype == np.uint16
    Q2, _, _ = make_qkv(w, seed=3)
    Q3, _, _ = make_qkv(w, seed=4)
    assert np.array_equal(Q, Q2) and not np.array_equal(Q, Q3)
    assert not np.array_equal(Q, K)  # separate streams per tensor
    # one head drawn alone equals that head of the full draw
    Qh, Kh, Vh = make_qkv(w, seed=3, heads=[2])
    assert np.array_equal(Qh[:, 0], Q[:, 2]) and np.array_equal(Vh[:, 0], V[:, 2])


def test_position_term_only_on_image_tokens():
    # joint: text and padding tokens carry no position term, so Q and K there are 0.5 * N(0, 1) alone;
    # image tokens add the rank-8 term, shared between Q and K of a head
    w = make_workload("joint", H=2)
    Q, K, _ = make_qkv(w, seed=5)
    q, k = bf16_bits_to_f32(Q)[0, 0], bf16_bits_to_f32(K)[0, 0]
    img = [s for kind, s, l in w.segments if kind == SEG_IMAGE][0]
    assert abs(np.std(q[:img]) - 0.5) < 0.01
    assert np.std(q[img:]) > 0.6
    # within a head, image-token Q.K correlates with position: nearby tokens score above far ones
    near = np.mean(np.sum(q[img:img + 2000] * k[img + 1:img + 2001], axis=1))
    far = np.mean(np.sum(q[img:img + 2000] * k[img + 8000:img + 10000], axis=1))
    assert near > far + 5.0


def test_head_masks_keep_enough_heads():
    w = WORKLOADS["stack"]
    for layer in range(w.layers):
        m = head_mask_for_layer(w, layer)
        assert m.sum() == 16 and m.sum() >= w.min_active
        runs = m.reshape(8, 4)
        assert np.all((runs == 0).all(1) | (runs == 1).all(1))  # whole runs of 4 dropped
