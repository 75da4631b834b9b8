"""The seeded input generator: Z-order placement and determinism (CPU)."""
import numpy as np
import torch

from synthetic import WORKLOADS, make_inputs, morton_order, quadtree_order_recursive


def test_morton_matches_recursive_quadrants():
    for G in (1, 2, 4, 8, 32, 128):
        assert np.array_equal(morton_order(G), quadtree_order_recursive(G))


def test_aligned_runs_are_squares():
    # Every aligned run of 4^j sequence positions covers a 2^j x 2^j pixel square; this
    # is what makes a level-l pooled token a 4^l x 4^l spatial average.
    G = 64
    order = morton_order(G)
    r, c = order // G, order % G
    for j in range(1, 6):
        run = 4 ** j
        side = 2 ** j
        rr = r.reshape(-1, run)
        cc = c.reshape(-1, run)
        assert np.all(rr.max(1) - rr.min(1) == side - 1)
        assert np.all(cc.max(1) - cc.min(1) == side - 1)
        assert np.all(rr.min(1) % side == 0) and np.all(cc.min(1) % side == 0)


def test_first_positions_follow_row_major_quadrants():
    # Within each 2x2 square the order is (0,0), (0,1), (1,0), (1,1): row bit above column bit.
    G = 4
    order = morton_order(G)
    assert order[:4].tolist() == [0, 1, 4, 5]
    assert order[4:8].tolist() == [2, 3, 6, 7]


def test_generator_is_deterministic_and_typed():
    a = make_inputs(1, 2, 256, 64, "bf16", "smooth", 7)
    b = make_inputs(1, 2, 256, 64, "bf16", "smooth", 7)
    for key in ("q", "k", "v", "do"):
        assert a[key].dtype == torch.bfloat16
        assert torch.equal(a[key], b[key])
    c = make_inputs(1, 2, 256, 64, "f32", "normal", 7)
    assert c["q"].dtype == torch.float32
    assert not torch.equal(a["q"].float(), c["q"])


def test_smooth_fields_are_spatially_smooth():
    # Neighbouring pixels are strongly correlated, unlike i.i.d. noise.
    x = make_inputs(1, 1, 4096, 64, "f32", "smooth", 3, with_do=False)["q"][0, 0]
    G = 64
    order = morton_order(G)
    img = torch.empty(G * G, 64)
    img[torch.from_numpy(order)] = x
    img = img.reshape(G, G, 64)
    a = img[:, :-1].reshape(-1)
    b = img[:, 1:].reshape(-1)
    corr = torch.corrcoef(torch.stack([a, b]))[0, 1]
    assert corr > 0.9
    assert 0.5 < float(x.std()) < 2.0


def test_config_table():
    assert [w.N for w in WORKLOADS.values()] == [1024, 4096, 16384, 65536, 262144, 65536]
    assert [w.D for w in WORKLOADS.values()] == [64, 64, 64, 64, 64, 128]
    assert WORKLOADS["headline-65536"].level_sizes() == [65536, 4096, 256, 16]
    assert WORKLOADS["headline-65536"].kv_len == 144 and WORKLOADS["scaleout-262144"].kv_len == 288
