"""The seeded input recipe (CPU): shapes, determinism, routing laws, weights, token rounding.

These inputs feed both the oracle and the CUDA path, so their stated properties are pinned here:
k distinct experts per token, softmax weights, bf16 round-to-nearest-even tokens, the mask of the
masked sweep, tokens drawn last, and the Zipf law of the prefill and replica routing.
"""
import numpy as np
import pytest

from combine_get_dispatch_histogram_b200 import inputs


@pytest.mark.parametrize("name", ["tiny", "decode", "sweep_T16_mask5", "replica", "prefill"])
def test_workload_inputs(name):
    w = inputs.named(name)
    a = inputs.make_inputs(w, tokens=False)
    b = inputs.make_inputs(w, tokens=False)
    R, T, k, E = w.num_ranks, w.num_tokens, w.num_topk, w.num_experts
    assert a.topk_idx.shape == (R, T, k) and a.topk_idx.dtype == np.int32
    assert a.topk_weights.shape == (R, T, k) and a.topk_weights.dtype == np.float32
    assert np.array_equal(a.topk_idx, b.topk_idx) and np.array_equal(a.topk_weights, b.topk_weights)
    idx = a.topk_idx.reshape(-1, k)
    assert idx.min() >= 0 and idx.max() < E
    assert np.all(np.sort(idx, axis=1)[:, 1:] != np.sort(idx, axis=1)[:, :-1])   # distinct per token
    wts = a.topk_weights.reshape(-1, k)
    assert np.all(wts > 0) and np.allclose(wts.sum(axis=1), 1.0, atol=1e-6)
    want_active = np.ones(R, np.uint8)
    for r in w.inactive:
        want_active[r] = 0
    assert np.array_equal(a.active, want_active)
    assert a.x is None


def test_masked_sweep_and_names():
    w = inputs.named("sweep_T64_mask5")
    assert (w.num_ranks, w.num_tokens, w.num_topk, w.num_experts, w.hidden) == (8, 64, 8, 256, 7168)
    assert w.inactive == (5,)
    assert inputs.named("sweep_T64").inactive == ()
    r = inputs.named("replica")
    assert (r.num_experts, r.num_extra, r.num_physical, r.num_topk, r.hidden) == (64, 16, 80, 6, 4096)


def test_tokens_are_drawn_last():
    """Dropping the token tensor leaves routing and weights unchanged."""
    w = inputs.named("tiny")
    a = inputs.make_inputs(w, tokens=True)
    b = inputs.make_inputs(w, tokens=False)
    assert np.array_equal(a.topk_idx, b.topk_idx) and np.array_equal(a.topk_weights, b.topk_weights)
    assert a.x.shape == (w.num_ranks, w.num_tokens, w.hidden) and a.x.dtype == np.uint16


def test_tokens_round_to_nearest_even():
    """bf16 bits equal an independent round-to-nearest-even of the same float32 draws."""
    bits = inputs.bf16_tokens(np.random.default_rng(3), 64, 256)
    f = np.random.default_rng(3).standard_normal((64, 256), dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    want = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)    # finite draws: no NaN case
    assert np.array_equal(bits, want)


def test_zipf_first_slot_follows_the_law():
    """With the Gumbel top-k draw, slot 0 is distributed exactly as p[perm[i]] ~ (i+1)^-s."""
    n, E, k, s = 200_000, 64, 6, 1.5
    idx = inputs.zipf_topk(np.random.default_rng(11), n, E, k, s)
    perm = np.random.default_rng(11).permutation(E)                    # the generator's first draw
    p = (np.arange(1, E + 1, dtype=np.float64) ** -s)
    p /= p.sum()
    freq = np.bincount(idx[:, 0], minlength=E) / n
    for i in range(8):                                                  # the eight most popular
        sigma = np.sqrt(p[i] * (1 - p[i]) / n)
        assert abs(freq[perm[i]] - p[i]) < 6 * sigma, (i, freq[perm[i]], p[i])
    assert np.all(np.sort(idx, axis=1)[:, 1:] != np.sort(idx, axis=1)[:, :-1])


def test_uniform_routing_is_uniform():
    n, E, k = 100_000, 32, 4
    idx = inputs.uniform_topk(np.random.default_rng(5), n, E, k)
    for j in range(k):
        freq = np.bincount(idx[:, j], minlength=E) / n
        sigma = np.sqrt((1 / E) * (1 - 1 / E) / n)
        assert np.all(np.abs(freq - 1 / E) < 6 * sigma)
