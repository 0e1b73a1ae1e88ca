"""Pins for the oracle's bit allocation (O7), packing and the whole layer."""
import itertools
import json
import os

import numpy as np
import pytest

from oracle import alloc, pack, pipeline
from synth import tiny_layer


@pytest.mark.parametrize("L", [3, 5, 8])
def test_greedy_equals_brute_force_equal_sizes(L):
    rng = np.random.default_rng(L)
    for _ in range(5):
        s = np.exp(rng.normal(size=L) * 2)
        sizes = [16] * L
        got = alloc.allocate_budget(s, sizes, 2.5, 2, 4)
        best = min(alloc.expected_cost(s, b)
                   for b in itertools.product((2, 3, 4), repeat=L)
                   if sum(b) * 16 <= 2.5 * 16 * L)
        assert sum(b * 16 for b in got) <= 2.5 * 16 * L
        assert abs(alloc.expected_cost(s, got) - best) <= 1e-12 * best


def test_allocation_unequal_sizes_feasible_and_maximal():
    rng = np.random.default_rng(3)
    s = np.exp(rng.normal(size=7) * 2)
    sizes = [4096 * 4096, 1024 * 4096, 1024 * 4096, 4096 * 4096, 14336 * 4096, 14336 * 4096, 4096 * 14336]
    b = alloc.allocate_budget(s, sizes, 2.5)
    used = sum(bi * si for bi, si in zip(b, sizes))
    assert used <= 2.5 * sum(sizes)
    assert all(2 <= bi <= 4 for bi in b)
    for i in range(7):        # no further upgrade fits
        assert b[i] == 4 or used + sizes[i] > 2.5 * sum(sizes)


def test_allocation_ties_go_to_lower_index():
    b = alloc.allocate_budget([1.0, 1.0, 1.0, 1.0], [1, 1, 1, 1], 2.25)
    assert b == [3, 2, 2, 2]


def test_topn_types():
    s = [1.0, 5.0, 2.0, 1.0, 6.0, 2.5]
    types = ["q", "k", "v", "q", "k", "v"]
    assert alloc.allocate_topn_types(s, types, 2, 1) == [2, 3, 2, 2, 3, 2]
    assert alloc.allocate_topn_types(s, types, 2, 2) == [2, 3, 3, 2, 3, 3]


def test_pack_hand_worked_words(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "pack_words.json")))
    w4 = pack.pack(np.array([g["int4_codes"]]), 4)
    assert [hex(int(v)) for v in w4[0]] == g["int4_words"]
    w2 = pack.pack(np.array([g["int2_codes"]]), 2)
    assert [hex(int(v)) for v in w2[0]] == g["int2_words"]


@pytest.mark.parametrize("bits,n", [(4, 64), (2, 64), (4, 13), (2, 37)])
def test_pack_roundtrip(bits, n):
    rng = np.random.default_rng(n)
    codes = rng.integers(0, 2 ** bits, size=(5, n))
    w = pack.pack(codes, bits)
    assert w.shape == (5, pack.words_per_row(n, bits))
    assert np.array_equal(pack.unpack(w, n, bits), codes)


def test_three_bit_not_packable():
    with pytest.raises(ValueError):
        pack.pack(np.zeros((1, 8)), 3)


def test_whole_layer_tiny_config():
    W, X, G = tiny_layer()
    r = pipeline.quantize_layer(X, G, W, bits=4, group=128)
    assert r["codes"].min() >= 0 and r["codes"].max() <= 15
    # the loss of the KronQ result is below the plain RTN loss on the raw W
    from oracle import loss, sweep
    _, Qr = sweep.rtn(W, 4, 128)
    assert r["loss"] < loss.kfac_loss(W - Qr, r["HX"], r["HG"])
    # the loss in the original space equals the rotated-space loss
    dWt = r["Wt"] - r["Q"]
    assert abs(loss.kfac_loss(dWt, r["HXt"], r["HGt"]) - r["loss"]) <= 1e-9 * r["loss"]
