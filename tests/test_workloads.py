"""The seeded input recipe: value sets and distributions, bf16 rounding,
determinism per seed, and the paged cache's table (CPU only)."""

import numpy as np

from workloads import CONFIGS, bf16_bits, bf16_to_f64, gen_decode, gen_prefill, unpage


def test_prefill_recipe_values_and_determinism():
    a = gen_prefill(N=777, Hq=4, d=64, H_I=4, D_I=64, seed=3)
    b = gen_prefill(N=777, Hq=4, d=64, H_I=4, D_I=64, seed=3)
    c = gen_prefill(N=777, Hq=4, d=64, H_I=4, D_I=64, seed=4)
    for name in ("q", "k", "v", "qI", "kI", "w"):
        assert a[name].dtype == np.uint16
        assert np.array_equal(a[name], b[name])          # same seed, same bits
        assert not np.array_equal(a[name], c[name])      # another seed, another draw
    qI, kI, w = (bf16_to_f64(a[x]) for x in ("qI", "kI", "w"))
    assert set(np.unique(qI)) == set(range(-3, 4)) and set(np.unique(kI)) == set(range(-3, 4))
    assert set(np.unique(w)) == {0, 1, 2, 3}
    q = bf16_to_f64(a["q"])
    assert abs(q.mean()) < 0.02 and abs(q.std() - 1.0) < 0.02   # N(0,1), 199k draws
    # every value is its own bf16 rounding (the generator stores bf16 bits)
    assert np.array_equal(bf16_bits(q.astype(np.float32)), a["q"])


def test_streams_are_independent_of_shapes_of_other_tensors():
    # one stream per tensor: changing the indexer shape leaves q, k, v unchanged
    a = gen_prefill(N=100, Hq=2, d=64, H_I=2, D_I=32, seed=0)
    b = gen_prefill(N=100, Hq=2, d=64, H_I=8, D_I=64, seed=0)
    for name in ("q", "k", "v"):
        assert np.array_equal(a[name], b[name])


def test_paged_decode_table_is_a_permutation_and_unpages_to_the_lengths():
    lengths = [1, 64, 65, 1000, 130]
    d = gen_decode(B=5, lengths=lengths, Hq=8, d=64, H_I=2, D_I=32, paged=True, seed=2)
    table, P = d["page_table"], d["k"].shape[0]
    n_pages = [(L + 63) // 64 for L in lengths]
    assert table.shape == (5, max(n_pages)) and P == sum(n_pages)
    used = np.concatenate([table[b, :n] for b, n in enumerate(n_pages)])
    assert np.array_equal(np.sort(used), np.arange(P))           # every page once
    for b, n in enumerate(n_pages):
        assert np.all(table[b, n:] == -1)
        assert unpage(d["kI"], table[b], lengths[b]).shape == (lengths[b], 32)
    assert not np.array_equal(used, np.arange(P))                 # shuffled


def test_decode_lengths_of_the_paged_workload():
    c = dict(CONFIGS["decode_paged_16x256k"])
    c.update(Hq=1, d=8, H_I=1, D_I=8)          # the workload's lengths and pages, small rows
    d = gen_decode(seed=0, **c)
    L = d["lengths"]
    assert len(L) == 16 and L.min() >= 16384 and L.max() <= 262144 and len(np.unique(L)) > 8
    assert d["page_table"].shape == (16, int(((L + 63) // 64).max()))
