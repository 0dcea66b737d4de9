"""CPU checks of the C ABI library: it loads, exports every declared entry point,
and its host-side code agrees with the oracle (recipe, per-pass order) and with the
search's documented work units (the search schedule). No GPU compute is called
here."""

import os
import re

import numpy as np
import pytest

from oracle import emeans_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def em():
    import importlib.util

    spec = importlib.util.spec_from_file_location("_b", os.path.join(ROOT, "mini_ema_means_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    import mini_ema_means_b200

    return mini_ema_means_b200


def _declared_functions():
    with open(os.path.join(ROOT, "include", "emeans.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(em_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(em):
    declared = _declared_functions()
    assert len(declared) >= 25
    for name in declared:
        assert hasattr(em.lib, name), f"{name} is declared in include/emeans.h but not exported"
    assert sorted(em.ABI_FUNCTIONS) == declared


def test_binding_constants_match_the_header(em):
    """Every EM_OPT_*, EM_E_*, EM_PHASE_* and EM_REVIVE_* value of the binding is the
    header's."""
    with open(os.path.join(ROOT, "include", "emeans.h")) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    header = {name: int(val) for name, val in re.findall(r"\b(EM_(?:OPT|E|PHASE|REVIVE)_[A-Z_]+)\s*=\s*(-?\d+)", text)}
    header.update({name: int(val) for name, val in
                   re.findall(r"#define\s+(EM_(?:OPT|E|PHASE|REVIVE)_[A-Z_]+)\s+\(?(-?\d+)\)?", text)})
    assert header["EM_OPT_SPHERICAL"] == 16
    for name, val in header.items():
        assert getattr(em, name) == val, name


def test_library_is_the_in_tree_build(em):
    assert os.path.dirname(em.LIB_PATH) == os.path.join(ROOT, "mini_ema_means_b200")


def test_host_recipe_needs_an_explicit_law(em):
    # "auto" (2) depends on d, which the model knows; the host-only recipe refuses it
    with pytest.raises(em.EmeansError):
        em.compute_recipe(10_000, 64, 5.0, 2)


@pytest.mark.parametrize("n,k,T,law,b,a", [
    (10_000, 64, 5, 0, 0, 0.0), (1_000_000, 4096, 5, 0, 0, 0.0), (1_000_000, 16384, 5, 0, 0, 0.0),
    (10_000_000, 65536, 5, 0, 0, 0.0), (100_000_000, 262144, 3, 0, 0, 0.0), (10_000_000, 65536, 5, 1, 0, 0.0),
    (120, 3, 2.5, 0, 12, 0.35), (1_000_000, 4096, 5, 0, 8192, 0.0), (12345, 100, 2.5, 0, 0, 0.0),
    (1000, 10, 0.5, 0, 0, 0.0), (3, 1, 1.0, 0, 0, 0.0), (999_999, 7, 1.3, 1, 0, 0.05),
])
def test_host_recipe_matches_oracle(em, n, k, T, law, b, a):
    r = em.compute_recipe(n, k, T, law, b, a)
    o = O.recipe(n, k, T, ["throughput", "quality"][law], b or None, a or None)
    assert r["batch_size"] == o["batch_size"]
    assert r["alpha0"] == pytest.approx(o["alpha0"], rel=1e-13)
    assert r["total_steps"] == o["total_steps"]
    assert r["passes"] == len(o["epoch_rows"]) and r["rows_last_pass"] == o["epoch_rows"][-1]
    assert r["steps_full_pass"] == -(-n // o["batch_size"]) and r["steps_last_pass"] == o["steps_per_pass"][-1]


@pytest.mark.parametrize("n", [1, 2, 3, 5, 120, 10_000, 65_537, 1_000_000])
@pytest.mark.parametrize("stream,which", [(1, 0), (2, 0), (2, 3)])
def test_host_order_is_the_oracles_bijection(em, n, stream, which):
    idx = np.arange(min(n, 20_000), dtype=np.int64)
    if n > 20_000:
        idx = np.unique(np.concatenate([idx, np.random.default_rng(0).integers(0, n, 5000), [n - 1]]))
    got = em.permutation(n, 1234, stream, which, idx)
    ref = O.permute(idx.astype(np.uint64), n, 1234, stream, which)
    assert np.array_equal(got, ref)


def test_host_order_full_bijection_small(em):
    for n in (7, 1000, 4097):
        p = em.permutation(n, 99, 2, 1, np.arange(n))
        assert np.array_equal(np.sort(p), np.arange(n))


def test_argument_errors(em):
    with pytest.raises(em.EmeansError) as e:
        em.compute_recipe(0, 10, 5)
    assert e.value.code == em.EM_E_INVAL
    with pytest.raises(em.EmeansError):
        em.compute_recipe(100, 10, -1.0)
    with pytest.raises(em.EmeansError):
        em.permutation(10, 1, 2, 0, np.array([10]))


def test_create_without_gpu_fails_loudly(em):
    if em.em_device_count() > 0:
        pytest.skip("a CUDA device is present")
    assert not em.em_create(32, 64, 1234)
    assert b"no CUDA device" in em.em_last_error()
    with pytest.raises(em.EmeansError) as e:
        em.Model(32, 64)
    assert e.value.code == em.EM_E_NODEVICE


# The search's work units, as the search kernel takes them: the first m_full 128-row
# tiles are one unit each over all ceil(k / 256) centroid tiles; every later row
# tile is `split` units, group g covering centroid tiles [g * tpg, (g + 1) * tpg)
# with tpg = ceil(n_tiles / split); min(units, sms) persistent CTAs take the units
# round-robin.
def _units(m_tiles, n_tiles, split, m_full):
    tpg = -(-n_tiles // split)
    units = m_full + (m_tiles - m_full) * split
    u = np.arange(units)
    whole = u < m_full
    v = u - m_full
    m = np.where(whole, u, m_full + v // split)
    g = np.where(whole, 0, v % split)
    nt0 = np.where(whole, 0, g * tpg)
    nt1 = np.where(whole, n_tiles, np.minimum(nt0 + tpg, n_tiles))
    return u, m, g, np.maximum(nt1 - nt0, 0)


@pytest.mark.parametrize("rows,k,expect", [
    (65536, 16384, (2, 444)),   # deep96 batch: 512 row tiles, only the last wave's 68 split
    (65536, 4096, (2, 444)),    # emb768 batch
    (1048576, 65536, (1, 0)),   # sift128 batch: 8192 row tiles fill the waves nearly evenly
    (40000, 2000, (8, 296)),
    (20000, 300, (2, 148)),
    (3000, 40, (1, 0)),         # one centroid tile: never split
    (1, 1, (1, 0)),
])
def test_search_schedule_choices(em, rows, k, expect):
    assert em.search_schedule(rows, k, 148) == expect


def test_search_schedule_covers_every_tile_once_and_keeps_the_longest_cta(em):
    for sms in (148, 132, 7):
        for rows in (1, 127, 128, 5000, 18944, 20000, 40000, 65536, 131072, 1048576):
            for k in (1, 256, 300, 2000, 4096, 16384, 65536):
                split, m_full = em.search_schedule(rows, k, sms)
                m_tiles, n_tiles = -(-rows // 128), -(-k // 256)
                assert split in (1, 2, 4, 8) and (split == 1 or split <= n_tiles)
                assert m_full == 0 or m_full < m_tiles
                assert m_full % sms == 0 and (m_full == 0 or split > 1)
                u, m, g, length = _units(m_tiles, n_tiles, split, m_full)
                # every row tile: all of its centroid tiles, in one unit or in `split`
                assert np.array_equal(np.bincount(m, weights=length, minlength=m_tiles), np.full(m_tiles, n_tiles))
                per_row = np.bincount(m, minlength=m_tiles)
                assert np.all(per_row[:m_full] == 1) and np.all(per_row[m_full:] == split)
                # the longest CTA is within 1.5 % of the best schedule that splits every
                # row tile the same number of ways
                grid = min(len(u), sms)
                longest = np.bincount(u % grid, weights=length).max()
                best_uniform = min(-(-(m_tiles * s) // sms) * -(-n_tiles // s) for s in (1, 2, 4, 8)
                                   if s == 1 or s <= n_tiles)
                assert longest <= best_uniform / 0.985, (sms, rows, k, split, m_full, longest, best_uniform)


def test_search_schedule_argument_errors(em):
    for args in ((0, 10, 148), (10, 0, 148), (10, 10, 0)):
        with pytest.raises(em.EmeansError) as e:
            em.search_schedule(*args)
        assert e.value.code == em.EM_E_INVAL
