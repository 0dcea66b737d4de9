"""CPU checks of the C ABI library: it loads, exports every declared entry point,
and its host-side code (recipe, per-pass order) agrees with the oracle. No GPU
compute is called here."""

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
