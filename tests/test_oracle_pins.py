"""The CPU oracle against what the pages and the mathematics fix (no GPU)."""

import pytest
import torch

import oracle
from oracle_pins import ALL_PINS, load_table, permute_formulation, table_names


def _bound(lib_of):
    """The oracle bound to one build of its C library: the plain single-threaded
    one, or the OpenMP one that splits the outer (r, b) loops over the cores."""
    def run(xs, mode, chunked):
        return oracle.ulysses_a2a(xs, mode, chunked, lib=lib_of())

    def pitched(*args, **kw):
        return oracle.ulysses_a2a_pitched(*args, lib=lib_of(), **kw)

    run.pitched = pitched
    return run


_run = _bound(oracle._get_lib)
BUILDS = {"plain": _run, "openmp": _bound(oracle.omp_lib)}


@pytest.mark.parametrize("build", sorted(BUILDS))
@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin, build):
    pin(BUILDS[build])


@pytest.mark.parametrize("build", sorted(BUILDS))
@pytest.mark.parametrize("E", [1, 2, 4, 8])
def test_hand_tables_every_element_size(E, build):
    from oracle_pins import pin_hand_tables
    pin_hand_tables(BUILDS[build], elem_bytes=E)


def test_openmp_build_uses_several_threads_and_matches_on_a_larger_shape():
    # the split over (r, b) must not change a byte, also with more (r, b)
    # pairs than threads and a ragged plane count
    from synth import unique_slabs
    xs = unique_slabs((5, 33, 12, 7), 6, 4)
    y_plain = oracle.ulysses_a2a(xs, 0)
    y_omp = oracle.ulysses_a2a(xs, 0, lib=oracle.omp_lib())
    assert all(torch.equal(a, b) for a, b in zip(y_plain, y_omp))
    back = oracle.ulysses_a2a(y_omp, 1, lib=oracle.omp_lib())
    assert all(torch.equal(a, b) for a, b in zip(back, xs))
    assert oracle.omp_threads() >= 1


def test_tables_are_well_formed():
    # each table lists every input symbol exactly once across its outputs
    for name in table_names():
        w, (B, S, H, D), ins, outs = load_table(name)
        assert len(ins) == w and len(outs) == w
        assert sorted(s for l in ins for s in l) == sorted(s for l in outs for s in l)
        assert all(len(l) == B * S * H * D for l in ins + outs)


def test_output_shapes_follow_run_armed():
    # FastVideo API docs, ulysses_a2a `run_armed`: mode 0 -> [B, S_local*w, H//w, D];
    # mode 1 -> [B, S_global//w, H_local*w, D]
    assert oracle.output_shape((2, 4725, 40, 128), 0, 8) == (2, 4725 * 8, 5, 128)
    assert oracle.output_shape((2, 4725 * 8, 5, 128), 1, 8) == (2, 4725, 40, 128)
    assert oracle.mode0_local_tuple((2, 4725 * 8, 5, 128), 1, 8) == (2, 4725, 40, 128)
    w = 4
    x = [torch.zeros(1, 3, 8, 2, dtype=torch.bfloat16) for _ in range(w)]
    y = oracle.ulysses_a2a(x, 0)
    assert all(tuple(t.shape) == (1, 12, 2, 2) for t in y)
    z = oracle.ulysses_a2a(y, 1)
    assert all(tuple(t.shape) == (1, 3, 8, 2) for t in z)


def test_rejects_bad_arguments():
    x = [torch.zeros(1, 2, 3, 4) for _ in range(2)]
    with pytest.raises(ValueError):
        oracle.ulysses_a2a(x, 0)          # H = 3 not divisible by w = 2
    with pytest.raises(ValueError):
        oracle.ulysses_a2a([torch.zeros(1, 3, 2, 4) for _ in range(2)], 1)  # S_global % w
    lib = oracle._get_lib()
    import ctypes
    arr = (ctypes.c_void_p * 2)(None, None)
    assert lib.oracle_ulysses_a2a(arr, arr, 1, 1, 2, 1, 2, 0, 2) == -1
    good = [torch.zeros(4) for _ in range(4)]
    a = (ctypes.c_void_p * 2)(good[0].data_ptr(), good[1].data_ptr())
    b = (ctypes.c_void_p * 2)(good[2].data_ptr(), good[3].data_ptr())
    assert lib.oracle_ulysses_a2a(a, b, 1, 1, 2, 1, 2, 2, 4) == -1    # mode 2
    assert lib.oracle_ulysses_a2a(a, b, -1, 1, 2, 1, 2, 0, 4) == -1   # B < 0
    assert lib.oracle_ulysses_a2a(a, b, 1, 1, 2, 1, 2, 0, 4) == 0


def test_empty_index_sets_are_a_no_op():
    # the definition over an empty index set moves nothing; NULL slabs allowed
    import ctypes
    lib = oracle._get_lib()
    nul = (ctypes.c_void_p * 2)(None, None)
    for (B, S, H, D) in [(0, 3, 4, 2), (2, 0, 4, 2), (2, 3, 0, 2), (2, 3, 4, 0)]:
        assert lib.oracle_ulysses_a2a(nul, nul, B, S, H, D, 2, 0, 2) == 0
        assert lib.oracle_ulysses_a2a_chunked(nul, nul, B, S, H, D, 2, 1, 2) == 0
        x = [torch.zeros(B, S, H, D) for _ in range(2)]
        y = oracle.ulysses_a2a(x, 0)
        assert all(tuple(t.shape) == (B, S * 2, H // 2, D) for t in y)
    # a zero size does not hide a non-empty slab's NULL pointer
    assert lib.oracle_ulysses_a2a(nul, nul, 1, 1, 2, 1, 2, 0, 2) == -1


# ---- the same facts over random small shapes (property test) ------------------

from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@settings(max_examples=200, deadline=None, derandomize=True, database=None)
@given(w=st.integers(1, 6), hw=st.integers(1, 4), B=st.integers(1, 3), S=st.integers(1, 9),
       D=st.integers(1, 9), E=st.sampled_from([1, 2, 4, 8]), seed=st.integers(0, 2**31 - 1))
def test_oracle_properties_on_random_shapes(w, hw, B, S, D, E, seed):
    """mode 1 undoes mode 0, the maps agree with the independent permute
    formulation, and chunked equals unchunked, on random small shapes."""
    H = hw * w
    dt = {1: torch.uint8, 2: torch.int16, 4: torch.int32, 8: torch.int64}[E]
    g = torch.Generator().manual_seed(seed)
    xs = [torch.randint(0, 100, (B, S, H, D), generator=g, dtype=torch.int64).to(dt)
          for _ in range(w)]
    y = oracle.ulysses_a2a(xs, 0)
    want = permute_formulation(xs, 0, w)
    for r in range(w):
        assert torch.equal(y[r], want[r])
    z = oracle.ulysses_a2a(y, 1)
    for j in range(w):
        assert torch.equal(z[j], xs[j])
    yc = oracle.ulysses_a2a(xs, 0, chunked=True)
    for r in range(w):
        assert torch.equal(yc[r], y[r])
