"""Plant plausible mistakes in a copy of the CPU oracle and check the pins catch them.

Each mutation edits one spot of ``oracle/ulysses_oracle.c`` in a temporary copy,
builds it with gcc and runs every pin from ``oracle_pins``. A mutation that no pin
notices would mean the pins leave that part of the oracle unchecked. Every
mutation below keeps all memory accesses inside the slabs (checked by reading the
index bounds), so a broken copy can give wrong bytes but never crash.
"""

import os

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "ulysses_oracle.c")

MUTATIONS = {
    # mode 0 reads the destination rank's slab instead of the source rank's
    "mode0_wrong_source_rank": (
        "const char *src = (const char *)in[j] + a * E;",
        "const char *src = (const char *)in[r] + a * E;"),
    # mode 1 writes into the source rank's slab
    "mode1_wrong_dest_rank": (
        "char *dst = (char *)out[j] + a * E;",
        "char *dst = (char *)out[r] + a * E;"),
    # the head group taken from the strided side follows j instead of r
    "head_group_index": (
        "int64_t a = at4(b, s, r * Hw + hp, d,",
        "int64_t a = at4(b, s, (int64_t)j * Hw + hp, d,"),
    # the gathered sequence block follows r instead of j
    "sequence_block_index": (
        "int64_t c = at4(b, (int64_t)j * S_local + s, hp, d,",
        "int64_t c = at4(b, (int64_t)r * S_local + s, hp, d,"),
    # gathered side indexed with the local sequence length as its row count
    "gathered_row_extent": (
        "S_global, Hw, D);",
        "S_local, Hw, D);"),
    # batch-plane offset forgotten in the row-major offset
    "drops_plane_offset": (
        "return ((b * S + s) * Hn + h) * D + d;",
        "return (s * Hn + h) * D + d;"),
    # head and feature strides transposed in the row-major offset
    "head_feature_transposed": (
        "return ((b * S + s) * Hn + h) * D + d;",
        "return (b * S + s) * Hn * D + d * Hn + h;"),
    # last sequence row of every block never copied
    "drops_last_row": (
        "for (int64_t s = 0; s < S_local; ++s)",
        "for (int64_t s = 0; s < S_local - 1; ++s)"),
    # copies only the first byte of each element
    "partial_element": (
        "memcpy(dst, src, (size_t)E);\n                            } else {",
        "memcpy(dst, src, (size_t)1);\n                            } else {"),
    # chunked driver steps planes with the wrong stride
    "chunked_plane_stride": (
        "const int64_t plane = S_local * H * D;",
        "const int64_t plane = S_local * D * w;"),
    # pitched side indexed as if dense (row pitch ignored)
    "pitch_ignored": (
        "int64_t a = (b * S_local + s) * row_pitch",
        "int64_t a = (b * S_local + s) * (H * D)"),
    # pitched side: head group taken from the source rank
    "pitched_head_group": (
        "+ (r * Hw + hp) * D + d;",
        "+ ((int64_t)j * Hw + hp) * D + d;"),
    # mode 1 copies the wrong way round (reads the destination layout's offset)
    "mode1_swapped_offsets": (
        "const char *src = (const char *)in[r] + c * E;",
        "const char *src = (const char *)in[r] + a * E;"),
}


def _run_all_pins(lib):
    def run(xs, mode, chunked):
        return oracle.ulysses_a2a(xs, mode, chunked, lib=lib)

    def pitched(*a, **k):
        return oracle.ulysses_a2a_pitched(*a, lib=lib, **k)

    run.pitched = pitched
    failed = []
    for pin in ALL_PINS:
        try:
            pin(run)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


# the same edits applied to the second copy of a loop (the pitched function)
MUTATIONS.update({
    "pitched_drops_last_row": (
        "for (int64_t s = 0; s < S_local; ++s)",
        "for (int64_t s = 0; s < S_local - 1; ++s)", 1),
    "pitched_partial_element": (
        "memcpy(dst, src, (size_t)E);\n                            } else {",
        "memcpy(dst, src, (size_t)1);\n                            } else {", 1),
})


def _apply(text, old, new, nth=0):
    """Replace the nth occurrence (0-based) of `old` in `text`."""
    at = -1
    for _ in range(nth + 1):
        at = text.find(old, at + 1)
        assert at >= 0, "mutation anchor not found"
    return text[:at] + new + text[at + len(old):]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, tmp_path):
    old, new, *nth = MUTATIONS[name]
    text = open(SRC).read()
    mutated = tmp_path / "mutated.c"
    mutated.write_text(_apply(text, old, new, nth[0] if nth else 0))
    so = oracle.build(force=True, src=str(mutated), out=str(tmp_path / f"lib_{name}.so"),
                      extra=("-Wno-unused-variable", "-Wno-error"))
    lib = oracle.load_library(so)
    failed = _run_all_pins(lib)
    assert failed, f"no pin noticed mutation {name}"
