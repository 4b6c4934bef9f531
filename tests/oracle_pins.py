"""Checks that pin the CPU oracle to facts fixed outside the oracle itself.

Each pin takes ``run(inputs, mode, chunked) -> outputs`` (the oracle bound to one
build of its C library) and raises ``AssertionError`` when the oracle disagrees
with the fact it checks. ``test_oracle_pins.py`` runs them against the real
oracle; ``test_oracle_mutations.py`` runs them against deliberately broken copies
of the oracle to show that each plausible mistake trips at least one pin.

What the pins rest on (none of it is the oracle's own loop restated):
  * hand-derived tables for tiny shapes (``tests/golden/``);
  * w = 1 is the identity in both modes;
  * mode 1 undoes mode 0 and vice versa, bit for bit;
  * the output shapes printed in the FastVideo API docs' ``run_armed``;
  * a special case that is a textbook matrix transpose (S_local = 1, H = w);
  * an independent formulation through ``torch.permute`` / ``reshape`` (a library
    routine), checked on unique-id inputs so every element is traceable;
  * the chunked per-plane loop gives the same bytes as one call;
  * the copy moves bytes, never values: NaN payloads and -0.0 survive.
"""

from __future__ import annotations

import os

import torch

from synth import normal_slabs, unique_slabs, rank_tagged_slabs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

INT_TYPES = {1: torch.uint8, 2: torch.int16, 4: torch.int32, 8: torch.int64}


def load_table(name):
    """Parse a hand-derived table: returns (w, (B,S,H,D), inputs, outputs) as symbol lists."""
    w = None
    shape = None
    ins, outs = {}, {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, _, rest = line.partition(":")
            parts = head.split()
            if parts[0] == "w":
                w = int(parts[1])
            elif parts[0] == "shape":
                shape = tuple(int(v) for v in parts[1:5])
            elif parts[0] == "in":
                ins[int(parts[1])] = rest.split()
            elif parts[0] == "out":
                outs[int(parts[1])] = rest.split()
    return w, shape, [ins[k] for k in range(w)], [outs[k] for k in range(w)]


def table_names():
    return sorted(n for n in os.listdir(GOLDEN) if n.startswith("hand_"))


def pin_hand_tables(run, elem_bytes=2):
    for name in table_names():
        w, (B, S, H, D), ins, outs = load_table(name)
        symbols = sorted({s for lst in ins for s in lst})
        code = {s: i + 1 for i, s in enumerate(symbols)}
        dt = INT_TYPES[elem_bytes]
        x = [torch.tensor([code[s] for s in lst], dtype=dt).reshape(B, S, H, D) for lst in ins]
        y_want = [torch.tensor([code[s] for s in lst], dtype=dt).reshape(B, S * w, H // w, D)
                  for lst in outs]
        for chunked in (False, True):
            y = run(x, 0, chunked)
            for r in range(w):
                assert torch.equal(y[r], y_want[r]), f"{name}: mode 0 rank {r} (chunked={chunked})"
            back = run(y_want, 1, chunked)
            for j in range(w):
                assert torch.equal(back[j], x[j]), f"{name}: mode 1 rank {j} (chunked={chunked})"


def pin_identity_w1(run):
    for shape in [(1, 3, 5, 7), (2, 4, 3, 16), (3, 1, 1, 1)]:
        x = normal_slabs(shape, 1, "bf16", seed0=7)
        for mode in (0, 1):
            y = run(x, mode, False)
            assert torch.equal(y[0].view(torch.int16), x[0].view(torch.int16)), f"w=1 mode {mode} {shape}"


ROUND_TRIP_CASES = [
    # (w, B, S_local, H, D)
    (2, 1, 4, 4, 8),
    (3, 2, 5, 6, 4),
    (4, 2, 3, 8, 2),
    (5, 1, 2, 10, 3),
    (8, 2, 3, 16, 2),
]


def pin_round_trip(run):
    for (w, B, S, H, D) in ROUND_TRIP_CASES:
        x = normal_slabs((B, S, H, D), w, "bf16", seed0=11)
        y = run(x, 0, False)
        for r in range(w):
            assert tuple(y[r].shape) == (B, S * w, H // w, D)
        z = run(y, 1, False)
        for j in range(w):
            assert torch.equal(z[j].view(torch.int16), x[j].view(torch.int16)), f"mode1(mode0) {w,B,S,H,D}"
        # the other order: start from the gathered layout
        y2 = normal_slabs((B, S * w, H // w, D), w, "bf16", seed0=12)
        x2 = run(y2, 1, False)
        for j in range(w):
            assert tuple(x2[j].shape) == (B, S, H, D)
        y3 = run(x2, 0, False)
        for r in range(w):
            assert torch.equal(y3[r].view(torch.int16), y2[r].view(torch.int16)), f"mode0(mode1) {w,B,S,H,D}"


def pin_transpose_special_case(run):
    """S_local = 1, B = 1, H = w: stacking the slabs as a w x w grid of D-vectors,
    mode 0 is the block transpose of that grid (rank r's row j is rank j's head r)."""
    for w, D in [(2, 1), (3, 1), (4, 3), (7, 2)]:
        x = unique_slabs((1, 1, w, D), w, 4)
        grid = torch.stack([t.reshape(w, D) for t in x])          # [j, h, d]
        y = run(x, 0, False)
        got = torch.stack([t.reshape(w, D) for t in y])           # [r, j, d]
        assert torch.equal(got, grid.transpose(0, 1)), f"transpose w={w} D={D}"


def permute_formulation(xs, mode, w):
    """Independent library formulation of both maps via a 6D permute (CPU torch)."""
    if mode == 0:
        B, S, H, D = xs[0].shape
        X = torch.stack(xs).view(w, B, S, w, H // w, D)              # [j, b, s, r, h', d]
        Y = X.permute(3, 1, 0, 2, 4, 5).reshape(w, B, S * w, H // w, D)   # [r, b, (j s), h', d]
        return list(Y.unbind(0))
    B, SG, Hl, D = xs[0].shape
    S = SG // w
    Y = torch.stack(xs).view(w, B, w, S, Hl, D)                      # [r, b, j, s, h', d]
    X = Y.permute(2, 1, 3, 0, 4, 5).reshape(w, B, S, w * Hl, D)       # [j, b, s, (r h'), d]
    return list(X.unbind(0))


PERMUTE_CASES = [
    (2, 1, 64, 4, 64),
    (3, 2, 7, 9, 5),
    (4, 3, 5, 8, 16),
    (8, 2, 9, 40, 4),
    (6, 1, 1, 6, 1),
]


def pin_permute_unique_ids(run):
    for (w, B, S, H, D) in PERMUTE_CASES:
        for E in (4, 8):
            x = unique_slabs((B, S, H, D), w, E)
            y = run(x, 0, False)
            want = permute_formulation(x, 0, w)
            for r in range(w):
                assert torch.equal(y[r], want[r]), f"mode 0 vs permute {w,B,S,H,D} E={E}"
            # every id appears exactly once across all outputs: a bijection
            allv = torch.cat([t.reshape(-1) for t in y]).sort().values
            ref = torch.cat([t.reshape(-1) for t in x]).sort().values
            assert torch.equal(allv, ref)
            yg = unique_slabs((B, S * w, H // w, D), w, E)
            z = run(yg, 1, False)
            want1 = permute_formulation(yg, 1, w)
            for j in range(w):
                assert torch.equal(z[j], want1[j]), f"mode 1 vs permute {w,B,S,H,D} E={E}"


def pin_rank_tagged_bf16_width(run):
    """2-byte elements: high byte = source rank, checked against the permute form."""
    for (w, B, S, H, D) in [(4, 2, 6, 8, 12), (8, 1, 5, 16, 8)]:
        x = rank_tagged_slabs((B, S, H, D), w)
        y = run(x, 0, False)
        want = permute_formulation(x, 0, w)
        for r in range(w):
            assert torch.equal(y[r], want[r])
        z = run(y, 1, False)
        for j in range(w):
            assert torch.equal(z[j], x[j])


def pin_chunked_equals_unchunked(run):
    for (w, B, S, H, D) in [(2, 3, 4, 4, 8), (4, 4, 3, 8, 2), (3, 2, 5, 3, 6)]:
        x = unique_slabs((B, S, H, D), w, 4)
        for mode, xs in ((0, x), (1, unique_slabs((B, S * w, H // w, D), w, 4))):
            a = run(xs, mode, False)
            b = run(xs, mode, True)
            for k in range(w):
                assert torch.equal(a[k], b[k]), f"chunked != unchunked mode {mode} {w,B,S,H,D}"
            want = permute_formulation(xs, mode, w)
            for k in range(w):
                assert torch.equal(b[k], want[k]), f"chunked vs permute mode {mode} {w,B,S,H,D}"


def pin_bits_not_values(run):
    """NaN payloads and signed zeros pass through untouched (a bit copy)."""
    w, B, S, H, D = 2, 1, 2, 2, 4
    x = normal_slabs((B, S, H, D), w, "fp32", seed0=3)
    bits = [t.view(torch.int32).clone() for t in x]
    bits[0].view(-1)[0] = 0x7FC01234      # quiet NaN with a payload
    bits[0].view(-1)[5] = 0x7F800001      # signalling NaN
    bits[1].view(-1)[3] = int(-2**31)     # -0.0
    xs = [b.view(torch.float32) for b in bits]
    y = run(xs, 0, False)
    want = permute_formulation([b for b in bits], 0, w)
    for r in range(w):
        assert torch.equal(y[r].view(torch.int32), want[r]), "bit pattern changed"


def _pitched_run_default(run):
    """The pitched oracle bound to the same library build as `run` (see oracle_pins users)."""
    return getattr(run, "pitched", None)


def pin_pitched_packed_qkv(run):
    """q, k, v read in place from a packed [B, S, 3, H, D] buffer (row pitch 3*H*D) give
    the same result as the dense oracle on torch's own q/k/v slices."""
    pitched = _pitched_run_default(run)
    if pitched is None:
        return
    for (w, B, S, H, D) in [(2, 1, 3, 4, 2), (4, 2, 5, 8, 3), (3, 2, 4, 6, 2)]:
        packed = unique_slabs((B, S, 3, H, D), w, 4)
        for c in range(3):
            dense_in = [t[:, :, c].contiguous() for t in packed]
            want = run(dense_in, 0, False)
            got = pitched([t.reshape(-1) for t in packed], 0, w, B, S, H, D, 3 * H * D,
                          offset=c * H * D)
            for r in range(w):
                assert torch.equal(got[r].reshape(want[r].shape), want[r]), f"pitched mode 0 c={c}"


def pin_pitched_mode1_writes_only_its_slot(run):
    """Mode 1 into slot c of packed [B, S, 3, H, D] outputs: that slot equals the dense
    oracle's output, the other two slots keep their poison bytes."""
    pitched = _pitched_run_default(run)
    if pitched is None:
        return
    w, B, S, H, D = 4, 2, 3, 8, 2
    ys = unique_slabs((B, S * w, H // w, D), w, 4)
    want = run(ys, 1, False)
    for c in range(3):
        outs = [torch.full((B * S * 3 * H * D,), -1, dtype=torch.int32) for _ in range(w)]
        pitched([t.reshape(-1) for t in ys], 1, w, B, S, H, D, 3 * H * D, offset=c * H * D,
                out_bufs=outs)
        for j in range(w):
            v = outs[j].view(B, S, 3, H, D)
            assert torch.equal(v[:, :, c], want[j]), f"pitched mode 1 slot {c}"
            for other in range(3):
                if other != c:
                    assert bool((v[:, :, other] == -1).all()), "a gap element was written"


def pin_pitched_hand_table(run):
    """w=2, B=1, S_local=2, H=2, D=1, row pitch 3: rows are (head 0, head 1, gap).
    Derived by hand as in hand_w2_B1_S2_H2_D1.txt: rank r keeps head r."""
    pitched = _pitched_run_default(run)
    if pitched is None:
        return
    # x0 = [a0 a1 g | a2 a3 g], x1 = [b0 b1 g | b2 b3 g], g = gap
    a0, a1, a2, a3, b0, b1, b2, b3, g = 1, 2, 3, 4, 5, 6, 7, 8, 99
    x = [torch.tensor([a0, a1, g, a2, a3, g], dtype=torch.int32),
         torch.tensor([b0, b1, g, b2, b3, g], dtype=torch.int32)]
    out = pitched(x, 0, 2, 1, 2, 2, 1, 3)
    assert out[0].tolist() == [a0, a2, b0, b2]
    assert out[1].tolist() == [a1, a3, b1, b3]
    back = pitched(out, 1, 2, 1, 2, 2, 1, 3,
                   out_bufs=[torch.full((6,), 0, dtype=torch.int32) for _ in range(2)])
    assert back[0].tolist() == [a0, a1, 0, a2, a3, 0]
    assert back[1].tolist() == [b0, b1, 0, b2, b3, 0]


ALL_PINS = [
    pin_hand_tables,
    pin_identity_w1,
    pin_round_trip,
    pin_transpose_special_case,
    pin_permute_unique_ids,
    pin_rank_tagged_bf16_width,
    pin_chunked_equals_unchunked,
    pin_bits_not_values,
    pin_pitched_packed_qkv,
    pin_pitched_mode1_writes_only_its_slot,
    pin_pitched_hand_table,
]
