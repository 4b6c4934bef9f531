"""The Python binding's argument marshalling (CPU only, no CUDA context).

``marshal_slabs`` turns a call's tensors into the C ABI's arguments and
rejects what the op cannot take; ``DescBuffer`` is the descriptor a context
refills on every call. Both run on every call, so these tests pin what they
hand to the library: dimensions in the mode-0 frame (FastVideo API docs,
device_communicators/ulysses_a2a, ``run_armed``: mode 1 takes
[B, S_local*w, H/w, D] slabs), pointers in rank order, and the row pitch of a
view into a packed q/k/v projection.
"""

import ctypes

import pytest
import torch

from sequence_all_re_b200 import _lib, marshal_slabs


def _slabs(shape, w, dtype=torch.bfloat16):
    return [torch.zeros(shape, dtype=dtype) for _ in range(w)]


@pytest.mark.parametrize("mode", [0, 1])
def test_dimensions_pointers_and_allocated_outputs(mode):
    w, B, S, H, D = 4, 2, 5, 8, 16
    in_shape = (B, S, H, D) if mode == 0 else (B, S * w, H // w, D)
    out_shape = (B, S * w, H // w, D) if mode == 0 else (B, S, H, D)
    xs = _slabs(in_shape, w)
    got_w, dims, out, ip, op, pitch = marshal_slabs(xs, mode, None, "cpu", 2)
    assert (got_w, dims, pitch) == (w, (B, S, H, D), 0)
    assert [tuple(o.shape) for o in out] == [out_shape] * w
    assert all(o.dtype == torch.bfloat16 for o in out)
    assert ip == [t.data_ptr() for t in xs]
    assert op == [o.data_ptr() for o in out]
    # given outputs are used as they are
    mine = _slabs(out_shape, w)
    _, _, out2, _, op2, _ = marshal_slabs(xs, mode, mine, "cpu", 2)
    assert out2 is mine and op2 == [o.data_ptr() for o in mine]


@pytest.mark.parametrize("mode", [0, 1])
def test_row_pitch_of_a_packed_projection_view(mode):
    # q of a packed [B, S, 3, H, D] tensor: strides (S*3*H*D, 3*H*D, D, 1)
    w, B, S, H, D = 2, 3, 4, 4, 8
    packed = [torch.zeros(B, S, 3, H, D, dtype=torch.bfloat16) for _ in range(w)]
    views = [p[:, :, 0] for p in packed]
    dense = _slabs((B, S * w, H // w, D), w)
    xs, out = (views, dense) if mode == 0 else (dense, views)
    _, dims, _, _, _, pitch = marshal_slabs(xs, mode, out, "cpu", 2, allow_pitch=True)
    assert dims == (B, S, H, D) and pitch == 3 * H * D
    with pytest.raises(ValueError, match="contiguous"):
        marshal_slabs(xs, mode, out, "cpu", 2, allow_pitch=False)
    # the [B, S_local*w, H/w, D] side takes no pitch: a transposed view of it is refused
    strided_dense = [torch.zeros(B, H // w, S * w, D, dtype=torch.bfloat16).transpose(1, 2)
                     for _ in range(w)]
    xs2, out2 = (views, strided_dense) if mode == 0 else (strided_dense, views)
    with pytest.raises(ValueError, match=r"\[B, S_local\*w, H/w, D\] slabs must be contiguous"):
        marshal_slabs(xs2, mode, out2, "cpu", 2, allow_pitch=True)


def test_pitch_must_be_shared_and_well_formed():
    w, B, S, H, D = 2, 2, 4, 4, 8
    a = torch.zeros(B, S, 3, H, D, dtype=torch.bfloat16)[:, :, 0]
    b = torch.zeros(B, S, 2, H, D, dtype=torch.bfloat16)[:, :, 1]
    out = _slabs((B, S * w, H // w, D), w)
    with pytest.raises(ValueError, match="shared by all slabs"):
        marshal_slabs([a, b], 0, out, "cpu", 2, allow_pitch=True)
    # heads not adjacent (a transposed view) is not a row-pitched slab
    t = torch.zeros(B, S, D, H, dtype=torch.bfloat16).transpose(2, 3)
    with pytest.raises(ValueError, match="strides"):
        marshal_slabs([t, t.clone()], 0, out, "cpu", 2, allow_pitch=True)


@pytest.mark.parametrize("case, match", [
    ("no slabs", "at least one"),
    ("mode 2", "mode must be 0 or 1"),
    ("3D", "4D"),
    ("elem bytes", "4-byte elements"),
    ("shape", "share shape and dtype"),
    ("dtype", "share shape and dtype"),
    ("device", "must be on cuda"),
    ("out count", "one output per rank"),
    ("out shape", "outputs must be"),
    ("out dtype", "outputs must be"),
])
def test_rejections(case, match):
    w, B, S, H, D = 2, 1, 4, 4, 8
    xs = _slabs((B, S, H, D), w)
    out = _slabs((B, S * w, H // w, D), w)
    kw = dict(xs=xs, mode=0, out=out, device_type="cpu", elem_bytes=2)
    if case == "no slabs":
        kw["xs"] = []
    elif case == "mode 2":
        kw["mode"] = 2
    elif case == "3D":
        kw["xs"] = _slabs((S, H, D), w)
    elif case == "elem bytes":
        kw["elem_bytes"] = 4
    elif case == "shape":
        kw["xs"] = [xs[0], torch.zeros(B, S + 1, H, D, dtype=torch.bfloat16)]
    elif case == "dtype":
        kw["xs"] = [xs[0], torch.zeros(B, S, H, D, dtype=torch.float16)]
    elif case == "device":
        kw["device_type"] = "cuda"
    elif case == "out count":
        kw["out"] = out[:1]
    elif case == "out shape":
        kw["out"] = [out[0], torch.zeros(B, S * w, H, D, dtype=torch.bfloat16)]
    elif case == "out dtype":
        kw["out"] = [out[0], out[1].half()]
    with pytest.raises(ValueError, match=match):
        marshal_slabs(**kw)


def _read_desc(ref_holder):
    d = ref_holder.desc
    return (d.B, d.S_local, d.H, d.D, d.w, d.mode, d.chunked, d.ntensors, d.row_pitch)


def test_desc_buffer_refill_and_growth():
    buf = _lib.DescBuffer(capacity=2)
    ref = buf.fill([0x1000, 0x2000], [0x3000, 0], 2, 5, 8, 16, 2, 1, 2, 384, 0)
    assert ref is buf.ref
    assert _read_desc(buf) == (2, 5, 8, 16, 2, 1, 2, 0, 384)
    assert [buf.desc.in_slabs[i] for i in range(2)] == [0x1000, 0x2000]
    assert [buf.desc.out_slabs[i] for i in range(2)] == [0x3000, None]
    # more slabs than the arrays hold: they grow and the descriptor follows
    ins = [0x10000 * (k + 1) for k in range(6)]
    outs = [0x20000 * (k + 1) for k in range(6)]
    buf.fill(ins, outs, 1, 64, 24, 128, 3, 0, 0, 0, 2)
    assert _read_desc(buf) == (1, 64, 24, 128, 3, 0, 0, 2, 0)
    assert [buf.desc.in_slabs[i] for i in range(6)] == ins
    assert [buf.desc.out_slabs[i] for i in range(6)] == outs
    assert ctypes.addressof(buf.ins) == ctypes.cast(buf.desc.in_slabs, ctypes.c_void_p).value


def test_desc_buffer_matches_a_fresh_descriptor():
    args = ([0xA0, 0xB0, 0xC0], [0xD0, 0xE0, 0xF0], 4, 7, 9, 64, 3, 1, 1, 0, 0)
    fresh, keep = _lib.make_desc(*args)
    buf = _lib.DescBuffer()
    buf.fill(*args)
    for name, _ in _lib.DescT._fields_:
        if name in ("in_slabs", "out_slabs"):
            assert [getattr(fresh, name)[i] for i in range(3)] == \
                   [getattr(buf.desc, name)[i] for i in range(3)]
        else:
            assert getattr(fresh, name) == getattr(buf.desc, name), name
