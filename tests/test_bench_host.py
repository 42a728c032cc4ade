"""bench.py's host-side layout of a record's buffers, on CPU tensors.

A record's activations and outputs are 256-byte aligned views of one buffer each (one copy in and
one copy out per end-to-end step); the end-to-end steps that overlap their copies rebuild the same
views over a second pair of buffers.  These tests check the offsets, the views' places in the
buffers, and that layers of a group read their first member's activations in either buffer set.
"""
import numpy as np
import torch

import bench


def test_packed_offsets_are_aligned_and_disjoint():
    sizes = [10240, 34816, 1, 255, 256, 257, 0]
    offs, total = bench.packed_offsets(sizes)
    assert offs[0] == 0 and all(o % 256 == 0 for o in offs)
    for (o, n), o2 in zip(zip(offs, sizes), offs[1:] + [total]):
        assert o + n <= o2
    assert total % 256 == 0 and total >= 256
    assert bench.packed_offsets([]) == ([], 256)


def _layers():
    # a BenQ layer with its own x, a multi-part BenQ layer, and an MDBF group of two layers whose
    # second member reads the first one's x
    xs = [(1, 1024), (1, 512), (1, 768)]
    xoff, xtot = bench.packed_offsets([a * b * 2 for a, b in xs])
    ys = [((1, 256), torch.float32), ((1, 96), torch.bfloat16), ((1, 64), torch.float32), ((1, 64), torch.float32)]
    yoff, ytot = bench.packed_offsets([a * b * (4 if d == torch.float32 else 2) for (a, b), d in ys])
    xbuf, ybuf = torch.zeros(xtot, dtype=torch.uint8), torch.zeros(ytot, dtype=torch.uint8)
    L = [{} for _ in range(4)]
    for i, ((shape, d), o) in enumerate(zip(ys, yoff)):
        nb = shape[0] * shape[1] * (4 if d == torch.float32 else 2)
        L[i]["y"] = ybuf[o:o + nb].view(d).view(shape)
        L[i]["_yo"] = (o, nb)
    for i, (shape, o) in enumerate(zip(xs, xoff)):
        nb = shape[0] * shape[1] * 2
        L[i]["x"] = xbuf[o:o + nb].view(torch.bfloat16).view(shape)
        L[i]["_xo"] = (o, nb)
    L[1]["_ys_offs"] = np.array([0, 32, 96])
    L[1]["ys"] = [L[1]["y"][:, 0:32], L[1]["y"][:, 32:96]]
    L[2]["group_members"] = [L[2], L[3]]
    L[3]["group_skip"] = True
    L[3]["x"] = L[2]["x"]
    inp = bench.Inputs.__new__(bench.Inputs)
    inp.layers = L
    return inp, xbuf, ybuf


def test_views_over_a_second_buffer_pair_keep_offsets_shapes_and_group_inputs():
    inp, xbuf, ybuf = _layers()
    x2, y2 = torch.zeros_like(xbuf), torch.zeros_like(ybuf)
    for xb, yb in ((xbuf, ybuf), (x2, y2)):
        vs = inp.views(torch, xb, yb)
        for L, v in zip(inp.layers, vs):
            assert v["y"].shape == L["y"].shape and v["y"].dtype == L["y"].dtype
            assert v["y"].untyped_storage().data_ptr() == yb.untyped_storage().data_ptr()
            assert v["y"].data_ptr() - yb.data_ptr() == L["_yo"][0]
            assert v["x"].shape == L["x"].shape and v["x"].dtype == torch.bfloat16
            assert v["x"].data_ptr() - xb.data_ptr() == L["x"].data_ptr() - xbuf.data_ptr()
        # the group's second member reads the first member's x of the same buffer set
        assert vs[3]["x"].data_ptr() == vs[2]["x"].data_ptr()
        # the multi-part outputs are column slices of the layer's own output view
        assert [t.shape for t in vs[1]["ys"]] == [(1, 32), (1, 64)]
        assert vs[1]["ys"][1].data_ptr() == vs[1]["y"].data_ptr() + 32 * 2
        # writing through a view lands in its own buffer only
        vs[0]["y"].fill_(1.0)
        assert yb[:1024].view(torch.float32).eq(1.0).all()
    assert not torch.equal(ybuf, torch.zeros_like(ybuf)) and not torch.equal(y2, torch.zeros_like(y2))


def test_use_swaps_a_records_views_and_back():
    inp, xbuf, ybuf = _layers()
    x2, y2 = torch.zeros_like(xbuf), torch.zeros_like(ybuf)
    first, second = inp.views(torch, xbuf, ybuf), inp.views(torch, x2, y2)
    inp.use(second)
    assert all(L["y"].data_ptr() - y2.data_ptr() == L["_yo"][0] for L in inp.layers)
    assert inp.layers[3]["x"].data_ptr() == inp.layers[2]["x"].data_ptr()
    inp.use(first)
    assert all(L["y"].data_ptr() - ybuf.data_ptr() == L["_yo"][0] for L in inp.layers)
