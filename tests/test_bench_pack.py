"""The end-to-end measurement's packing of a step's tensors into one buffer (one copy each
way per step): 256-byte aligned pieces, views with the tensors' dtypes and shapes, and the
bytes of every tensor through a packed buffer unchanged."""

import pytest

torch = pytest.importorskip("torch")

import bench  # noqa: E402


def test_pack_layout_and_views_round_trip():
    g = torch.Generator().manual_seed(3)
    ts = [torch.randn((4, 2, 17, 8, 128), generator=g).to(torch.bfloat16),
          torch.randn((4, 2, 17, 8, 128), generator=g).to(torch.bfloat16),
          torch.randn((4, 2, 17, 4096), generator=g).to(torch.bfloat16),
          torch.randn((4, 2, 16, 4096), generator=g).to(torch.bfloat16),
          torch.randint(0, 1000, (4, 16), generator=g, dtype=torch.int32),
          torch.randint(0, 1000, (4, 17), generator=g, dtype=torch.int32),
          torch.randn((3,), generator=g)]
    offs, size = bench.pack_layout(ts)
    assert all(o % 256 == 0 for o in offs) and size % 256 == 0
    ends = [o + t.numel() * t.element_size() for o, t in zip(offs, ts)]
    assert all(e <= o2 for e, o2 in zip(ends, offs[1:])) and ends[-1] <= size < ends[-1] + 256
    buf = torch.zeros(size, dtype=torch.uint8)
    vs = bench.pack_views(buf, ts, offs)
    for v, t in zip(vs, ts):
        assert v.dtype == t.dtype and v.shape == t.shape
        v.copy_(t)
    copy = buf.clone()  # what one copy of the packed block carries
    for v, t in zip(bench.pack_views(copy, ts, offs), ts):
        assert torch.equal(v, t)
