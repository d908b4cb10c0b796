"""Host-side pieces of bench.py that need no GPU: the packed step inputs of
the end-to-end measurement (one pinned buffer, one copy) must hold every
input unchanged, each view at a 256-byte aligned offset of its buffer (the
library's 16-byte and 4-byte alignment checks), in the input's dtype and
shape."""
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def test_packed_inputs_views(monkeypatch):
    import bench
    # pinned memory needs a CUDA driver; on the CPU the host twin is plain memory
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    g = torch.Generator().manual_seed(3)
    inputs = {
        "q": torch.randn((5, 16, 128), generator=g).to(torch.bfloat16),
        "bt": torch.randint(0, 1000, (5, 37), generator=g, dtype=torch.int32),
        "cl": torch.randint(1, 500, (5,), generator=g, dtype=torch.int32),
        "kn": torch.randn((5, 8, 128), generator=g).to(torch.bfloat16),
        "sm": torch.randint(-1, 9000, (5,), generator=g, dtype=torch.int32),
    }
    p = bench.Packed(inputs, torch.device("cpu"))
    base = p.dev.data_ptr()
    end = 0
    for n, t in inputs.items():
        v = p.views[n]
        assert v.dtype == t.dtype and v.shape == t.shape and v.is_contiguous()
        assert torch.equal(v, t), n
        assert (v.data_ptr() - base) % 256 == 0, n
        assert v.data_ptr() >= base + end, "views overlap"
        end = v.data_ptr() - base + t.numel() * t.element_size()
    assert end == p.nbytes
    # a refreshed host buffer reaches every view with one copy
    p.host.zero_()
    p.h2d()
    assert all(int(v.abs().sum()) == 0 for v in (p.views["bt"], p.views["cl"]))
