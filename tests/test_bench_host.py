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


def test_clock_sampler_keeps_only_samples_inside_windows(monkeypatch):
    # the sampler process is replaced by injected lines; end() takes one
    # synchronous query (faked here) so every window has a sample
    import subprocess
    import types

    import bench

    def no_popen(*a, **k):
        raise OSError("no nvidia-smi here")

    monkeypatch.setattr(subprocess, "Popen", no_popen)
    line = "0, {sm}, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, {cap}\n"
    monkeypatch.setattr(subprocess, "run", lambda *a, **k: types.SimpleNamespace(
        stdout=line.format(sm=1900, cap="Active")))
    c = bench.ClockSampler(0, enabled=True)
    c.samples = [(1.0, line.format(sm=500, cap="Not Active")),    # before the window: idle, dropped
                 (2.5, line.format(sm=1965, cap="Not Active"))]
    monkeypatch.setattr(bench.time, "time", lambda: 2.0)
    c.begin()
    monkeypatch.setattr(bench.time, "time", lambda: 3.0)
    c.end()
    c.samples.append((9.0, line.format(sm=300, cap="Not Active")))  # after: dropped
    rec = c.stop()
    assert rec["samples"] == 2
    assert rec["sm_mhz"] == (1965 + 1900) / 2 and rec["sm_max_mhz"] == 1965
    assert rec["reasons"] == ["sw_power_cap"]
    assert bench.ClockSampler(0, enabled=False).stop() is None
