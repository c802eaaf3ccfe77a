"""Host-side pieces of bench.py's end-to-end measurement, on CPU: the packed
input buffer that carries one decode step's inputs across in a single copy
must hold every tensor at its own aligned offset, unchanged, and the views
the loop writes the block tables through must alias that buffer."""
import numpy as np
import torch

import bench


def _step_inputs(B=6, H=4, Hkv=2, D=128, W=9):
    g = torch.Generator().manual_seed(11)
    return (torch.randn(B, H, D, generator=g).to(torch.bfloat16),
            torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16),
            torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16),
            torch.arange(B, dtype=torch.int64) * 16 + 3,
            torch.randint(0, 1000, (B, W), generator=g, dtype=torch.int32),
            torch.randint(0, 100, (B,), generator=g, dtype=torch.int32))


def test_packed_buffers_layout_and_views(monkeypatch):
    # no GPU here: pinning is a no-op and the "device" buffer is a CPU tensor
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    ts = _step_inputs()
    host, devb, hv, dv = bench.packed_buffers(ts, "cpu")
    sizes = [t.numel() * t.element_size() for t in ts]
    assert host.numel() == devb.numel() == sum((n + 255) // 256 * 256 for n in sizes)
    assert host.dtype == devb.dtype == torch.uint8
    offs = [h.data_ptr() - host.data_ptr() for h in hv]
    assert all(o % 256 == 0 for o in offs)
    # disjoint, in order
    for (o, n), o2 in zip(zip(offs, sizes), offs[1:]):
        assert o + n <= o2
    for t, h, d in zip(ts, hv, dv):
        assert h.shape == d.shape == t.shape and h.dtype == d.dtype == t.dtype
        assert torch.equal(h, t)
    # tables written through the numpy views land in the buffer that is copied
    bt_np, sl_np = hv[4].numpy(), hv[5].numpy()
    bt_np[:] = 7
    sl_np[:] = 5
    devb.copy_(host)
    assert torch.equal(dv[4], torch.full_like(ts[4], 7)) and torch.equal(dv[5], torch.full_like(ts[5], 5))
    for t, d in zip(ts[:4], dv[:4]):
        assert torch.equal(d, t)


def test_packed_buffers_pad_odd_sizes(monkeypatch):
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    ts = (torch.ones(3, dtype=torch.int32), torch.arange(5, dtype=torch.int64), torch.zeros(7, dtype=torch.bfloat16))
    host, _, hv, _ = bench.packed_buffers(ts, "cpu")
    assert host.numel() == 3 * 256
    assert [h.data_ptr() - host.data_ptr() for h in hv] == [0, 256, 512]
    assert np.array_equal(hv[1].numpy(), np.arange(5))
