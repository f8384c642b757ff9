"""The seeded generator: its integer stream is SplitMix64 as published, and any
slice can be regenerated on its own (host side; the device side is compared
bit for bit in the GPU tests)."""
import torch

from workloads import gen


def test_splitmix_stream_matches_scalar_definition():
    key = gen.tensor_key(0, 7)
    idx = torch.arange(0, 4096, dtype=torch.int64)
    z = gen._splitmix64(idx, key)
    for i in [0, 1, 2, 1000, 4095]:
        ref = gen.splitmix64_reference(key, i)
        assert (int(z[i]) & ((1 << 64) - 1)) == ref


def test_values_from_scalar_definition():
    key = gen.tensor_key(0, gen.TID_W1)
    v = gen.normal((64,), 0.02, tensor_id=gen.TID_W1, dtype=torch.float32)
    c = torch.tensor(0.02 / gen._IH_STD, dtype=torch.float32)
    for i in range(64):
        z = gen.splitmix64_reference(key, i)
        s = sum((z >> (16 * q)) & 0xFFFF for q in range(4)) - 131070
        assert v[i].item() == (torch.tensor(float(s), dtype=torch.float32) * c).item()


def test_slices_regenerate_exactly():
    full = gen.normal((12, 40), 1.0, tensor_id=3, chunk=97)
    part = gen.rows((12, 40), [0, 5, 11], 1.0, tensor_id=3)
    assert torch.equal(part, full[[0, 5, 11]])
    assert torch.equal(gen.normal((5, 40), 1.0, tensor_id=3, offset=40 * 7), full[7:12])


def test_distribution_moments():
    v = gen.normal((1 << 20,), 0.5, tensor_id=1, mu=1.0, dtype=torch.float32)
    assert abs(v.mean().item() - 1.0) < 2e-3
    assert abs(v.std().item() - 0.5) < 2e-3
    assert (v - 1.0).abs().max().item() <= 0.5 * 3.47
