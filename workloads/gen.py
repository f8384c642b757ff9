"""Seeded synthetic tensors shared by the oracle side and the device side.

This module holds no arithmetic of the sharded-linear method.  It only turns
(seed, tensor id, element index) into a number, so the host (oracle input) and
the device (kernel input) can materialise bit-identical tensors without copying
one from the other.

Generator
---------
* Counter-based: element ``i`` of tensor ``t`` is ``splitmix64(key + (i+1)*G)``
  with ``key = seed XOR (t * G)`` and ``G = 0x9E3779B97F4A7C15`` (Steele, Lea,
  Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014; the
  finaliser constants are the published SplitMix64 ones).
* The 64-bit output is cut into four 16-bit uniforms ``u0..u3`` and
  ``s = u0+u1+u2+u3 - 131070`` (an Irwin-Hall sum with its mean removed).  The sum
  of four uniforms is a bounded stand-in for a normal draw (support is +-3.46
  sigma); it needs only integer work, so CPU and GPU give the same bits.
* ``value = fp32(s) * fp32(sigma / std(s)) (+ fp32(mu))``, each an IEEE single
  rounding, then rounded to the storage dtype (bf16 round-to-nearest-even or
  kept fp32).

The same torch integer ops run on CPU or CUDA, so ``normal(..., device='cuda')``
and ``normal(..., device='cpu')`` agree bit for bit.
"""
from __future__ import annotations

import math

import torch

_GAMMA = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1

# Irwin-Hall sum of four U{0..65535}: mean 131070, variance 4*(65536^2-1)/12.
_IH_MEAN = 131070
_IH_STD = math.sqrt(4.0 * (65536.0 * 65536.0 - 1.0) / 12.0)

# Tensor ids of the workloads.  A layer l of a stack adds 16*l.
TID_X, TID_W1, TID_W2, TID_BIAS, TID_SCALE = 0, 1, 2, 3, 4


def _s64(v: int) -> int:
    """Reinterpret an unsigned 64-bit integer as signed (torch has no uint64 math)."""
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 lanes (torch's >> is arithmetic)."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _splitmix64(idx: torch.Tensor, key: int) -> torch.Tensor:
    z = idx.add(1).mul_(_s64(_GAMMA)).add_(_s64(key))
    z = (z ^ _lsr(z, 30)).mul_(_s64(_MIX1))
    z = (z ^ _lsr(z, 27)).mul_(_s64(_MIX2))
    return z ^ _lsr(z, 31)


def _irwin_hall(z: torch.Tensor) -> torch.Tensor:
    s = (z & 0xFFFF) + (_lsr(z, 16) & 0xFFFF) + (_lsr(z, 32) & 0xFFFF) + _lsr(z, 48)
    return s - _IH_MEAN


def tensor_key(seed: int, tensor_id: int) -> int:
    return (seed ^ ((tensor_id * _GAMMA) & _MASK64)) & _MASK64


def normal(shape, sigma: float, *, tensor_id: int, seed: int = 0, mu: float = 0.0,
           dtype: torch.dtype = torch.bfloat16, device="cpu", offset: int = 0,
           chunk: int = 1 << 26) -> torch.Tensor:
    """Approximately N(mu, sigma) tensor, elements ``offset ..`` of stream ``tensor_id``.

    ``offset`` lets a caller materialise any contiguous slice (for example a few
    rows of a large weight) without generating the rest.
    """
    shape = tuple(int(d) for d in shape)
    n = 1
    for d in shape:
        n *= d
    out = torch.empty(n, dtype=dtype, device=device)
    key = tensor_key(seed, tensor_id)
    c = torch.tensor(sigma / _IH_STD, dtype=torch.float32, device=device)
    m = torch.tensor(mu, dtype=torch.float32, device=device)
    for lo in range(0, n, chunk):
        hi = min(n, lo + chunk)
        idx = torch.arange(offset + lo, offset + hi, dtype=torch.int64, device=device)
        v = _irwin_hall(_splitmix64(idx, key)).to(torch.float32).mul_(c)
        if mu != 0.0:
            v.add_(m)
        out[lo:hi] = v.to(dtype)
    return out.view(shape)


def rows(full_shape, row_ids, sigma: float, *, tensor_id: int, seed: int = 0,
         mu: float = 0.0, dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """Selected rows of a row-major 2-D tensor, generated on the host."""
    r, c = int(full_shape[0]), int(full_shape[1])
    parts = []
    for i in row_ids:
        i = int(i)
        assert 0 <= i < r
        parts.append(normal((c,), sigma, tensor_id=tensor_id, seed=seed, mu=mu,
                            dtype=dtype, offset=i * c))
    return torch.stack(parts) if parts else torch.empty((0, c), dtype=dtype)


def splitmix64_reference(key: int, i: int) -> int:
    """Scalar SplitMix64 in Python integers: the published algorithm, for tests."""
    z = (key + (i + 1) * _GAMMA) & _MASK64
    z = ((z ^ (z >> 30)) * _MIX1) & _MASK64
    z = ((z ^ (z >> 27)) * _MIX2) & _MASK64
    return z ^ (z >> 31)
