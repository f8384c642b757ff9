"""Shared helpers of the GPU parity tests: tolerances, conversions, comparisons."""
import numpy as np
import torch

import oracle as O

# Tolerances stated by the target: relative Frobenius error of floats,
# bf16-in/fp32-accumulate 5e-3, fp32 1e-5; ids bit-exact except where the
# oracle's top-2 logit gap is below 1e-3 (then any id within 1e-3 of the max).
TOL_BF16 = 5e-3
TOL_FP32 = 1e-5
TIE_GAP = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a (bf16 / fp32) tensor, on the host."""
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def rel(got, ref) -> float:
    return O.rel_frobenius(got if isinstance(got, np.ndarray) else f64(got), ref)


def check_ids(got_ids, res: O.LMHeadResult, rows=None):
    """Argmax ids: exact, or within TIE_GAP of the max where the oracle's gap is small."""
    got_ids = np.asarray(got_ids)
    rows = range(len(got_ids)) if rows is None else rows
    for i, b in enumerate(rows):
        g = int(got_ids[i])
        if res.gap[i] >= TIE_GAP:
            assert g == int(res.ids[i]), (b, g, int(res.ids[i]), res.gap[i])
        else:
            assert res.logits[i, g] >= res.logits[i].max() - TIE_GAP, (b, g)


def check_shard_ids(got_idx, got_max, res: O.LMHeadResult, tol=TOL_BF16):
    got_idx = np.asarray(got_idx)
    tp, B = res.shard_idx.shape
    for r in range(tp):
        for b in range(B):
            if res.shard_idx[r, b] < 0:
                assert got_idx[r, b] == -1
                assert got_max[r, b] == -np.inf
                continue
            g = int(got_idx[r, b])
            if res.shard_gap[r, b] >= TIE_GAP:
                assert g == res.shard_idx[r, b], (r, b, g, res.shard_idx[r, b])
            else:
                assert res.logits[b, g] >= res.shard_max[r, b] - TIE_GAP
            assert abs(got_max[r, b] - res.shard_max[r, b]) <= tol * max(1.0, abs(res.shard_max[r, b]))
    return True
