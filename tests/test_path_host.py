"""Host-side layout helpers of path.py for the TP linears split over GPUs: the
token slices of the sequence-parallel layout (nanotron "MLP Module": each rank
keeps ``[batch, seq // tp, hidden]``), checked against the oracle's
``seq_scatter`` and against each other.  CPU only."""
import numpy as np
import pytest
import torch

import oracle as O
from tensor_transformer_linear_b200 import path


@pytest.mark.parametrize("batch,seq,tp,N", [(2, 8, 2, 3), (3, 12, 4, 5), (1, 16, 8, 1)])
def test_token_slices_match_the_oracle_scatter(batch, seq, tp, N):
    x = np.random.default_rng(3).standard_normal((batch * seq, N))
    ref = O.seq_scatter(x, batch, seq, tp)          # [tp][batch][seq/tp][N]
    for r in range(tp):
        got = path.sp_slice(torch.from_numpy(x), batch, seq, tp, r).numpy()
        assert np.array_equal(got, ref[r])
        assert got.shape[0] * got.shape[1] == path.sp_rows(batch, seq, tp)
    assert path.recv_buffer_numel(tp, batch, seq, N) == tp * batch * (seq // tp) * N


@pytest.mark.parametrize("seq,tp", [(8, 2), (12, 4), (16, 8), (5, 1)])
def test_token_owner_is_the_rank_whose_slice_holds_the_token(seq, tp):
    batch, N = 2, 1
    tok = np.tile(np.arange(seq, dtype=np.float64), batch).reshape(batch * seq, N)
    for r in range(tp):
        held = path.sp_slice(torch.from_numpy(tok), batch, seq, tp, r).numpy().ravel()
        for t in held.astype(int):
            assert path.sp_token_owner(int(t), seq, tp) == r


def test_indivisible_sequence_is_rejected():
    with pytest.raises(ValueError):
        path.sp_rows(2, 10, 4)
