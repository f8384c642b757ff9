"""The GEMMs with a stream-K workspace (tpl_*_ws): the last full tile wave and
the partial one are split over the CTA pairs by K steps, and a tile split
between two pairs is finished by the pair that computes its head, which adds
the other pair's fp32 partial.  Shapes are chosen so that the last wave is
partial (tiles = waves * 74 + remainder on a 148-SM B200), with one and several
waves before it, K tails, two contraction widths, fused pieces and the
multi-GPU gather / scatter forms.  Checked against the oracle (relative
Frobenius and element-wise bounds) and against the plain schedule."""
import numpy as np
import pytest
import torch

import oracle as O
import tensor_transformer_linear_b200 as T
from workloads import gen

from . import _bounds as Bd
from ._parity import TOL_BF16, f64, rel

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _t(shape, sigma, tid, seed=5):
    return gen.normal(shape, sigma, tensor_id=tid, seed=seed)


@pytest.fixture(scope="module")
def ws():
    return T.gemm_workspace(DEV)


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert T.tpl_get_device_status() == 0


COLUMN = [
    # subs, tp, align, M, K, bias, act     tiles of 256 x 256 (pairs: 74)
    ([2560], 8, 1, 2048, 512, True, "gelu_erf"),             # 8 x 10 = 80: one wave + 6
    ([4096, 1024, 1024], 8, 128, 4096, 4096, True, "none"),  # the fused QKV: 384 = 5 x 74 + 14
    ([3072, 512, 512], 4, 128, 3000, 200, False, "none"),    # ragged M and K: 12 x 16 = 192
    ([14336 // 4], 2, 1, 6144, 256, False, "gelu_tanh"),     # 24 x 14 = 336: 4 waves + 40
]


@pytest.mark.parametrize("case", COLUMN)
def test_column_linear_stream_k(case, ws):
    subs, tp, align, M, K, with_bias, act = case
    part = O.partition_subparams(subs, tp, align)
    x, w = _t((M, K), 1.0, 0), _t((sum(subs), K), 0.02, 1)
    b = _t((sum(subs),), 0.02, 3) if with_bias else None
    p = T.tpl_partition_subparams(subs, tp, align)
    xd, wd, bd = x.to(DEV), w.to(DEV), (b.to(DEV) if b is not None else None)
    y = T.tpl_column_linear(p, xd, wd, bd, act, workspace=ws)
    y2 = T.tpl_column_linear(p, xd, wd, bd, act, workspace=ws)      # the workspace reused
    plain = T.tpl_column_linear(p, xd, wd, bd, act)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    rows = sorted({0, 1, M // 3, M // 2, M - 1} | set(range(255, M, 997)))
    ref, own, _ = Bd.column(f64(x)[rows], f64(w), None if b is None else f64(b), part, act)
    for g, r, e in zip(T.shard_views(y, p, M), ref, own):
        g = f64(g)[rows]
        assert rel(g, r) <= TOL_BF16
        Bd.check(g, r, e)
    # only the order of fp32 additions differs on split tiles
    d = (y.float() - plain.float()).abs()
    assert float(d.max()) <= 2.0 ** -6 * float(plain.float().abs().max())


ROW = [
    # k_w, M, N, bias, residual
    ([512, 512], 4096, 1280, True, True),            # 16 x 5 = 80 tiles
    ([1792] * 8, 8192, 4096, False, False),          # the MLP's c_proj: 512 = 6 x 74 + 68
    ([200, 200, 192], 2600, 2304, False, True),      # two widths, ragged M: 11 x 9 = 99
]


@pytest.mark.parametrize("case", ROW)
def test_row_linear_stream_k(case, ws):
    k_w, M, N, with_bias, with_res = case
    tp = len(k_w)
    h, w2 = _t((M, sum(k_w)), 1.0, 5), _t((N, sum(k_w)), 0.02, 2)
    b = _t((N,), 0.02, 3) if with_bias else None
    res = _t((M, N), 1.0, 6) if with_res else None
    hp, wp = T.pack_row_weight(h, k_w).to(DEV), T.pack_row_weight(w2, k_w).to(DEV)
    bd = b.to(DEV) if b is not None else None
    rd = res.to(DEV) if res is not None else None
    y = T.tpl_row_linear_reduce(hp, k_w, M, wp, bd, rd, workspace=ws)
    plain = T.tpl_row_linear_reduce(hp, k_w, M, wp, bd, rd)
    torch.cuda.synchronize()
    rows = sorted({0, M // 2, M - 1} | set(range(100, M, 733)))
    hs = [s[rows] for s in O.row_weight_slices(f64(h), k_w)]
    ref, own, _ = Bd.row(hs, O.row_weight_slices(f64(w2), k_w), None if b is None else f64(b),
                         None if res is None else f64(res)[rows])
    assert rel(f64(y)[rows], ref) <= TOL_BF16
    Bd.check(f64(y)[rows], ref, own)
    d = (y.float() - plain.float()).abs()
    assert float(d.max()) <= 2.0 ** -6 * float(plain.float().abs().max())


def test_small_workspace_runs_the_plain_schedule(ws):
    M, K, N = 2048, 512, 2560
    p = T.tpl_partition_subparams([N], 8, 1)
    x, w = _t((M, K), 1.0, 0).to(DEV), _t((N, K), 0.02, 1).to(DEV)
    small = ws[: ws.numel() // 2]
    y = T.tpl_column_linear(p, x, w, None, "none", workspace=small)
    plain = T.tpl_column_linear(p, x, w, None, "none")
    torch.cuda.synchronize()
    assert torch.equal(y, plain)


def test_gather_and_scatter_stream_k(ws):
    # one rank's shards of an MLP split over 8 GPUs: 8192 tokens, c_fc 4096 -> 1792
    # (224 tiles = 3 x 74 + 2) and c_proj 1792 -> 4096 (512 tiles)
    tp, batch, seq, K, I, N = 8, 8, 1024, 512, 1792, 4096
    M, seg = batch * seq, seq // tp
    x = _t((M, K), 1.0, 0)
    w1 = _t((I, K), 0.02, 1)
    slices = [x.view(batch, tp, seg, K)[:, q].contiguous().to(DEV) for q in range(tp)]
    p = T.tpl_partition_subparams([I], 1, 1)
    w1d = w1.to(DEV)
    h = T.tpl_column_linear_gather(p, slices, batch, seq, w1d, None, "gelu_erf", workspace=ws)
    h_plain = T.tpl_column_linear_gather(p, slices, batch, seq, w1d, None, "gelu_erf")
    torch.cuda.synchronize()
    rows = sorted({0, M // 2, M - 1} | set(range(77, M, 1499)))
    ref, own, _ = Bd.column(f64(x)[rows], f64(w1), None, O.partition_subparams([I], 1, 1),
                            "gelu_erf")
    g = f64(h).reshape(M, I)[rows]
    assert rel(g, ref[0]) <= TOL_BF16
    Bd.check(g, ref[0], own[0])
    assert float((h.float() - h_plain.float()).abs().max()) <= 2.0 ** -6 * float(
        h_plain.float().abs().max())

    w2 = _t((N, I), 0.02, 2).to(DEV)
    recv = [torch.full((tp * batch * seg * N,), float("nan"), dtype=torch.bfloat16, device=DEV)
            for _ in range(tp)]
    recv_plain = [torch.empty_like(r) for r in recv]
    hv = h.view(M, I)
    T.tpl_row_linear_scatter(hv, w2, batch, seq, 3, tp, recv, workspace=ws)
    T.tpl_row_linear_scatter(hv, w2, batch, seq, 3, tp, recv_plain)
    torch.cuda.synchronize()
    # slot 3 of every rank: rank 3's partial of that rank's tokens
    part, pown = Bd.partials([f64(hv)[rows]], [f64(w2)])
    full = np.stack([f64(r).reshape(tp, batch * seg, N)[3] for r in recv])    # [q][b*seg][N]
    got = O.seq_gather(full.reshape(tp, batch, seg, N), batch, seq, tp)[rows]
    assert rel(got, part[0]) <= TOL_BF16
    Bd.check(got, part[0], pown[0])
    for r, rp in zip(recv, recv_plain):
        a, b_ = r.view(tp, -1)[3].float(), rp.view(tp, -1)[3].float()
        assert float((a - b_).abs().max()) <= 2.0 ** -6 * float(b_.abs().max())
