"""GPU parity of every kernel against the fp64 oracle on small and ragged shapes.

Inputs come from the seeded generator on the host and are copied to the GPU;
the oracle reads the same (bf16-exact) values in float64.  Shapes span several
tiles plus ragged tails in M, N and K, uneven sub-parameter pieces, empty
inputs and tie cases.  All calls go through the C ABI (ctypes binding).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import tensor_transformer_linear_b200 as T
from workloads import gen

from . import _bounds as Bd
from ._parity import TOL_BF16, TOL_FP32, check_ids, check_shard_ids, f64, rel

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _t(shape, sigma, tid, dtype=torch.bfloat16, seed=0, mu=0.0):
    return gen.normal(shape, sigma, tensor_id=tid, seed=seed, dtype=dtype, mu=mu)


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert T.tpl_get_device_status() == 0


# ---------------------------------------------------------------- generator

def test_generator_device_matches_host_bitwise():
    for dtype, sigma, mu in [(torch.bfloat16, 0.02, 0.0), (torch.float32, 0.1, 1.0)]:
        h = gen.normal((1000, 77), sigma, tensor_id=5, dtype=dtype, mu=mu, chunk=4096)
        d = gen.normal((1000, 77), sigma, tensor_id=5, dtype=dtype, mu=mu, device=DEV, chunk=4096)
        assert torch.equal(h, d.cpu())


# ------------------------------------------------------------------ RMSNorm

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("M,H", [(1, 64), (7, 4096), (133, 8192), (33, 72), (5, 12288),
                                 (300, 256), (3, 1000)])
@pytest.mark.parametrize("mode", ["none", "centered", "plain"])
def test_rmsnorm(dtype, M, H, mode):
    x = _t((M, H), 1.0, 0, dtype)
    s = _t((H,), 0.1, 4, torch.float32) if mode != "none" else None
    y = T.tpl_rmsnorm(x.to(DEV), s.to(DEV) if s is not None else None, mode == "centered")
    torch.cuda.synchronize()
    ref, own = Bd.rmsnorm(f64(x), None if s is None else f64(s), mode == "centered", 1e-6)
    bf16 = dtype == torch.bfloat16
    assert rel(y, ref) <= (TOL_BF16 if bf16 else TOL_FP32)
    Bd.check(f64(y), ref, own, u_out=Bd.U_BF16 if bf16 else Bd.U_FP32)


def test_rmsnorm_in_place_and_empty():
    x = _t((64, 4096), 1.0, 0).to(DEV)
    ref, own = Bd.rmsnorm(f64(x))
    T.tpl_rmsnorm(x, None, False, 1e-6, y=x)
    assert rel(x, ref) <= TOL_BF16
    Bd.check(f64(x), ref, own)
    e = torch.empty((0, 4096), dtype=torch.bfloat16, device=DEV)
    T.tpl_rmsnorm(e)


# ------------------------------------------------------------ column linear

COLUMN_CASES = [
    # sub_sizes, tp, align, M, K, bias, act
    ([4096 // 8, 1024 // 8, 1024 // 8], 8, 16, 130, 256, True, "none"),   # GQA-like, small
    ([1024], 4, 1, 32, 256, False, "gelu_tanh"),
    ([136, 24, 8], 1, 8, 257, 72, True, "gelu_erf"),                     # ragged pieces and K
    ([256, 256, 256], 2, 128, 1, 64, True, "none"),                      # M = 1
    ([1792 * 2], 2, 1, 200, 520, False, "gelu_erf"),                     # K ragged > 1 block
    ([512, 384, 384], 3, 128, 129, 8, True, "gelu_tanh"),                # uneven ranks, K = 8
    ([14336 // 16], 8, 1, 384, 4096, False, "gelu_erf"),                 # long K
]


@pytest.mark.parametrize("case", COLUMN_CASES)
def test_column_linear_bf16(case):
    subs, tp, align, M, K, with_bias, act = case
    part = O.partition_subparams(subs, tp, align)
    x = _t((M, K), 1.0, 0)
    w = _t((sum(subs), K), 0.02, 1)
    b = _t((sum(subs),), 0.02, 3) if with_bias else None
    p = T.tpl_partition_subparams(subs, tp, align)
    y = T.tpl_column_linear(p, x.to(DEV), w.to(DEV), b.to(DEV) if b is not None else None, act)
    torch.cuda.synchronize()
    ref, own, _ = Bd.column(f64(x), f64(w), None if b is None else f64(b), part, act)
    got = [f64(v) for v in T.shard_views(y, p, M)]
    err = O.rel_frobenius(np.concatenate([g.ravel() for g in got]),
                          np.concatenate([r.ravel() for r in ref]))
    assert err <= TOL_BF16, err
    for r_, (g, r, e) in enumerate(zip(got, ref, own)):
        assert O.rel_frobenius(g, r) <= TOL_BF16
        Bd.check(g, r, e, what=f"rank {r_}")


def test_column_linear_fp32_tiny_mlp_shapes():
    part = O.partition_subparams([1024], 4, 1)
    x = _t((32, 256), 1.0, 0, torch.float32)
    w = _t((1024, 256), 0.02, 1, torch.float32)
    p = T.tpl_partition_subparams([1024], 4, 1)
    y = T.tpl_column_linear(p, x.to(DEV), w.to(DEV), None, "gelu_tanh")
    torch.cuda.synchronize()
    ref, own, _ = Bd.column(f64(x), f64(w), None, part, "gelu_tanh", simt=True)
    for g, r, e in zip(T.shard_views(y, p, 32), ref, own):
        assert rel(g, r) <= TOL_FP32
        Bd.check(f64(g), r, e, u_out=Bd.U_FP32)


def test_column_linear_fp32_ragged_with_bias():
    subs, tp = [70, 30, 30], 3
    part = O.partition_subparams(subs, tp, 10)
    x = _t((67, 33), 1.0, 0, torch.float32)
    w = _t((130, 33), 0.5, 1, torch.float32)
    b = _t((130,), 0.5, 3, torch.float32)
    p = T.tpl_partition_subparams(subs, tp, 10)
    y = T.tpl_column_linear(p, x.to(DEV), w.to(DEV), b.to(DEV), "gelu_erf")
    torch.cuda.synchronize()
    ref, own, _ = Bd.column(f64(x), f64(w), f64(b), part, "gelu_erf", simt=True)
    for g, r, e in zip(T.shard_views(y, p, 67), ref, own):
        assert rel(g, r) <= TOL_FP32
        Bd.check(f64(g), r, e, u_out=Bd.U_FP32)


def test_column_linear_many_pieces_two_launches():
    # 16 ranks x 5 sub-parameters = 80 pieces: more than one launch's piece table
    subs, tp = [16 * 16, 16 * 8, 16 * 8, 16 * 24, 16 * 8], 16
    part = O.partition_subparams(subs, tp, 8)
    x = _t((150, 128), 1.0, 0)
    w = _t((sum(subs), 128), 0.05, 1)
    b = _t((sum(subs),), 0.05, 3)
    p = T.tpl_partition_subparams(subs, tp, 8)
    y = T.tpl_column_linear(p, x.to(DEV), w.to(DEV), b.to(DEV), "none")
    torch.cuda.synchronize()
    ref, own, _ = Bd.column(f64(x), f64(w), f64(b), part)
    for g, r, e in zip(T.shard_views(y, p, 150), ref, own):
        assert rel(g, r) <= TOL_BF16
        Bd.check(f64(g), r, e)


def test_column_linear_raster_leaves_results_bitwise_equal(monkeypatch):
    # The CTA-pair GEMM's raster (m-blocks per group, TPL_GEMM_GROUP_M, read per
    # call) only reorders whole tiles; each tile's K sum runs in the same order,
    # so every setting gives the same bits.  K = 8192 is where the library's own
    # choice drops from 16 to 8 blocks per group.
    subs, tp, M, K = [2048], 2, 1300, 8192
    x = _t((M, K), 1.0, 0, seed=7).to(DEV)
    w = _t((sum(subs), K), 0.01, 1, seed=7).to(DEV)
    p = T.tpl_partition_subparams(subs, tp, 1)
    outs = []
    for g in ("", "1", "3", "16"):
        monkeypatch.setenv("TPL_GEMM_GROUP_M", g)
        outs.append(T.tpl_column_linear(p, x, w, None, "gelu_erf"))
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    part = O.partition_subparams(subs, tp, 1)
    rows = [0, 1, 511, 512, 1299]
    ref, own, _ = Bd.column(f64(x.cpu()[rows]), f64(w.cpu()), None, part, "gelu_erf")
    for g, r, e in zip(T.shard_views(outs[0], p, M), ref, own):
        Bd.check(f64(g[rows]), r, e)


def test_column_linear_empty_rows():
    p = T.tpl_partition_subparams([256], 2, 1)
    x = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    w = _t((256, 64), 0.02, 1).to(DEV)
    y = torch.zeros(8, dtype=torch.bfloat16, device=DEV)
    T.tpl_column_linear(p, x, w, None, "none", y=y)
    assert int(y.abs().sum()) == 0


# --------------------------------------------------------------- row linear

ROW_CASES = [
    # tp, Kr, M, N, bias, residual
    (8, 64, 130, 256, False, False),
    (2, 72, 257, 300, True, True),
    (1, 4096, 128, 512, False, True),
    (4, 8, 1, 8, True, False),
    (8, 1792 // 4, 384, 4096 // 8, False, False),
]


@pytest.mark.parametrize("case", ROW_CASES)
def test_row_linear_reduce_bf16(case):
    tp, Kr, M, N, with_bias, with_res = case
    k_w = [Kr] * tp
    h = _t((M, Kr * tp), 1.0, 5)
    w2 = _t((N, Kr * tp), 0.02, 2)
    b = _t((N,), 0.02, 3) if with_bias else None
    res = _t((M, N), 1.0, 6) if with_res else None
    hp = T.pack_row_weight(h, k_w)           # rank-major H blocks [M][Kr]
    wp = T.pack_row_weight(w2, k_w)
    parts = torch.empty(tp * M * N, dtype=torch.float32, device=DEV)
    y = T.tpl_row_linear_reduce(hp.to(DEV), k_w, M, wp.to(DEV),
                                b.to(DEV) if b is not None else None,
                                res.to(DEV) if res is not None else None, partials=parts)
    torch.cuda.synchronize()
    hs = O.row_weight_slices(f64(h), k_w)
    ws = O.row_weight_slices(f64(w2), k_w)
    ref, own, _ = Bd.row(hs, ws, None if b is None else f64(b), None if res is None else f64(res))
    assert rel(y, ref) <= TOL_BF16
    Bd.check(f64(y), ref, own)
    pref, pown = Bd.partials(hs, ws)
    pg = f64(parts).reshape(tp, M, N)
    for r in range(tp):
        assert O.rel_frobenius(pg[r], pref[r]) <= 1e-5   # fp32 partials of bf16 inputs
        Bd.check(pg[r], pref[r], pown[r], u_out=Bd.U_FP32, what=f"partial {r}")


def test_row_linear_residual_aliases_output():
    tp, Kr, M, N = 4, 64, 200, 384
    k_w = [Kr] * tp
    h = _t((M, Kr * tp), 1.0, 5)
    w2 = _t((N, Kr * tp), 0.02, 2)
    x = _t((M, N), 1.0, 6)
    xd = x.to(DEV)
    T.tpl_row_linear_reduce(T.pack_row_weight(h, k_w).to(DEV), k_w, M,
                            T.pack_row_weight(w2, k_w).to(DEV), None, xd, y=xd)
    torch.cuda.synchronize()
    ref, own, _ = Bd.row(O.row_weight_slices(f64(h), k_w), O.row_weight_slices(f64(w2), k_w),
                         None, f64(x))
    assert rel(xd, ref) <= TOL_BF16
    Bd.check(f64(xd), ref, own)


def test_row_linear_fp32_uneven_ranks():
    k_w = [40, 40, 24, 24]
    M, N = 33, 70
    h = _t((M, sum(k_w)), 1.0, 5, torch.float32)
    w2 = _t((N, sum(k_w)), 0.1, 2, torch.float32)
    b = _t((N,), 0.1, 3, torch.float32)
    res = _t((M, N), 1.0, 6, torch.float32)
    parts = torch.empty(4 * M * N, dtype=torch.float32, device=DEV)
    y = T.tpl_row_linear_reduce(T.pack_row_weight(h, k_w).to(DEV), k_w, M,
                                T.pack_row_weight(w2, k_w).to(DEV), b.to(DEV), res.to(DEV),
                                partials=parts)
    torch.cuda.synchronize()
    hs, ws = O.row_weight_slices(f64(h), k_w), O.row_weight_slices(f64(w2), k_w)
    ref, own, _ = Bd.row(hs, ws, f64(b), f64(res), simt=True)
    assert rel(y, ref) <= TOL_FP32
    Bd.check(f64(y), ref, own, u_out=Bd.U_FP32)
    pg = f64(parts).reshape(4, M, N)
    pref, pown = Bd.partials(hs, ws, simt=True)
    for r, pr in enumerate(pref):
        assert O.rel_frobenius(pg[r], pr) <= TOL_FP32
        Bd.check(pg[r], pr, pown[r], u_out=Bd.U_FP32)


@pytest.mark.parametrize("k_w,M,N", [([16, 16, 8], 200, 136), ([72, 64, 64, 64], 300, 256),
                                     ([336, 336, 328], 1, 40)])
def test_row_linear_bf16_two_rank_widths(k_w, M, N):
    # remainder units on the lowest ranks: two contiguous groups of equal width
    h = _t((M, sum(k_w)), 1.0, 5)
    w2 = _t((N, sum(k_w)), 0.05, 2)
    tp = len(k_w)
    parts = torch.empty(tp * M * N, dtype=torch.float32, device=DEV)
    y = T.tpl_row_linear_reduce(T.pack_row_weight(h, k_w).to(DEV), k_w, M,
                                T.pack_row_weight(w2, k_w).to(DEV), partials=parts)
    torch.cuda.synchronize()
    hs, ws = O.row_weight_slices(f64(h), k_w), O.row_weight_slices(f64(w2), k_w)
    ref, own, _ = Bd.row(hs, ws)
    assert rel(y, ref) <= TOL_BF16
    Bd.check(f64(y), ref, own)
    pg = f64(parts).reshape(tp, M, N)
    pref, pown = Bd.partials(hs, ws)
    for r, pr in enumerate(pref):
        assert O.rel_frobenius(pg[r], pr) <= 1e-5
        Bd.check(pg[r], pr, pown[r], u_out=Bd.U_FP32)


def test_row_linear_bf16_three_rank_widths_rejected():
    h = torch.zeros(4 * 40, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(8 * 40, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(T.TplError) as e:
        T.tpl_row_linear_reduce(h, [16, 8, 16], 4, w)
    assert e.value.name == "TPL_ERR_UNSUPPORTED"


def test_tp_mlp_uneven_partition_end_to_end():
    # intermediate 1000 over tp 3 in units of 8: widths 336, 336, 328
    M, H, I, tp = 257, 256, 1000, 3
    x = _t((M, H), 1.0, 0)
    w1, w2 = _t((I, H), 0.05, 1), _t((H, I), 0.05, 2)
    p = T.tpl_partition_subparams([I], tp, 8)
    k_w = [p.shard_width[r] for r in range(tp)]
    hbuf = T.tpl_column_linear(p, x.to(DEV), w1.to(DEV), None, "gelu_erf")
    y = T.tpl_row_linear_reduce(hbuf, k_w, M, T.pack_row_weight(w2, k_w).to(DEV))
    torch.cuda.synchronize()
    part = O.partition_subparams([I], tp, 8)
    ref = O.row_linear_reduce(O.column_linear(f64(x), f64(w1), None, part, "gelu_erf"),
                              O.row_weight_slices(f64(w2), part.shard_width))
    assert part.shard_width == [336, 336, 328]
    assert rel(y, ref) <= TOL_BF16
    bref, own, car = Bd.mlp(f64(x), f64(w1), f64(w2), tp, "gelu_erf", align=8)
    Bd.check(f64(y), bref, own, car)


# ---------------------------------------------------------------- LM head

LM_CASES = [
    # B, K, V, tp, n_chunks, logits
    (3, 64, 1000, 4, 2, True),
    (32, 4096, 9000, 8, 4, True),
    (17, 200, 37, 4, 2, True),          # shards of 10 ids: several shards inside one slab
    (1, 8, 9, 8, 1, False),             # empty shards
    (48, 128, 2000, 3, 5, True),        # B > 32, uneven
    (128, 256, 5000, 4, 2, True),       # one full 128-row batch tile
    (129, 128, 3000, 2, 3, True),       # two batch tiles, the second with one row
    (256, 192, 40000, 8, 4, True),      # two full batch tiles of 160 columns: one TMEM buffer
    # vocab ranges of the transposed kernel on 148 SMs: 255-row ranges that are
    # one short last slab next to 256-row ones that are one whole slab, and
    # 512-row ranges with no short slab at all
    (8, 64, 148 * 255 + 50, 4, 2, True),
    (5, 128, 148 * 512, 8, 1, False),
]


@pytest.mark.parametrize("case", LM_CASES)
def test_lmhead_argmax(case):
    B, K, V, tp, nc, with_logits = case
    x = _t((B, K), 1.0, 0)
    w = _t((V, K), 0.02, 1)
    ws = T.lmhead_workspace(B, V, tp, nc)
    logits = torch.empty(B * V, dtype=torch.float32, device=DEV) if with_logits else None
    for rep in range(2):                 # the workspace is reused without clearing
        ids, smax, sidx = T.tpl_lmhead_argmax(x.to(DEV), w.to(DEV), tp, nc, ws, logits=logits)
        torch.cuda.synchronize()
        res = O.lmhead_argmax(f64(x), f64(w), tp, nc)
        check_ids(ids.cpu().numpy(), res)
        check_shard_ids(sidx.cpu().numpy(), smax.cpu().numpy(), res)
        if with_logits:
            assert rel(logits.view(B, V), res.logits) <= 1e-5
            Bd.check(f64(logits.view(B, V)), res.logits, Bd.logits(f64(x), f64(w)),
                     u_out=Bd.U_FP32)
        assert int(ws.abs().sum()) == 0


def test_lmhead_planted_ids_and_tie_break():
    B, K, V, tp, nc = 4, 128, 4000, 8, 4
    lay = O.vocab_layout(V, tp, nc)
    x = _t((B, K), 1.0, 0)
    w = _t((V, K), 0.01, 1).clone()
    planted = [lay.shard - 1, lay.shard, V - 1, 3 * lay.shard + lay.split_sizes[0]]
    for b, v in enumerate(planted):
        w[v] = (2.0 * x[b].float() / x[b].float().norm()).to(torch.bfloat16)
    w[7 * lay.shard - 5] = w[planted[1]]          # exact tie in a later shard
    ws = T.lmhead_workspace(B, V, tp, nc)
    ids, smax, sidx = T.tpl_lmhead_argmax(x.to(DEV), w.to(DEV), tp, nc, ws)
    torch.cuda.synchronize()
    assert ids.cpu().tolist() == planted
    assert int(sidx[6, 1]) == 7 * lay.shard - 5
