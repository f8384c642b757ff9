"""GPU parity at the five workloads' full sizes, in the launch configuration the
bench times (same calls, same shapes), checked against the fp64 oracle.

Device tensors are made on the GPU by the seeded generator; the oracle gets the
same tensors (bit for bit, see test_generator_device_matches_host_bitwise)
regenerated on the host.  Where the oracle cannot finish the whole output in
seconds it computes sampled token rows (rows are independent through every
step of the path); the LM head is compared in full.
"""
import numpy as np
import pytest
import torch

import oracle as O
import tensor_transformer_linear_b200 as T
from workloads import configs as C
from workloads import gen

from . import _bounds as Bd
from ._parity import TOL_BF16, TOL_FP32, check_ids, check_shard_ids, f64, rel

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _sample_rows(M, n=29, seed=0):
    rng = np.random.default_rng(seed)
    rows = {0, 1, M // 2, M - 1} | set(int(r) for r in rng.integers(0, M, n))
    return sorted(rows)


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert T.tpl_get_device_status() == 0


def test_tiny_tp_mlp_fp32_fused_full():
    # the whole block in one launch (tpl_tp_mlp_fp32), h kept on chip
    w = C.TINY_MLP
    x = C.mlp_x(w)
    w1, w2 = C.mlp_w1(w), C.mlp_w2(w)
    blk = T.TPMLP(w1.to(DEV), w2.to(DEV), w.tp, w.act, norm=False)
    n0 = T.tpl_launch_count()
    y = blk(x.to(DEV))
    torch.cuda.synchronize()
    assert blk.fused_fp32 and T.tpl_launch_count() - n0 == 1
    ref = O.tp_mlp(f64(x), f64(w1), f64(w2), w.tp, w.act)
    assert rel(y, ref) <= TOL_FP32
    bref, own, car = Bd.mlp(f64(x), f64(w1), f64(w2), w.tp, w.act, bf16=False)
    Bd.check(f64(y), bref, own, car, u_out=Bd.U_FP32)


def test_tiny_tp_mlp_fp32_full():
    w = C.TINY_MLP
    x = C.mlp_x(w)
    w1, w2 = C.mlp_w1(w), C.mlp_w2(w)
    blk = T.TPMLP(w1.to(DEV), w2.to(DEV), w.tp, w.act, norm=False, fused_fp32=False)
    y = blk(x.to(DEV))
    torch.cuda.synchronize()
    part = O.partition_subparams([w.inter], w.tp, 1)
    h_ref, h_own, _ = Bd.column(f64(x), f64(w1), None, part, w.act, simt=True)
    h_got = T.shard_views(blk._bufs["h"], blk.part, w.M)
    for g, r, e in zip(h_got, h_ref, h_own):
        assert rel(g, r) <= TOL_FP32
        Bd.check(f64(g), r, e, u_out=Bd.U_FP32)
    ref = O.tp_mlp(f64(x), f64(w1), f64(w2), w.tp, w.act)
    assert rel(y, ref) <= TOL_FP32
    bref, own, car = Bd.mlp(f64(x), f64(w1), f64(w2), w.tp, w.act, bf16=False)
    Bd.check(f64(y), bref, own, car, u_out=Bd.U_FP32)


def test_gqa_fused_qkv_full_size():
    w = C.GQA_QKV
    x, wq, b = C.qkv_x(w, DEV), C.qkv_w(w, DEV), C.qkv_bias(w, DEV)
    p = T.tpl_partition_subparams(w.sub_sizes, w.tp, w.align)
    y = T.tpl_column_linear(p, x, wq, b, "none")
    torch.cuda.synchronize()
    rows = _sample_rows(w.M)
    xr = gen.rows((w.M, w.hidden), rows, 1.0, tensor_id=gen.TID_X)
    part = O.partition_subparams(list(w.sub_sizes), w.tp, w.align)
    ref, own, _ = Bd.column(f64(xr), f64(C.qkv_w(w)), f64(C.qkv_bias(w)), part)
    got = [f64(v[rows]) for v in T.shard_views(y, p, w.M)]
    for g, r, e in zip(got, ref, own):
        assert O.rel_frobenius(g, r) <= TOL_BF16
        Bd.check(g, r, e)
    assert O.rel_frobenius(np.concatenate(got, 1), np.concatenate(ref, 1)) <= TOL_BF16


def test_rmsnorm_tp_mlp_full_size():
    w = C.TP_MLP
    x = C.mlp_x(w, DEV)
    s = C.mlp_scale(w, 0, DEV)
    blk = T.TPMLP(C.mlp_w1(w, 0, DEV), C.mlp_w2(w, 0, DEV), w.tp, w.act, scale=s,
                  centered=True, norm=True)
    y = blk(x)
    torch.cuda.synchronize()
    rows = _sample_rows(w.M)
    xr = gen.rows((w.M, w.hidden), rows, 1.0, tensor_id=gen.TID_X)
    ref, own, car = Bd.mlp(f64(xr), f64(C.mlp_w1(w)), f64(C.mlp_w2(w)), w.tp, w.act,
                           scale=f64(C.mlp_scale(w)), centered=True, norm=True)
    assert rel(y[rows], ref) <= TOL_BF16
    Bd.check(f64(y[rows]), ref, own, car)
    # the RMSNorm output of the same rows (first step of the block)
    xn = blk._bufs["xn"].view(w.M, w.hidden)[rows]
    nref, nown = Bd.rmsnorm(f64(xr), f64(C.mlp_scale(w)), True)
    assert rel(xn, nref) <= TOL_BF16
    Bd.check(f64(xn), nref, nown)


def test_decode_lmhead_full_size():
    w = C.LM_HEAD
    x, wl = C.lm_x(w, DEV), C.lm_w(w, DEV)
    ws = T.lmhead_workspace(w.batch, w.vocab, w.tp, w.n_chunks)
    logits = torch.empty(w.batch * w.vocab, dtype=torch.float32, device=DEV)
    ids, smax, sidx = T.tpl_lmhead_argmax(x, wl, w.tp, w.n_chunks, ws, logits=logits)
    ids2, smax2, sidx2 = T.tpl_lmhead_argmax(x, wl, w.tp, w.n_chunks, ws)   # no logits, reused ws
    torch.cuda.synchronize()
    del wl
    res = O.lmhead_argmax(f64(C.lm_x(w)), f64(C.lm_w(w)), w.tp, w.n_chunks)
    check_ids(ids.cpu().numpy(), res)
    check_shard_ids(sidx.cpu().numpy(), smax.cpu().numpy(), res)
    assert torch.equal(ids, ids2) and torch.equal(sidx, sidx2) and torch.equal(smax, smax2)
    assert rel(logits.view(w.batch, w.vocab), res.logits) <= 1e-5
    Bd.check(f64(logits.view(w.batch, w.vocab)), res.logits,
             Bd.logits(f64(C.lm_x(w)), f64(C.lm_w(w))), u_out=Bd.U_FP32)
    # the chunk layout the ids follow (global id = r * shard + chunk offset + j)
    lay = O.vocab_layout(w.vocab, w.tp, w.n_chunks)
    assert lay.shard == 16032 and lay.split_sizes == [4008] * 4
    assert all(r * lay.shard <= int(sidx[r, b]) < (r + 1) * lay.shard
               for r in range(w.tp) for b in range(w.batch))


@pytest.mark.slow
def test_four_layer_stack_full_size():
    w = C.STACK4
    x = C.mlp_x(w, DEV)
    layers = [T.TPMLP(C.mlp_w1(w, l, DEV), C.mlp_w2(w, l, DEV), w.tp, w.act, norm=True,
                      residual=True) for l in range(w.layers)]
    T.TPStack(layers)(x)
    torch.cuda.synchronize()
    rows = _sample_rows(w.M, n=11)
    got = f64(x[rows])
    del layers, x
    torch.cuda.empty_cache()
    x0 = f64(gen.rows((w.M, w.hidden), rows, 1.0, tensor_id=gen.TID_X))
    xr = x0
    for l in range(w.layers):
        w1, w2 = f64(C.mlp_w1(w, l)), f64(C.mlp_w2(w, l))
        xr = O.tp_mlp(xr, w1, w2, w.tp, w.act, norm=True, residual=True)
        del w1, w2
    err = O.rel_frobenius(got, xr)
    assert err <= TOL_BF16, err
    # element-wise: the bound carried through all four layers
    layers = [(f64(C.mlp_w1(w, l)), f64(C.mlp_w2(w, l))) for l in range(w.layers)]
    bref, own, car = Bd.stack(x0, layers, w.tp, w.act)
    del layers
    Bd.check(got, bref, own, car)
