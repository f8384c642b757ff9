"""GPU parity of the TP linears split over GPUs, with the ranks run one after
another on one GPU: every rank's scatter writes into the receive buffers of all
ranks (here local tensors standing in for its peers'; no kernel waits on
another), then every rank reduces its slots.  Checked against the fp64 oracle:
the reduce-scatter result, every slot's partial, the all-reduce form (every
rank's slice stored into every rank's full output), and the argmax merged over
ranks."""
import numpy as np
import pytest
import torch

import oracle as O
import tensor_transformer_linear_b200 as T
from workloads import gen

from . import _bounds as Bd
from ._parity import TOL_BF16, check_ids, f64, rel

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _t(shape, sigma, tid, seed=5):
    return gen.normal(shape, sigma, tensor_id=tid, seed=seed)


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert T.tpl_get_device_status() == 0


@pytest.mark.parametrize("tp,batch,seq,inter,N,with_bias,with_res", [
    (4, 2, 256, 512, 256, True, True),       # M = 512: CTA-pair kernel
    (2, 1, 64, 128, 130, False, True),       # M = 64: single-CTA kernel; N % 8 != 0
    (8, 1, 1024, 1792, 512, False, False),   # tp 8, the MLP's contraction split
    (3, 2, 96, 200, 64, True, False),        # uneven contraction split 72/64/64
])
def test_scatter_then_reduce_is_the_reduce_scatter(tp, batch, seq, inter, N, with_bias,
                                                   with_res):
    part = O.partition_subparams([inter], tp, 8)
    k_w = part.shard_width
    M, seg = batch * seq, seq // tp
    H = _t((M, inter), 1.0, 0)
    W2 = _t((N, inter), 0.02, 2)
    bias = _t((N,), 0.02, 3) if with_bias else None
    res = _t((M, N), 1.0, 4) if with_res else None

    recv = [torch.full((tp * batch * seg * N,), float("nan"), dtype=torch.bfloat16, device=DEV)
            for _ in range(tp)]
    koff = 0
    for r in range(tp):
        hr = H[:, koff:koff + k_w[r]].contiguous().to(DEV)
        wr = W2[:, koff:koff + k_w[r]].contiguous().to(DEV)
        T.tpl_row_linear_scatter(hr, wr, batch, seq, r, tp, recv)
        koff += k_w[r]
    torch.cuda.synchronize()

    bias_d = bias.to(DEV) if bias is not None else None
    ys = []
    for q in range(tp):
        rq = None
        if res is not None:   # rank q's token slice of the residual stream
            rq = res.view(batch, tp, seg, N)[:, q].contiguous().to(DEV)
        ys.append(T.tpl_reduce_slots(recv[q], tp, N, bias_d, rq))
    torch.cuda.synchronize()
    got = np.stack([f64(y).reshape(batch, seg, N) for y in ys])

    h_parts, off = [], 0
    for k in k_w:
        h_parts.append(f64(H)[:, off:off + k])
        off += k
    w_parts = O.row_weight_slices(f64(W2), k_w)
    res_sp = O.seq_scatter(f64(res), batch, seq, tp) if res is not None else None
    ref = O.row_linear_reduce_scatter(h_parts, w_parts, batch, seq,
                                      bias=None if bias is None else f64(bias),
                                      residual_sp=res_sp)
    assert rel(got, ref) <= TOL_BF16
    full, own, car = Bd.scatter_reduce(h_parts, w_parts, None if bias is None else f64(bias),
                                       None if res is None else f64(res))
    sp = lambda a: O.seq_scatter(a, batch, seq, tp)
    Bd.check(got, sp(full), sp(own), sp(car))

    # Slot s of rank q's buffer is rank s's partial of rank q's tokens.
    parts, pown = Bd.partials(h_parts, w_parts)
    for q in range(tp):
        slots = f64(recv[q]).reshape(tp, batch, seg, N)
        for s in range(tp):
            assert rel(slots[s], sp(parts[s])[q]) <= TOL_BF16
            Bd.check(slots[s], sp(parts[s])[q], sp(pown[s])[q], what=f"slot {s} of rank {q}")


@pytest.mark.parametrize("tp,batch,seq,inter,N,with_bias,res_mode", [
    (4, 2, 256, 512, 256, True, "in_place"),    # vector kernel, residual = the output
    (2, 1, 64, 128, 130, False, "separate"),    # N % 8 != 0: scalar kernel
    (8, 1, 1024, 1792, 512, False, "none"),     # tp 8, the MLP's contraction split
    (3, 2, 96, 200, 64, True, "separate"),      # uneven contraction split 72/64/64
])
def test_scatter_then_reduce_allgather_is_the_full_row_linear_on_every_rank(
        tp, batch, seq, inter, N, with_bias, res_mode):
    part = O.partition_subparams([inter], tp, 8)
    k_w = part.shard_width
    M = batch * seq
    H = _t((M, inter), 1.0, 0)
    W2 = _t((N, inter), 0.02, 2)
    bias = _t((N,), 0.02, 3) if with_bias else None
    res = _t((M, N), 1.0, 4) if res_mode != "none" else None

    recv = [torch.full((M * N,), float("nan"), dtype=torch.bfloat16, device=DEV)
            for _ in range(tp)]
    if res_mode == "in_place":      # every rank's output starts as its residual stream
        outs = [res.to(DEV) for _ in range(tp)]
    else:
        outs = [torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
                for _ in range(tp)]
    koff = 0
    for r in range(tp):
        hr = H[:, koff:koff + k_w[r]].contiguous().to(DEV)
        wr = W2[:, koff:koff + k_w[r]].contiguous().to(DEV)
        T.tpl_row_linear_scatter(hr, wr, batch, seq, r, tp, recv)
        koff += k_w[r]
    bias_d = bias.to(DEV) if bias is not None else None
    for q in range(tp):
        res_q = None
        if res_mode == "in_place":
            res_q = outs[q]
        elif res_mode == "separate":
            res_q = res.to(DEV)
        T.tpl_reduce_slots_allgather(recv[q], tp, batch, seq, N, q, outs, bias=bias_d,
                                     residual=res_q)
    torch.cuda.synchronize()

    h_parts, off = [], 0
    for k in k_w:
        h_parts.append(f64(H)[:, off:off + k])
        off += k
    ref = O.row_linear_reduce(h_parts, O.row_weight_slices(f64(W2), k_w),
                              None if bias is None else f64(bias),
                              None if res is None else f64(res))
    full, own, car = Bd.scatter_reduce(h_parts, O.row_weight_slices(f64(W2), k_w),
                                       None if bias is None else f64(bias),
                                       None if res is None else f64(res))
    for q in range(tp):
        assert rel(outs[q], ref) <= TOL_BF16, q
        assert torch.equal(outs[q], outs[0]), q      # every rank holds the same Y
    Bd.check(f64(outs[0]), full, own, car)


def test_reduce_slots_in_place_on_the_residual():
    tp, rows, N = 3, 40, 64
    recv = _t((tp, rows, N), 1.0, 6).to(DEV)
    res = _t((rows, N), 1.0, 7)
    y = res.to(DEV)
    T.tpl_reduce_slots(recv, tp, N, None, y, y=y)
    torch.cuda.synchronize()
    ref = f64(recv).sum(axis=0) + f64(res)
    assert rel(y, ref) <= TOL_BF16
    sref, own = Bd.slot_sum(list(f64(recv)), f64(res))
    Bd.check(f64(y), sref, own)


@pytest.mark.parametrize("tp,rows,N,with_bias,scale_mode,in_place", [
    (8, 100, 4096, True, "centered", True),    # the MLP's hidden: one vector per thread
    (3, 37, 264, False, None, False),           # narrow rows: 33 vectors on 64 threads
    (4, 9, 8192, False, "plain", False),        # two vectors per thread
    (10, 5, 16384, False, "plain", True),       # four per thread, the widest row; tp > 8
])
def test_reduce_slots_rmsnorm(tp, rows, N, with_bias, scale_mode, in_place):
    recv = _t((tp, rows, N), 1.0, 6).to(DEV)
    res = _t((rows, N), 1.0, 7)
    bias = _t((N,), 0.02, 8).to(DEV) if with_bias else None
    scale = (gen.normal((N,), 0.1, tensor_id=9, dtype=torch.float32).to(DEV)
             if scale_mode else None)
    centered = scale_mode == "centered"
    y = res.to(DEV) if in_place else torch.empty((rows, N), dtype=torch.bfloat16, device=DEV)
    xn = torch.empty((rows, N), dtype=torch.bfloat16, device=DEV)
    T.tpl_reduce_slots_rmsnorm(recv, tp, N, xn, scale=scale, centered=centered, bias=bias,
                               residual=y if in_place else res.to(DEV), y=y)
    y_plain = T.tpl_reduce_slots(recv, tp, N, bias, res.to(DEV))
    torch.cuda.synchronize()
    # the residual stream: tpl_reduce_slots' arithmetic, bit for bit, and the oracle
    assert torch.equal(y, y_plain)
    slots = list(f64(recv)) + ([np.broadcast_to(f64(bias), (rows, N))] if with_bias else [])
    sref, own = Bd.slot_sum(slots, f64(res))
    Bd.check(f64(y), sref, own)
    # the next layer's input: RMSNorm of the stored bf16 y (google-research
    # allgather_layernorm), against the oracle and against tpl_rmsnorm on y
    xref, own_n = Bd.rmsnorm(f64(y), None if scale is None else f64(scale), centered)
    assert rel(xn, xref) <= TOL_BF16
    Bd.check(f64(xn), xref, own_n)
    unfused = T.tpl_rmsnorm(y, scale, centered, 1e-6)
    assert rel(xn, f64(unfused)) <= 1e-2 * TOL_BF16


@pytest.mark.parametrize("B,K,V,tp", [(32, 256, 4999, 4), (5, 64, 37, 8)])
def test_lmhead_argmax_merged_over_ranks(B, K, V, tp):
    x = _t((B, K), 1.0, 0)
    w = _t((V, K), 0.02, 1).clone()
    shard = -(-V // tp)
    if V > 3 * shard:
        # batch row 0's maximum planted twice, on ranks 1 and 3: an exact tie
        # across ranks, which the lower global id must win
        w[shard + 7] = (3.0 * x[0].float() / x[0].float().norm()).to(torch.bfloat16)
        w[3 * shard + 2] = w[shard + 7]
    smax = torch.empty((tp, B), dtype=torch.float32, device=DEV)
    sidx = torch.empty((tp, B), dtype=torch.int32, device=DEV)
    for s in range(tp):
        lo, hi = s * shard, min(V, (s + 1) * shard)
        if lo >= hi:                       # a rank whose vocab slice is empty
            smax[s].fill_(float("-inf"))
            sidx[s].fill_(-1)
            continue
        ws = T.lmhead_workspace(B, hi - lo, 1, 1)
        _, m, i = T.tpl_lmhead_argmax(x.to(DEV), w[lo:hi].contiguous().to(DEV), 1, 1, ws)
        smax[s], sidx[s] = m[0], i[0]
    ids = T.tpl_argmax_merge(smax, sidx, shard)
    torch.cuda.synchronize()
    res = O.lmhead_argmax(f64(x), f64(w), tp, 1)
    check_ids(ids.cpu().numpy(), res)
    if V > 3 * shard:
        assert int(ids[0]) == shard + 7


@pytest.mark.parametrize("tp,batch,seq,K,subs,align,with_bias,act", [
    (4, 2, 512, 256, [1024], 1, True, "gelu_erf"),            # c_fc shard, CTA-pair kernel
    (2, 1, 256, 128, [512, 256, 256], 128, True, "none"),      # fused QKV pieces per rank
    (8, 1, 1024, 64, [256], 1, False, "gelu_tanh"),            # tp 8, 128-token slices
    (1, 1, 128, 64, [256], 1, True, "none"),                   # M = 128: single-CTA kernel
])
def test_gather_column_is_the_column_linear_of_the_gathered_tokens(tp, batch, seq, K, subs, align,
                                                                   with_bias, act):
    M, seg = batch * seq, seq // tp
    x = _t((M, K), 1.0, 0)
    W = _t((sum(subs), K), 0.02, 1)
    b = _t((sum(subs),), 0.02, 3) if with_bias else None
    part = O.partition_subparams(subs, tp, align)
    ref, own, _ = Bd.column(f64(x), f64(W), None if b is None else f64(b), part, act)
    # rank q's token slice: tokens q * seg .. of every sequence
    slices = [x.view(batch, tp, seg, K)[:, q].contiguous().to(DEV) for q in range(tp)]
    for r in range(tp):
        widths = [part.width[r][j] for j in range(len(subs))]
        rows = [slice(part.src_off[r][j], part.src_off[r][j] + widths[j])
                for j in range(len(subs))]
        w_r = torch.cat([W[s] for s in rows]).contiguous().to(DEV)
        b_r = torch.cat([b[s] for s in rows]).contiguous().to(DEV) if b is not None else None
        p_r = T.tpl_partition_subparams(widths, 1, 1)
        y_r = T.tpl_column_linear_gather(p_r, slices, batch, seq, w_r, b_r, act)
        torch.cuda.synchronize()
        assert rel(f64(y_r).reshape(M, part.shard_width[r]), ref[r]) <= TOL_BF16
        Bd.check(f64(y_r).reshape(M, part.shard_width[r]), ref[r], own[r])
