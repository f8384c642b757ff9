"""The fp32 TP MLP block in one launch (tpl_tp_mlp_fp32) against the fp64
oracle (nanotron "MLP Module"; google-research residual section): ragged token
tiles, every tp the kernel takes, both GELU forms and none, biases, the
residual separate and aliasing the output, the other shapes it takes, and the
fall-back of TPMLP to two launches for shapes it does not."""
import pytest
import torch

import oracle as O
import tensor_transformer_linear_b200 as T
from workloads import gen

from . import _bounds as Bd
from ._parity import TOL_FP32, f64, rel

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _t(shape, sigma, tid, seed=13):
    return gen.normal(shape, sigma, tensor_id=tid, seed=seed, dtype=torch.float32)


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert T.tpl_get_device_status() == 0


CASES = [
    # M, H, I, tp, act, biases, residual
    (32, 256, 1024, 4, "gelu_tanh", False, None),       # the tiny MLP's shape
    (37, 256, 1024, 2, "gelu_erf", True, "separate"),   # 3 token tiles, the last of 5 rows
    (5, 128, 2048, 16, "none", True, "alias"),          # slices of 128, one per rank
    (16, 512, 512, 1, "gelu_tanh", False, "alias"),     # tp 1: all slices in one shard
    (100, 64, 256, 8, "gelu_erf", True, None),          # slices of 16 columns
]


@pytest.mark.parametrize("case", CASES)
def test_tp_mlp_fp32_against_the_oracle(case):
    M, H, I, tp, act, biases, res = case
    x = _t((M, H), 1.0, 0)
    w1, w2 = _t((I, H), 0.05, 1), _t((H, I), 0.05, 2)
    b1 = _t((I,), 0.02, 3) if biases else None
    b2 = _t((H,), 0.02, 4) if biases else None
    part = O.partition_subparams([I], tp, 1)
    w2p = T.pack_row_weight(w2.to(DEV), list(part.shard_width))
    xd = x.to(DEV)
    if res == "alias":
        y = xd.clone()
        T.tpl_tp_mlp_fp32(xd, w1.to(DEV), w2p, tp, act, b1=_d(b1), b2=_d(b2), residual=y, y=y)
    else:
        y = T.tpl_tp_mlp_fp32(xd, w1.to(DEV), w2p, tp, act, b1=_d(b1), b2=_d(b2),
                              residual=xd if res == "separate" else None)
    torch.cuda.synchronize()
    # the oracle: column-parallel shards, activation, row-parallel partials summed
    hs = O.column_linear(f64(x), f64(w1), None if b1 is None else f64(b1), part)
    hs = [O.activation(h, act) for h in hs]
    ref = O.row_linear_reduce(hs, O.row_weight_slices(f64(w2), part.shard_width),
                              None if b2 is None else f64(b2),
                              f64(x) if res is not None else None)
    assert rel(y, ref) <= TOL_FP32
    h_ref, own_h, car_h = Bd.column(f64(x), f64(w1), None if b1 is None else f64(b1), part, act,
                                    simt=True)
    h_proxy = [Bd.stored(h, o, c, Bd.U_FP32) for h, o, c in zip(h_ref, own_h, car_h)]
    bref, own, car = Bd.row(h_ref, O.row_weight_slices(f64(w2), part.shard_width),
                            None if b2 is None else f64(b2),
                            f64(x) if res is not None else None, simt=True, h_proxy=h_proxy)
    Bd.check(f64(y), bref, own, car, u_out=Bd.U_FP32)


def _d(t):
    return None if t is None else t.to(DEV)


def test_tpmlp_falls_back_to_two_launches():
    # H 512, I 2048 needs more shared memory than the fused kernel has
    M, H, I, tp = 24, 512, 2048, 4
    x, w1, w2 = _t((M, H), 1.0, 0), _t((I, H), 0.05, 1), _t((H, I), 0.05, 2)
    with pytest.raises(T.TplError) as e:
        part = T.tpl_partition_subparams([I], tp, 1)
        T.tpl_tp_mlp_fp32(x.to(DEV), w1.to(DEV),
                          T.pack_row_weight(w2.to(DEV), [part.shard_width[r] for r in range(tp)]),
                          tp, "gelu_tanh")
    assert e.value.name == "TPL_ERR_UNSUPPORTED"
    blk = T.TPMLP(w1.to(DEV), w2.to(DEV), tp, "gelu_tanh", norm=False)
    y = blk(x.to(DEV))
    torch.cuda.synchronize()
    assert not blk.fused_fp32
    assert rel(y, O.tp_mlp(f64(x), f64(w1), f64(w2), tp, "gelu_tanh")) <= TOL_FP32


def test_tp_mlp_fp32_empty():
    w1, w2 = _t((1024, 256), 0.05, 1).to(DEV), _t((256, 1024), 0.05, 2).to(DEV)
    y = T.tpl_tp_mlp_fp32(torch.empty((0, 256), device=DEV), w1, w2, 4, "none")
    assert y.shape == (0, 256)
