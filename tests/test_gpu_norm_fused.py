"""RMSNorm fused into the column-parallel GEMM (tpl_fold_norm_scale +
tpl_column_linear_rmsnorm), against the unchanged oracle, which normalises
first (google-research allgather_layernorm) and then runs the column linear.

The fold is checked bit for bit against the same fp32 product rounded on the
host; the fused linear on ragged shapes (M and K tails, fused pieces, bias,
both GELU forms, the single-CTA and CTA-pair kernels, with and without the
centred scale), on the RMSNorm + TP MLP block at full size and through two
layers of the residual stack.  The element-wise bound is the unfused path's:
rounding g into the weight once carries the same first-order error as
rounding the normalised x to bf16 (sum_k xn_k^2 (u W_k)^2 either way)."""
import numpy as np
import pytest
import torch

import oracle as O
import tensor_transformer_linear_b200 as T
from workloads import configs as C
from workloads import gen

from . import _bounds as Bd
from ._parity import TOL_BF16, f64, rel

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _t(shape, sigma, tid, dtype=torch.bfloat16, seed=9):
    return gen.normal(shape, sigma, tensor_id=tid, seed=seed, dtype=dtype)


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert T.tpl_get_device_status() == 0


@pytest.mark.parametrize("centered", [True, False])
def test_fold_is_the_rounded_fp32_product(centered):
    w = _t((300, 264), 0.05, 1)
    s = _t((264,), 0.1, 4, torch.float32)
    got = T.tpl_fold_norm_scale(w.to(DEV), s.to(DEV), centered)
    g = s + 1.0 if centered else s
    ref = (w.float() * g).to(torch.bfloat16)
    assert torch.equal(got.cpu(), ref)
    wd = w.to(DEV)
    T.tpl_fold_norm_scale(wd, s.to(DEV), centered, out=wd)       # in place
    assert torch.equal(wd.cpu(), ref)


CASES = [
    # subs, tp, align, M, K, bias, act, scale
    ([1024], 4, 1, 600, 512, False, "gelu_erf", "centered"),       # CTA pairs, M tail
    ([512, 128, 128], 4, 32, 100, 264, True, "none", "plain"),     # single CTA, K tail
    ([2048], 8, 1, 4096, 1024, True, "gelu_tanh", None),           # several waves, no scale
    ([14336], 8, 1, 1024, 4096, False, "gelu_erf", "centered"),    # the MLP's c_fc shape
]


@pytest.mark.parametrize("case", CASES)
def test_fused_rmsnorm_column_linear(case):
    subs, tp, align, M, K, with_bias, act, mode = case
    part = O.partition_subparams(subs, tp, align)
    x = _t((M, K), 1.0, 0)
    w = _t((sum(subs), K), 0.02, 1)
    b = _t((sum(subs),), 0.02, 3) if with_bias else None
    s = _t((K,), 0.1, 4, torch.float32) if mode else None
    p = T.tpl_partition_subparams(subs, tp, align)
    wd = w.to(DEV)
    if s is not None:
        wd = T.tpl_fold_norm_scale(wd, s.to(DEV), mode == "centered")
    ws = T.rmsnorm_linear_workspace(M, DEV)
    y = None
    for _ in range(2):           # the workspace is reused without clearing
        y = T.tpl_column_linear_rmsnorm(p, x.to(DEV), wd, b.to(DEV) if b is not None else None,
                                        1e-6, act, ws)
    torch.cuda.synchronize()
    xn, own_n = Bd.rmsnorm(f64(x), None if s is None else f64(s), mode == "centered")
    ref, own, car = Bd.column(xn, f64(w), None if b is None else f64(b), part, act,
                              x_proxy=Bd.stored(xn, own_n, None, Bd.U_BF16))
    for r_, (g, r, e, c) in enumerate(zip(T.shard_views(y, p, M), ref, own, car)):
        assert rel(g, r) <= TOL_BF16, r_
        Bd.check(f64(g), r, e, c, what=f"rank {r_}")


def test_fused_rmsnorm_tp_mlp_full_size():
    w = C.TP_MLP
    x = C.mlp_x(w, DEV)
    s = C.mlp_scale(w, 0, DEV)
    blk = T.TPMLP(C.mlp_w1(w, 0, DEV), C.mlp_w2(w, 0, DEV), w.tp, w.act, scale=s,
                  centered=True, norm=True, fused_norm=True)
    y = blk(x)
    torch.cuda.synchronize()
    rows = sorted({0, 1, w.M // 2, w.M - 1} | set(range(97, w.M, 571)))
    xr = gen.rows((w.M, w.hidden), rows, 1.0, tensor_id=gen.TID_X)
    ref, own, car = Bd.mlp(f64(xr), f64(C.mlp_w1(w)), f64(C.mlp_w2(w)), w.tp, w.act,
                           scale=f64(C.mlp_scale(w)), centered=True, norm=True)
    assert rel(y[rows], ref) <= TOL_BF16
    Bd.check(f64(y[rows]), ref, own, car)


def test_fused_rmsnorm_residual_stack():
    # x <- x + MLP(RMSNorm(x)), two layers, fused norm, residual in place
    M, H, I, tp = 2048, 1024, 4096, 8
    x = _t((M, H), 1.0, 0)
    layers = [(_t((I, H), 0.02, 1 + 16 * l), _t((H, I), 0.02, 2 + 16 * l)) for l in range(2)]
    xd = x.to(DEV)
    stack = T.TPStack([T.TPMLP(w1.to(DEV), w2.to(DEV), tp, "gelu_erf", norm=True,
                               residual=True, fused_norm=True) for w1, w2 in layers])
    stack(xd)
    torch.cuda.synchronize()
    rows = sorted({0, M // 2, M - 1} | set(range(50, M, 211)))
    ref, own, car = Bd.stack(f64(x)[rows], [(f64(a), f64(b)) for a, b in layers], tp,
                             "gelu_erf")
    got = f64(xd)[rows]
    assert rel(got, ref) <= TOL_BF16
    Bd.check(got, ref, own, car)
    plain = x.to(DEV)
    T.TPStack([T.TPMLP(w1.to(DEV), w2.to(DEV), tp, "gelu_erf", norm=True, residual=True)
               for w1, w2 in layers])(plain)
    torch.cuda.synchronize()
    assert rel(f64(xd), f64(plain)) <= TOL_BF16     # the fused and unfused paths agree


def test_fused_rmsnorm_rejects_a_short_workspace():
    p = T.tpl_partition_subparams([256], 2, 1)
    x = torch.zeros((300, 64), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((256, 64), dtype=torch.bfloat16, device=DEV)
    ws = T.rmsnorm_linear_workspace(100, DEV)         # sized for 100 rows
    with pytest.raises(T.TplError) as e:
        T.tpl_column_linear_rmsnorm(p, x, w, None, 1e-6, "none", ws)
    assert e.value.name == "TPL_ERR_SHAPE"
