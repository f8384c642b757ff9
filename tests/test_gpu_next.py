"""GPU parity of the next rows against the fp64 oracle: sequence-parallel
reduce-scatter / all-gather linears, the fused SwiGLU column linear and the
vocab-sharded embedding lookup (small and ragged shapes, both GEMM kernels)."""
import numpy as np
import pytest
import torch

import oracle as O
import tensor_transformer_linear_b200 as T
from workloads import gen

from . import _bounds as Bd
from ._parity import TOL_BF16, TOL_FP32, f64, rel

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _t(shape, sigma, tid, dtype=torch.bfloat16, seed=3):
    return gen.normal(shape, sigma, tensor_id=tid, seed=seed, dtype=dtype)


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert T.tpl_get_device_status() == 0


@pytest.mark.parametrize("dtype,tp,batch,seq,kr,N,with_bias,with_res", [
    (torch.bfloat16, 4, 2, 256, 64, 300, True, True),
    (torch.bfloat16, 8, 2, 512, 256, 512, False, True),
    (torch.bfloat16, 2, 3, 10, 72, 40, True, False),       # M = 30: single-CTA kernel
    (torch.float32, 3, 2, 12, 16, 20, True, True),
])
def test_row_linear_reduce_scatter(dtype, tp, batch, seq, kr, N, with_bias, with_res):
    k_w = [kr] * tp
    M = batch * seq
    h = _t((M, kr * tp), 1.0, 5, dtype)
    w2 = _t((N, kr * tp), 0.05, 2, dtype)
    b = _t((N,), 0.05, 3, dtype) if with_bias else None
    res = _t((tp, batch, seq // tp, N), 1.0, 6, dtype) if with_res else None
    y = T.tpl_row_linear_reduce_scatter(T.pack_row_weight(h, k_w).to(DEV), k_w, batch, seq,
                                        T.pack_row_weight(w2, k_w).to(DEV),
                                        None if b is None else b.to(DEV),
                                        None if res is None else res.to(DEV))
    torch.cuda.synchronize()
    ref = O.row_linear_reduce_scatter(O.row_weight_slices(f64(h), k_w),
                                      O.row_weight_slices(f64(w2), k_w), batch, seq,
                                      None if b is None else f64(b),
                                      None if res is None else f64(res))
    bf16 = dtype == torch.bfloat16
    assert rel(y, ref) <= (TOL_BF16 if bf16 else TOL_FP32)
    # element-wise, with the bound laid out like the output (rank-major slices)
    res_full = None if res is None else O.seq_gather(f64(res), batch, seq, tp)
    full, own, _ = Bd.row(O.row_weight_slices(f64(h), k_w), O.row_weight_slices(f64(w2), k_w),
                          None if b is None else f64(b), res_full, simt=not bf16)
    Bd.check(f64(y), O.seq_scatter(full, batch, seq, tp), O.seq_scatter(own, batch, seq, tp),
             u_out=Bd.U_BF16 if bf16 else Bd.U_FP32)


@pytest.mark.parametrize("dtype,subs,tp,batch,seq,K,act", [
    (torch.bfloat16, [512], 8, 2, 1024, 256, "gelu_erf"),     # 128-token slices
    (torch.bfloat16, [256, 128, 128], 2, 1, 256, 64, "none"), # fused pieces, one sequence
    (torch.float32, [30], 3, 2, 12, 16, "gelu_tanh"),
])
def test_column_linear_allgather(dtype, subs, tp, batch, seq, K, act):
    part = O.partition_subparams(subs, tp, 1)
    M = batch * seq
    x = _t((M, K), 1.0, 0, dtype)
    w = _t((sum(subs), K), 0.05, 1, dtype)
    x_sp = torch.from_numpy(O.seq_scatter(x.float().numpy(), batch, seq, tp)).to(dtype)
    p = T.tpl_partition_subparams(subs, tp, 1)
    y = T.tpl_column_linear_allgather(p, x_sp.contiguous().to(DEV), batch, seq, w.to(DEV), None,
                                      act)
    torch.cuda.synchronize()
    ref = O.column_linear_allgather(f64(x_sp), batch, seq, f64(w), None, part, act)
    bf16 = dtype == torch.bfloat16
    tol = TOL_BF16 if bf16 else TOL_FP32
    bref, own, _ = Bd.column(O.seq_gather(f64(x_sp), batch, seq, tp), f64(w), None, part, act,
                             simt=not bf16)
    for g, r, br, e in zip(T.shard_views(y, p, M), ref, bref, own):
        assert rel(g, r) <= tol
        Bd.check(f64(g), br, e, u_out=Bd.U_BF16 if bf16 else Bd.U_FP32)


def test_column_linear_allgather_needs_whole_tma_boxes_for_bf16():
    p = T.tpl_partition_subparams([256], 4, 1)
    x = torch.zeros((2 * 64, 64), dtype=torch.bfloat16, device=DEV)   # 16-token slices
    w = torch.zeros((256, 64), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(T.TplError) as e:
        T.tpl_column_linear_allgather(p, x, 2, 64, w)
    assert e.value.name == "TPL_ERR_UNSUPPORTED"


def test_sequence_parallel_block_round_trip():
    # x (rank-major) -> RMSNorm -> all-gather c_fc + GELU -> c_proj reduce-scatter + residual
    tp, batch, seq, H, I = 4, 2, 512, 256, 1024
    M = batch * seq
    x = _t((M, H), 1.0, 0)
    w1, w2 = _t((I, H), 0.05, 1), _t((H, I), 0.05, 2)
    x_sp = torch.from_numpy(O.seq_scatter(x.float().numpy(), batch, seq, tp)).to(torch.bfloat16)
    xd = x_sp.contiguous().to(DEV)
    xn = T.tpl_rmsnorm(xd.view(M, H))
    p = T.tpl_partition_subparams([I], tp, 1)
    k_w = [p.shard_width[r] for r in range(tp)]
    hbuf = T.tpl_column_linear_allgather(p, xn, batch, seq, w1.to(DEV), None, "gelu_erf")
    y = T.tpl_row_linear_reduce_scatter(hbuf, k_w, batch, seq,
                                        T.pack_row_weight(w2, k_w).to(DEV), None, xd)
    torch.cuda.synchronize()
    xs = f64(x_sp)
    xg = O.seq_gather(xs, batch, seq, tp)
    h_ref = O.column_linear(O.rmsnorm(xg), f64(w1), None, O.partition_subparams([I], tp, 1),
                            "gelu_erf")
    ref = O.row_linear_reduce_scatter(h_ref, O.row_weight_slices(f64(w2), k_w), batch, seq,
                                      None, xs)
    assert rel(y, ref) <= TOL_BF16
    full, own, car = Bd.mlp(xg, f64(w1), f64(w2), tp, "gelu_erf", norm=True, residual=True)
    Bd.check(f64(y), O.seq_scatter(full, batch, seq, tp), O.seq_scatter(own, batch, seq, tp),
             O.seq_scatter(car, batch, seq, tp))


@pytest.mark.parametrize("M,K,F,tp", [
    (300, 256, 1000, 4),      # ragged 128-column blocks per rank (250 columns)
    (64, 128, 2048, 8),       # single-CTA kernel
    (1024, 512, 4096, 8),     # CTA pairs, 512 columns per rank
    (129, 72, 24, 3),         # tiny ranks, K not a multiple of 64
])
def test_swiglu_column_linear(M, K, F, tp):
    x = _t((M, K), 1.0, 0)
    w = _t((2 * F, K), 0.05, 1)
    h = T.tpl_swiglu_column_linear(x.to(DEV), w.to(DEV), F, tp)
    torch.cuda.synchronize()
    ref, own = Bd.swiglu(f64(x), f64(w), F, tp)
    p = T.tpl_partition_subparams([F], tp, 1)
    for g, r, e in zip(T.shard_views(h, p, M), ref, own):
        assert rel(g, r) <= TOL_BF16
        Bd.check(f64(g), r, e)


def test_swiglu_rejects_fp32_and_indivisible():
    x = torch.zeros((4, 8), dtype=torch.float32, device=DEV)
    with pytest.raises(T.TplError) as e:
        T.tpl_swiglu_column_linear(x, torch.zeros((8, 8), device=DEV), 4, 2)
    assert e.value.name == "TPL_ERR_UNSUPPORTED"
    xb = torch.zeros((4, 8), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(T.TplError) as e:
        T.tpl_swiglu_column_linear(xb, torch.zeros((4, 8), dtype=torch.bfloat16, device=DEV), 2, 4)
    assert e.value.name == "TPL_ERR_INDIVISIBLE"


@pytest.mark.parametrize("dtype,V,H,tp", [
    (torch.bfloat16, 1000, 4096, 8),
    (torch.bfloat16, 37, 72, 4),
    (torch.float32, 11, 33, 4),        # odd width: scalar path
    (torch.float32, 128256, 64, 8),
])
def test_embedding_lookup(dtype, V, H, tp):
    table = _t((V, H), 1.0, 7, dtype)
    rng = np.random.default_rng(0)
    ids = np.concatenate([rng.integers(0, V, 200), [0, V - 1, -1, V, V + 17, -5]]).astype(np.int32)
    out = T.tpl_embedding_lookup(torch.from_numpy(ids).to(DEV), table.to(DEV), tp)
    torch.cuda.synchronize()
    ref = O.embedding_lookup(ids, f64(table), tp)
    np.testing.assert_array_equal(f64(out), ref)      # a copy or zeros: bit-exact
