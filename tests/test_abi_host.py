"""Host-side checks of libtpl.so that need no GPU.

The library loads, exports every symbol include/tpl.h declares, computes the
partition bit-exactly like the oracle, and rejects bad arguments on the host
with the documented status before touching CUDA.  Every call below that passes
a non-NULL fake pointer is one the host validation must reject, so nothing is
ever launched (these tests are also safe on a GPU machine).
"""
import ctypes
import os
import random
import re

import pytest

import oracle as O
import tensor_transformer_linear_b200 as T
from tensor_transformer_linear_b200 import _tpl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "tpl.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const char\*|tpl_status|uint64_t)\s+(tpl_\w+)\(",
                                 src, re.M)))


def test_library_exports_every_declared_symbol():
    L = T.lib()
    names = _declared()
    assert len(names) == 26, names
    for n in names:
        assert hasattr(L, n), n
    assert sorted(names) == sorted(_tpl.EXPORTED)


def test_status_strings():
    for code, name in _tpl.STATUS.items():
        assert T.tpl_status_string(code).startswith(name)


def _oracle_kind(subs, tp, align):
    try:
        return O.partition_subparams(subs, tp, align)
    except O.OracleError as e:
        return e.kind


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_partition_bit_exact_against_oracle(seed):
    rng = random.Random(seed)
    cases = [([4096, 1024, 1024], 8, 128), ([1024], 4, 1), ([14336], 8, 1), ([28672], 8, 1),
             ([128256], 8, 1)]
    for _ in range(300):
        n = rng.randint(1, 4)
        align = rng.choice([1, 2, 8, 128])
        cases.append(([align * rng.randint(1, 40) for _ in range(n)], rng.randint(1, 12), align))
    for subs, tp, align in cases:
        ref = _oracle_kind(subs, tp, align)
        if isinstance(ref, str):
            with pytest.raises(T.TplError) as e:
                T.tpl_partition_subparams(subs, tp, align)
            assert e.value.name == "TPL_ERR_" + ref, (subs, tp, align)
            continue
        got = T.tpl_partition_subparams(subs, tp, align).as_lists()
        assert got["width"] == ref.width
        assert got["src_off"] == ref.src_off
        assert got["dst_off"] == ref.dst_off
        assert got["shard_width"] == ref.shard_width
        assert got["shard_base"] == ref.shard_base


def test_partition_argument_errors():
    L = T.lib()
    p = _tpl.Partition()
    arr = (ctypes.c_int64 * 2)(8, 8)
    assert L.tpl_partition_subparams(None, 2, 2, 1, ctypes.byref(p)) == 1
    assert L.tpl_partition_subparams(arr, 2, 2, 1, None) == 1
    assert L.tpl_partition_subparams(arr, 0, 2, 1, ctypes.byref(p)) == 2
    assert L.tpl_partition_subparams(arr, 9, 2, 1, ctypes.byref(p)) == 2
    assert L.tpl_partition_subparams(arr, 2, 65, 1, ctypes.byref(p)) == 2
    assert L.tpl_partition_subparams(arr, 2, 2, 0, ctypes.byref(p)) == 2


FAKE = ctypes.c_void_p(0x10000)       # never dereferenced: every call below is rejected first
FAKE_ODD = ctypes.c_void_p(0x10001)


def test_column_linear_rejections():
    L = T.lib()
    p = T.tpl_partition_subparams([64, 32], 2, 8)
    s = ctypes.c_void_p(0)
    bp = ctypes.byref(p)
    assert L.tpl_column_linear(None, FAKE, 4, 64, FAKE, None, 1, 0, FAKE, s) == 1
    assert L.tpl_column_linear(bp, None, 4, 64, FAKE, None, 1, 0, FAKE, s) == 1
    assert L.tpl_column_linear(bp, FAKE, 4, 64, FAKE, None, 7, 0, FAKE, s) == 4   # dtype
    assert L.tpl_column_linear(bp, FAKE, 4, 64, FAKE, None, 1, 9, FAKE, s) == 4   # act
    assert L.tpl_column_linear(bp, FAKE, -1, 64, FAKE, None, 1, 0, FAKE, s) == 2
    assert L.tpl_column_linear(bp, FAKE, 4, 0, FAKE, None, 1, 0, FAKE, s) == 2
    assert L.tpl_column_linear(bp, FAKE, 0, 64, FAKE, None, 1, 0, FAKE, s) == 0   # empty: no-op
    assert L.tpl_column_linear(bp, None, 0, 64, None, None, 1, 0, None, s) == 0
    assert L.tpl_column_linear(bp, FAKE, 4, 60, FAKE, None, 1, 0, FAKE, s) == 5   # K % 8
    assert L.tpl_column_linear(bp, FAKE_ODD, 4, 64, FAKE, None, 1, 0, FAKE, s) == 5
    assert L.tpl_column_linear(bp, FAKE, 4, 64, FAKE_ODD, None, 0, 0, FAKE, s) == 5  # fp32 align
    bad = _tpl.Partition()
    ctypes.memmove(ctypes.byref(bad), bp, ctypes.sizeof(p))
    bad.src_off[1][1] = 90                                       # past the fused weight
    assert L.tpl_column_linear(ctypes.byref(bad), FAKE, 4, 64, FAKE, None, 1, 0, FAKE, s) == 2
    bad.src_off[1][1] = p.src_off[1][1]
    bad.width[0][0] = 0
    assert L.tpl_column_linear(ctypes.byref(bad), FAKE, 4, 64, FAKE, None, 1, 0, FAKE, s) == 2


def test_row_linear_rejections():
    L = T.lib()
    s = ctypes.c_void_p(0)
    kw = (ctypes.c_int64 * 2)(64, 64)
    assert L.tpl_row_linear_reduce(None, kw, 2, 4, 8, FAKE, None, None, 1, FAKE, None, s) == 1
    assert L.tpl_row_linear_reduce(None, kw, 2, 0, 8, None, None, None, 1, None, None, s) == 0
    assert L.tpl_row_linear_reduce(FAKE, None, 2, 4, 8, FAKE, None, None, 1, FAKE, None, s) == 1
    assert L.tpl_row_linear_reduce(FAKE, kw, 0, 4, 8, FAKE, None, None, 1, FAKE, None, s) == 2
    assert L.tpl_row_linear_reduce(FAKE, kw, 2, 4, 0, FAKE, None, None, 1, FAKE, None, s) == 2
    assert L.tpl_row_linear_reduce(FAKE, kw, 2, 4, 8, FAKE, None, None, 3, FAKE, None, s) == 4
    assert L.tpl_row_linear_reduce(FAKE, kw, 2, 0, 8, FAKE, None, None, 1, FAKE, None, s) == 0
    kw_bad = (ctypes.c_int64 * 2)(64, 0)
    assert L.tpl_row_linear_reduce(FAKE, kw_bad, 2, 4, 8, FAKE, None, None, 1, FAKE, None, s) == 2
    kw_odd = (ctypes.c_int64 * 2)(64, 60)
    assert L.tpl_row_linear_reduce(FAKE, kw_odd, 2, 4, 8, FAKE, None, None, 1, FAKE, None, s) == 5
    assert L.tpl_row_linear_reduce(FAKE_ODD, kw, 2, 4, 8, FAKE, None, None, 1, FAKE, None, s) == 5


def test_rmsnorm_rejections():
    L = T.lib()
    s = ctypes.c_void_p(0)
    f = ctypes.c_float(1e-6)
    assert L.tpl_rmsnorm(None, 4, 8, None, 0, f, 1, FAKE, s) == 1
    assert L.tpl_rmsnorm(FAKE, 4, 8, None, 0, f, 1, None, s) == 1
    assert L.tpl_rmsnorm(FAKE, 4, 8, None, 0, f, 5, FAKE, s) == 4
    assert L.tpl_rmsnorm(FAKE, -1, 8, None, 0, f, 1, FAKE, s) == 2
    assert L.tpl_rmsnorm(FAKE, 4, 0, None, 0, f, 1, FAKE, s) == 2
    assert L.tpl_rmsnorm(FAKE, 4, 8, None, 0, ctypes.c_float(-1.0), 1, FAKE, s) == 2
    assert L.tpl_rmsnorm(FAKE, 0, 8, None, 0, f, 1, FAKE, s) == 0
    assert L.tpl_rmsnorm(None, 0, 8, None, 0, f, 1, None, s) == 0
    assert L.tpl_rmsnorm(FAKE_ODD, 4, 8, None, 0, f, 1, FAKE, s) == 5


def test_lmhead_layout_and_rejections():
    # the layout rule is the oracle's (LMHead1D.from_model_args with tile 1)
    for V, tp, n in [(128256, 8, 4), (32000, 8, 3), (10, 4, 2), (72, 8, 4), (9, 8, 1), (1, 1, 1)]:
        try:
            O.vocab_layout(V, tp, n)
            ok = True
        except O.OracleError:
            ok = False
        if ok:
            assert T.tpl_lmhead_workspace_size(32, V, tp, n) >= tp * 32 * 8 + 4
        else:
            with pytest.raises(T.TplError) as e:
                T.tpl_lmhead_workspace_size(32, V, tp, n)
            assert e.value.name == "TPL_ERR_SHAPE"
    L = T.lib()
    s = ctypes.c_void_p(0)
    n = T.tpl_lmhead_workspace_size(32, 1000, 4, 2)
    args = lambda **kw: [kw.get("x", FAKE), kw.get("B", 32), kw.get("K", 64), kw.get("w", FAKE),
                         kw.get("V", 1000), kw.get("tp", 4), kw.get("nc", 2), None, FAKE, FAKE,
                         FAKE, kw.get("ws", FAKE), kw.get("wsb", n), s]
    assert L.tpl_lmhead_argmax(*args(x=None)) == 1
    assert L.tpl_lmhead_argmax(*args(ws=None)) == 1
    assert L.tpl_lmhead_argmax(*args(B=0)) == 2
    assert L.tpl_lmhead_argmax(*args(B=257)) == 2
    assert L.tpl_lmhead_argmax(*args(nc=0)) == 2
    assert L.tpl_lmhead_argmax(*args(V=72, tp=8, nc=4)) == 2
    assert L.tpl_lmhead_argmax(*args(wsb=n - 1)) == 2
    assert L.tpl_lmhead_argmax(*args(K=60)) == 5
    assert L.tpl_lmhead_argmax(*args(w=FAKE_ODD)) == 5


def test_next_rows_rejections():
    L = T.lib()
    s = ctypes.c_void_p(0)
    kw = (ctypes.c_int64 * 4)(64, 64, 64, 64)
    # seq not divisible by tp
    assert L.tpl_row_linear_reduce_scatter(FAKE, kw, 4, 2, 10, 8, FAKE, None, None, 1, FAKE, s) == 3
    assert L.tpl_row_linear_reduce_scatter(FAKE, None, 4, 2, 8, 8, FAKE, None, None, 1, FAKE, s) == 1
    assert L.tpl_row_linear_reduce_scatter(FAKE, kw, 4, 0, 8, 8, FAKE, None, None, 1, FAKE, s) == 2
    p = T.tpl_partition_subparams([256], 4, 1)
    bp = ctypes.byref(p)
    assert L.tpl_column_linear_allgather(bp, FAKE, 2, 6, 64, FAKE, None, 1, 0, FAKE, s) == 3
    assert L.tpl_column_linear_allgather(bp, FAKE, 2, 64, 64, FAKE, None, 1, 0, FAKE, s) == 8
    assert L.tpl_column_linear_allgather(None, FAKE, 2, 64, 64, FAKE, None, 1, 0, FAKE, s) == 1
    # SwiGLU: bf16 only; ranks without rows; bad sizes
    assert L.tpl_swiglu_column_linear(FAKE, 4, 64, FAKE, 256, 4, 0, FAKE, s) == 8
    assert L.tpl_swiglu_column_linear(FAKE, 4, 64, FAKE, 2, 4, 1, FAKE, s) == 3
    assert L.tpl_swiglu_column_linear(FAKE, 4, 60, FAKE, 256, 4, 1, FAKE, s) == 5
    assert L.tpl_swiglu_column_linear(None, 0, 64, None, 256, 4, 1, None, s) == 0
    # embedding
    assert L.tpl_embedding_lookup(FAKE, -1, FAKE, 10, 8, 2, 1, FAKE, s) == 2
    assert L.tpl_embedding_lookup(None, 0, None, 10, 8, 2, 1, None, s) == 0
    assert L.tpl_embedding_lookup(FAKE, 4, FAKE, 10, 8, 65, 1, FAKE, s) == 2
    assert L.tpl_embedding_lookup(FAKE, 4, FAKE_ODD, 10, 8, 2, 1, FAKE, s) == 5


def test_multi_gpu_rows_rejections():
    L = T.lib()
    s = ctypes.c_void_p(0)
    peers = (ctypes.c_void_p * 2)(FAKE, FAKE)
    assert L.tpl_row_linear_scatter(FAKE, 64, 2, 8, 16, FAKE, 0, 2, None, s) == 1
    assert L.tpl_row_linear_scatter(FAKE, 64, 2, 7, 16, FAKE, 0, 2, peers, s) == 3   # seq % tp
    assert L.tpl_row_linear_scatter(FAKE, 64, 2, 8, 16, FAKE, 2, 2, peers, s) == 2   # rank
    assert L.tpl_row_linear_scatter(FAKE, 60, 2, 8, 16, FAKE, 0, 2, peers, s) == 5   # K % 8
    assert L.tpl_row_linear_scatter(None, 64, 2, 8, 16, FAKE, 0, 2, peers, s) == 1
    assert L.tpl_row_linear_scatter(FAKE, 64, 2, 8, 16, FAKE, 0, 2,
                                    (ctypes.c_void_p * 2)(FAKE, None), s) == 1
    assert L.tpl_row_linear_scatter(FAKE, 64, 2, 8, 16, FAKE, 0, 2,
                                    (ctypes.c_void_p * 2)(FAKE, FAKE_ODD), s) == 5
    pr = T.tpl_partition_subparams([256], 1, 1)
    xs = (ctypes.c_void_p * 2)(FAKE, FAKE)
    gather = L.tpl_column_linear_gather
    assert gather(ctypes.byref(pr), None, 2, 2, 256, 64, FAKE, None, 0, FAKE, s) == 1
    assert gather(ctypes.byref(pr), xs, 2, 2, 255, 64, FAKE, None, 0, FAKE, s) == 3   # seq % tp
    assert gather(ctypes.byref(pr), xs, 2, 2, 128, 64, FAKE, None, 0, FAKE, s) == 8   # seg % 128
    assert gather(ctypes.byref(pr), xs, 17, 2, 17 * 128, 64, FAKE, None, 0, FAKE, s) == 8
    assert gather(ctypes.byref(pr), xs, 2, 2, 256, 60, FAKE, None, 0, FAKE, s) == 5  # K % 8
    assert gather(ctypes.byref(pr), (ctypes.c_void_p * 2)(FAKE, FAKE_ODD), 2, 2, 256, 64, FAKE,
                  None, 0, FAKE, s) == 5
    assert gather(ctypes.byref(pr), xs, 2, 2, 256, 64, FAKE, None, 7, FAKE, s) == 4  # act
    assert L.tpl_reduce_slots(FAKE, 0, 4, 8, None, None, FAKE, s) == 2
    assert L.tpl_reduce_slots(None, 2, 0, 8, None, None, None, s) == 0
    assert L.tpl_reduce_slots(None, 2, 4, 8, None, None, FAKE, s) == 1
    assert L.tpl_reduce_slots(FAKE, 2, 4, 8, None, None, FAKE_ODD, s) == 5
    assert L.tpl_reduce_slots(FAKE, 8, 2**60, 2**10, None, None, FAKE, s) == 2   # overflow
    ag = L.tpl_reduce_slots_allgather
    ys = (ctypes.c_void_p * 2)(FAKE, FAKE)
    assert ag(FAKE, 0, 2, 8, 16, None, None, 0, ys, s) == 2                 # tp
    assert ag(FAKE, 2, 2, 7, 16, None, None, 0, ys, s) == 3                 # seq % tp
    assert ag(FAKE, 2, 2, 8, 16, None, None, 2, ys, s) == 2                 # rank
    assert ag(FAKE, 2, 2, 8, 0, None, None, 0, ys, s) == 2                  # N
    assert ag(None, 2, 2, 8, 16, None, None, 0, ys, s) == 1
    assert ag(FAKE, 2, 2, 8, 16, None, None, 0, None, s) == 1
    assert ag(FAKE, 2, 2, 8, 16, None, None, 0, (ctypes.c_void_p * 2)(FAKE, None), s) == 1
    assert ag(FAKE, 2, 2, 8, 16, None, None, 1, (ctypes.c_void_p * 2)(FAKE_ODD, FAKE), s) == 5
    assert ag(FAKE, 2, 2, 8, 16, None, FAKE_ODD, 0, ys, s) == 5
    assert L.tpl_argmax_merge(FAKE, FAKE, 2, 0, 10, FAKE, s) == 2
    assert L.tpl_argmax_merge(FAKE, FAKE, 8, 4, 2**29, FAKE, s) == 2
    assert L.tpl_argmax_merge(None, FAKE, 2, 4, 10, FAKE, s) == 1
    assert L.tpl_argmax_merge(FAKE, FAKE, 2, 4, 10, FAKE_ODD, s) == 5


def test_selftest_rejections():
    L = T.lib()
    assert L.tpl_selftest_wait_timeout(0, None, None) == 2
    assert L.tpl_selftest_wait_timeout(2_000_000_000, None, None) == 2
    assert L.tpl_selftest_wait_timeout(1000, FAKE_ODD, None) == 5


def test_trace_set_rejections():
    L = T.lib()
    assert L.tpl_trace_set(FAKE, 0) == 2                # capacity out of range
    assert L.tpl_trace_set(FAKE, 2**32) == 2
    assert L.tpl_trace_set(FAKE_ODD, 16) == 5           # not 16-byte aligned


def test_reduce_slots_rmsnorm_rejections():
    L = T.lib()
    s = None
    assert L.tpl_reduce_slots_rmsnorm(FAKE, 0, 4, 64, None, None, FAKE, None, 0, 1e-6, FAKE, s) == 2
    assert L.tpl_reduce_slots_rmsnorm(FAKE, 2, 4, 64, None, None, FAKE, None, 0, -1.0, FAKE, s) == 2
    assert L.tpl_reduce_slots_rmsnorm(FAKE, 2, 4, 64, None, None, FAKE, None, 0, 1e-6, None, s) == 1
    assert L.tpl_reduce_slots_rmsnorm(FAKE, 2, 4, 60, None, None, FAKE, None, 0, 1e-6, FAKE, s) == 5
    assert L.tpl_reduce_slots_rmsnorm(FAKE, 2, 4, 64, None, None, FAKE, FAKE_ODD, 0, 1e-6, FAKE,
                                      s) == 5
    assert L.tpl_reduce_slots_rmsnorm(FAKE, 2, 4, 16392, None, None, FAKE, None, 0, 1e-6, FAKE,
                                      s) == 8
    assert L.tpl_reduce_slots_rmsnorm(None, 2, 0, 64, None, None, None, None, 0, 1e-6, None, s) == 0


def test_tp_mlp_fp32_rejections():
    L = T.lib()
    s = None
    ok = dict(M=32, H=256, I=1024, tp=4, act=2)

    def call(x=FAKE, w1=FAKE, w2=FAKE, y=FAKE, **kw):
        a = dict(ok, **kw)
        return L.tpl_tp_mlp_fp32(x, a["M"], a["H"], w1, None, a["I"], a["tp"], a["act"], w2,
                                 None, None, y, s)
    assert call(act=3) == 4                     # unknown activation
    assert call(M=-1) == 2 and call(H=0) == 2
    assert call(tp=3) == 3                      # 1024 % 3
    assert call(tp=3, I=960) == 8               # 16 % 3: slices would straddle shards
    assert call(H=250) == 8                     # H % 16
    assert call(I=1040) == 8                    # I % 64
    assert call(H=512, I=2048) == 8             # shared memory above 227 KB
    assert call(M=16 * 65536) == 2              # more token tiles than grid.y holds
    assert call(M=0, x=None, w1=None, w2=None, y=None) == 0
    assert call(x=None) == 1
    assert call(y=FAKE_ODD) == 5
